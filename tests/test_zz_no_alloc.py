"""ss2d_selective_scan_fwd_noalloc: the S6 forward for callers that cannot allocate device memory.

Such callers (a serving loop whose memory plan is fixed at start-up, a host program
that links only the C library and has no device allocator of its own) get a forward
scan that keeps its scratch -- the per-segment summaries of a sequence split into
segments -- in a static buffer inside the library instead of a workspace.  These
tests call it through the C ABI and compare it with ss2d_selective_scan_fwd, twice
in a row so that a second call reusing the buffer is covered too.

The file is named to be collected last: if it fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import selective_scan_crossscan_b200 as ss
import ss2d_inputs

FWD_TOL = 1e-4  # |y - y_ref| <= 1e-4 (1 + |y_ref|), the forward tolerance of the parity tests
BF16_TOL = 1e-2  # relative L2 for bf16 inputs
OK, ERR_SHAPE = 0, 2


def _lib():
    from selective_scan_crossscan_b200 import _build
    _build.build()
    lib = ss._load()
    P = ctypes.c_void_p
    lib.ss2d_selective_scan_fwd_noalloc.argtypes = [ctypes.POINTER(ss.Desc), P, P, P, P, P, P, P, ctypes.c_int,
                                                   P, P, P]
    lib.ss2d_selective_scan_fwd_noalloc.restype = ctypes.c_int
    return lib


def _call_noalloc(lib, inp, out_dtype):
    u = inp["u"]
    Bn, Ch, L = u.shape
    out = torch.empty((Bn, Ch, L), dtype=out_dtype, device=u.device)
    desc = ss.Desc(Bn, Ch // 4, 1, L, inp["A"].shape[1], ss._code(u.dtype), ss._code(out_dtype))
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.ss2d_selective_scan_fwd_noalloc(ctypes.byref(desc), p(u), p(inp["delta"]), p(inp["A"]), p(inp["B"]),
                                             p(inp["C"]), p(inp["D"]), p(inp["delta_bias"]), 1, p(out), None, stream)
    assert st == OK, lib.ss2d_last_cuda_error()
    return out


def _reference(inp, out_dtype):
    return ss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                                 True, out_dtype=out_dtype)


@pytest.mark.gpu
def test_noalloc_matches_selective_scan_fwd_on_two_calls():
    assert torch.cuda.is_available()
    lib = _lib()
    # few sequences and long ones, so the sequences are split into segments and the static scratch is used
    cases = [(ss2d_inputs.custom(1, 8, 64, 64, 16, a_init="s4d_real"), 21),
             (ss2d_inputs.custom(2, 24, 40, 48, 16, dtype="bf16", a_init="s4d_real"), 22)]
    for w, seed in cases:
        inp = {k: v.cuda() for k, v in ss2d_inputs.make_scan_inputs(w, seed=seed).items()}
        ref = _reference(inp, w.torch_dtype).double().cpu().numpy()
        for call in range(2):
            y = _call_noalloc(lib, inp, w.torch_dtype)
            torch.cuda.synchronize()
            got = y.double().cpu().numpy()
            if w.dtype == "f32":
                excess = np.abs(got - ref) - FWD_TOL * (1.0 + np.abs(ref))
                assert excess.max() <= 0, (w.name, call, float(excess.max()))
            else:
                rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
                assert rel <= BF16_TOL, (w.name, call, rel)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 75,772 sequences of 4,096 steps split in two: 75772 * 2 segments * 32 floats * 4 B = 19.4 MB > 16 MiB.
    # The size check runs on the host before anything is launched (the pointers are never touched).
    lib = _lib()
    desc = ss.Desc(1, 18943, 1, 4096, 16, ss.F32, ss.F32)
    a = ctypes.c_void_p(0x100000)
    st = lib.ss2d_selective_scan_fwd_noalloc(ctypes.byref(desc), a, a, a, a, a, None, None, 1, a, None, None)
    assert st == ERR_SHAPE
    assert b"static scratch" in lib.ss2d_last_cuda_error()
