"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
symbol that include/ss2d.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

import selective_scan_crossscan_b200 as ss
from selective_scan_crossscan_b200 import Desc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ss2d.h")

OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_WORKSPACE, ERR_LAUNCH, ERR_TIMEOUT, ERR_DEVICE = range(9)


@pytest.fixture(scope="module")
def lib():
    from selective_scan_crossscan_b200 import _build
    _build.build()
    return ss._load()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"^SS2D_API\s+[\w\s\*]+?\b(ss2d_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for required in ("ss2d_cross_scan", "ss2d_cross_merge", "ss2d_selective_scan_fwd", "ss2d_selective_scan_bwd",
                     "ss2d_forward", "ss2d_backward", "ss2d_workspace_bytes", "ss2d_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name


def _d(B=1, D=8, H=8, W=8, N=4, i=0, o=0):
    return ctypes.byref(Desc(B, D, H, W, N, i, o))


A16 = ctypes.c_void_p(0x10000)  # aligned non-null fake device addresses (never dereferenced:
B16 = ctypes.c_void_p(0x20000)  # validation fails or the device check stops the call first)


def test_null_and_shape_errors(lib):
    assert lib.ss2d_cross_scan(None, A16, B16, None) == ERR_NULL
    assert lib.ss2d_cross_scan(_d(), None, B16, None) == ERR_NULL
    assert lib.ss2d_cross_merge(_d(), A16, None, None) == ERR_NULL
    for bad in (dict(B=0), dict(D=0), dict(H=0), dict(W=-1), dict(N=0), dict(N=17), dict(B=70000)):
        assert lib.ss2d_cross_scan(_d(**bad), A16, B16, None) == ERR_SHAPE, bad
    assert lib.ss2d_cross_scan(_d(i=7), A16, B16, None) == ERR_DTYPE
    assert lib.ss2d_cross_merge(_d(o=-1), A16, B16, None) == ERR_DTYPE


def test_alignment_errors(lib):
    mis = ctypes.c_void_p(0x10004)
    assert lib.ss2d_cross_scan(_d(), mis, B16, None) == ERR_ALIGN
    assert lib.ss2d_selective_scan_fwd(_d(), A16, A16, mis, A16, A16, None, None, 1, B16, None, None) == ERR_ALIGN


def test_scan_fwd_argument_errors(lib):
    f = lib.ss2d_selective_scan_fwd
    assert f(_d(), None, A16, A16, A16, A16, None, None, 1, B16, None, None) == ERR_NULL  # u
    assert f(_d(), A16, A16, None, A16, A16, None, None, 1, B16, None, None) == ERR_NULL  # A
    assert f(_d(), A16, A16, A16, A16, A16, None, None, 1, None, None, None) == ERR_NULL  # out


def test_backward_argument_errors(lib):
    g = lib.ss2d_selective_scan_bwd
    ws = lib.ss2d_workspace_bytes(_d(), ss.OP_SELECTIVE_SCAN_BWD)
    assert ws > 0
    args = [A16] * 5
    # D given but dD missing
    assert g(_d(), *args, A16, None, 1, A16, None, A16, A16, A16, A16, A16, None, None, A16, ws, None) == ERR_NULL
    # workspace too small
    assert g(_d(), *args, None, None, 1, A16, None, A16, A16, A16, A16, A16, None, None, A16, ws - 1,
             None) == ERR_WORKSPACE
    assert g(_d(), *args, None, None, 1, A16, None, A16, A16, A16, A16, A16, None, None, None, ws,
             None) == ERR_WORKSPACE
    fb = lib.ss2d_backward
    wsb = lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD)
    assert fb(_d(), *args, None, None, 1, A16, None, A16, A16, A16, A16, A16, None, None, A16, wsb - 64,
              None) == ERR_WORKSPACE
    ff = lib.ss2d_forward
    wsf = lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD)
    assert ff(_d(), *args, None, None, 1, B16, None, None, 0, None) == ERR_WORKSPACE
    assert ff(_d(), *args, None, None, 1, B16, None, A16, wsf - 1, None) == ERR_WORKSPACE


def test_gated_scan_argument_errors(lib):
    # ss2d_selective_scan_fwd_ex / _bwd_ex: z and last_state are optional but must be aligned;
    # dz must be given exactly when z is
    mis = ctypes.c_void_p(0x10004)
    f = lib.ss2d_selective_scan_fwd_ex
    args = [A16] * 5
    assert f(_d(), *args, None, mis, None, 1, B16, None, None, None) == ERR_ALIGN  # z
    assert f(_d(), *args, None, None, None, 1, B16, mis, None, None) == ERR_ALIGN  # last_state
    assert f(_d(), *args, None, A16, None, 1, None, A16, None, None) == ERR_NULL   # out
    g = lib.ss2d_selective_scan_bwd_ex
    ws = lib.ss2d_workspace_bytes(_d(), ss.OP_SELECTIVE_SCAN_BWD)
    grads = [A16] * 5  # du, ddelta, dA, dB, dC
    assert g(_d(), *args, None, A16, None, 1, A16, None, *grads, None, None, None, A16, ws, None) == ERR_NULL
    assert g(_d(), *args, None, None, None, 1, A16, None, *grads, None, None, A16, A16, ws, None) == ERR_NULL
    assert g(_d(), *args, None, mis, None, 1, A16, None, *grads, None, None, A16, A16, ws, None) == ERR_ALIGN
    assert g(_d(), *args, None, A16, None, 1, A16, None, *grads, None, None, A16, A16, ws - 1,
             None) == ERR_WORKSPACE


def test_bimamba_argument_errors(lib):
    f = lib.ss2d_bimamba_forward
    wsf = lib.ss2d_workspace_bytes(_d(H=1, W=37), ss.OP_BIMAMBA_FORWARD)
    wsb = lib.ss2d_workspace_bytes(_d(H=1, W=37), ss.OP_BIMAMBA_BACKWARD)
    assert 0 < wsf < wsb
    args = [A16] * 5  # x, delta, A, B, C
    # a sequence is a 1 x L image
    assert f(_d(H=2, W=37), *args, None, None, None, 1, B16, None, A16, wsf, None) == ERR_SHAPE
    assert f(_d(H=1, W=37), *args, None, None, None, 1, None, None, A16, wsf, None) == ERR_NULL
    assert f(_d(H=1, W=37), *args, None, None, None, 1, B16, None, A16, wsf - 1, None) == ERR_WORKSPACE
    assert f(_d(H=1, W=37), *args, None, ctypes.c_void_p(0x10004), None, 1, B16, None, A16, wsf,
             None) == ERR_ALIGN
    g = lib.ss2d_bimamba_backward
    grads = [A16] * 5  # dx, ddelta, dA, dB, dC
    # z given but dz missing, and the reverse
    assert g(_d(H=1, W=37), *args, None, A16, None, 1, A16, None, *grads, None, None, None, A16, wsb,
             None) == ERR_NULL
    assert g(_d(H=1, W=37), *args, None, None, None, 1, A16, None, *grads, None, None, A16, A16, wsb,
             None) == ERR_NULL
    assert g(_d(H=1, W=37), *args, None, A16, None, 1, A16, None, *grads, None, None, A16, A16, wsb - 1,
             None) == ERR_WORKSPACE


def test_path_table_argument_errors(lib):
    mis = ctypes.c_void_p(0x10004)
    assert lib.ss2d_path_tables(_d(), 2, A16, None) == ERR_SHAPE  # unknown path set
    assert lib.ss2d_path_tables(_d(), 1, None, None) == ERR_NULL
    assert lib.ss2d_path_tables(_d(), 1, mis, None) == ERR_ALIGN
    assert lib.ss2d_cross_scan_table(_d(), None, A16, B16, None) == ERR_NULL
    assert lib.ss2d_cross_merge_table(_d(), mis, A16, B16, None) == ERR_ALIGN
    f = lib.ss2d_forward_table
    wsf = lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD_TABLE)
    wsb = lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD_TABLE)
    assert wsf > lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD) and wsb > lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD)
    args = [A16] * 5
    assert f(_d(), A16, *args, None, None, 1, B16, None, A16, wsf - 1, None) == ERR_WORKSPACE
    assert f(_d(), None, *args, None, None, 1, B16, None, A16, wsf, None) == ERR_NULL


def test_forward_proj_argument_errors(lib):
    f = lib.ss2d_forward_proj
    ws = lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD_PROJ)
    assert ws > lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD)
    w = [A16, A16, A16, A16]  # x, x_proj_weight, dt_proj_weight, dt_proj_bias
    assert f(_d(), 0, *w, A16, None, 1, B16, B16, None, A16, ws, None) == ERR_SHAPE   # dt_rank 0
    assert f(_d(), 33, *w, A16, None, 1, B16, B16, None, A16, ws, None) == ERR_SHAPE  # dt_rank > 32
    assert f(_d(), 2, *w, A16, None, 1, B16, None, None, A16, ws, None) == ERR_NULL   # x_dbl
    assert f(_d(), 2, *w, A16, None, 1, B16, B16, None, A16, ws - 1, None) == ERR_WORKSPACE


def test_backward_proj_argument_errors(lib):
    f = lib.ss2d_backward_proj
    ws = lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD_PROJ)
    assert ws > lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD)
    w = [A16, A16, A16, A16, A16, A16]  # x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D
    g = [B16, B16, B16, B16, B16, B16]  # dx, dx_proj_weight, ddt_proj_weight, ddt_proj_bias, dA, dD
    ok = (1, A16, None, A16)            # softplus, x_dbl, chunk_states, dy
    assert f(_d(), 0, *w, *ok, *g, A16, ws, None) == ERR_SHAPE    # dt_rank 0
    assert f(_d(), 33, *w, *ok, *g, A16, ws, None) == ERR_SHAPE   # dt_rank > 32
    assert f(_d(), 2, *w, 1, None, None, A16, *g, A16, ws, None) == ERR_NULL  # x_dbl
    assert f(_d(), 2, *w, *ok, B16, B16, B16, None, B16, B16, A16, ws, None) == ERR_NULL  # bias without its grad
    assert f(_d(), 2, *w[:5], None, *ok, *g, A16, ws, None) == ERR_NULL  # dD without D
    assert f(_d(), 2, *w, *ok, *g, A16, ws - 1, None) == ERR_WORKSPACE


def test_proj_conv_argument_errors(lib):
    f, g = lib.ss2d_forward_proj_conv, lib.ss2d_backward_proj_conv
    wsf = lib.ss2d_workspace_bytes(_d(), ss.OP_FORWARD_PROJ_CONV)
    wsb = lib.ss2d_workspace_bytes(_d(), ss.OP_BACKWARD_PROJ_CONV)
    assert wsb > wsf > 0
    w = [A16] * 8  # x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D
    assert f(_d(), 0, 4, *w, 1, B16, B16, None, A16, wsf, None) == ERR_SHAPE   # dt_rank 0
    assert f(_d(), 2, 0, *w, 1, B16, B16, None, A16, wsf, None) == ERR_SHAPE   # d_conv 0
    assert f(_d(), 2, 5, *w, 1, B16, B16, None, A16, wsf, None) == ERR_SHAPE   # d_conv 5
    assert f(_d(), 2, 4, A16, None, *w[2:], 1, B16, B16, None, A16, wsf, None) == ERR_NULL  # conv_weight
    assert f(_d(), 2, 4, *w, 1, B16, B16, None, A16, wsf - 1, None) == ERR_WORKSPACE
    gr = [B16] * 8  # dx, dconv_weight, dconv_bias, dx_proj_weight, ddt_proj_weight, ddt_proj_bias, dA, dD
    assert g(_d(), 2, 4, *w, 1, A16, None, A16, *gr, A16, wsb - 1, None) == ERR_WORKSPACE
    assert g(_d(), 2, 4, *w, 1, A16, None, A16, gr[0], gr[1], None, *gr[3:], A16, wsb, None) == ERR_NULL  # conv bias
    assert g(_d(), 2, 5, *w, 1, A16, None, A16, *gr, A16, wsb, None) == ERR_SHAPE


def test_valid_call_without_gpu_reports_device_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.ss2d_cross_scan(_d(), A16, B16, None) == ERR_DEVICE
    assert b"device" in lib.ss2d_last_cuda_error()


def test_workspace_and_chunk_state_sizes(lib):
    # chunk states: B * 4D * ceil(L / 16) * N fp32
    assert lib.ss2d_chunk_states_elems(_d(B=2, D=3, H=5, W=13, N=7)) == 2 * 12 * 5 * 7
    assert lib.ss2d_chunk_states_elems(_d(B=1, D=8, H=8, W=8, N=4)) == 32 * 4 * 4
    # the fused forward keeps one fp32 value per sequence step
    assert lib.ss2d_workspace_bytes(_d(B=2, D=3, H=5, W=13, N=7), ss.OP_FORWARD) >= 2 * 12 * 65 * 4
    assert lib.ss2d_workspace_bytes(_d(), 99) == ctypes.c_size_t(-1).value
    assert lib.ss2d_workspace_bytes(_d(N=0), ss.OP_FORWARD) == ctypes.c_size_t(-1).value


def test_status_strings(lib):
    for code in range(9):
        s = lib.ss2d_status_string(code).decode()
        assert s.startswith("SS2D_")
    assert b"unknown" in lib.ss2d_status_string(42)


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 2, 3, 3)
    with pytest.raises(ValueError):
        ss.cross_scan(x)


def test_binding_has_no_cpu_fallback():
    # the package holds no PyTorch re-implementation of the scan: every entry point calls the library
    src = open(os.path.join(ROOT, "selective_scan_crossscan_b200", "__init__.py")).read()
    for forbidden in ("torch.exp(", "torch.cumsum", "import oracle", "from oracle"):
        assert forbidden not in src
