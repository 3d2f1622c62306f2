"""selective_scan_crossscan_b200 -- VMamba's 2D selective scan (SS2D) on B200 (sm_100a).

A thin Python binding over the C ABI of ``libss2d.so`` (declared in
``include/ss2d.h``).  This module only marshals arguments: it makes tensors
contiguous, allocates outputs and workspaces with PyTorch, and passes raw device
pointers and the current CUDA stream.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback -- if the library is
missing or the device is not an sm_100 GPU, the calls raise.

Steps ("VMamba: Visual State Space Model", section "2D Selective Scan (SS2D) for
visual data", Fig. 2; the S6 arithmetic follows selective_scan_ref on
"vision mamba-yolov8", section "2. Vmamba module code"):

* ``cross_scan(x)``: (B, D, H, W) -> (B, 4, D, L): row-major, column-major, both reversed
* ``selective_scan_fwd(u, delta, A, B, C, ...)``: S6 forward over (B, 4D, L) sequences,
  with the optional output gate ``z`` (out * silu(z)) and the last state
* ``selective_scan_bwd(...)``: its gradients (and dz)
* ``selective_scan_fn``: the differentiable scan with selective_scan_fn's arguments
* ``cross_merge(ys, H, W)``: (B, 4, D, L) -> (B, D, H, W), (y0 + y2) + (y1 + y3)
* ``ss2d_forward`` / ``ss2d_backward``: the fused SS2D forward and backward
* ``SS2DFunction``: a torch.autograd.Function around the fused pair
* ``bimamba_forward`` / ``bimamba_backward`` / ``bimamba_scan``: the bidirectional scan of
  bimamba_inner_ref (a sequence and its reverse with A and A_b, outputs added)
* ``path_tables`` and the ``*_table`` calls: the same steps over another path set, e.g. the
  diagonal scans of "Visual Mamba实战从零开始搭建图像分类模型附PyTorch代码" (section 3)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "SS2DError", "cross_scan", "cross_merge", "selective_scan_fwd", "selective_scan_bwd", "selective_scan_fn",
    "SelectiveScanFunction", "ss2d_forward", "bimamba_forward", "bimamba_backward", "BiMambaFunction",
    "bimamba_scan", "path_tables", "cross_scan_table", "cross_merge_table", "ss2d_forward_table",
    "ss2d_backward_table", "PATHS_CROSS", "PATHS_DIAGONAL", "ss2d_forward_proj", "ss2d_backward_proj", "OP_BACKWARD_PROJ",
    "ss2d_forward_proj_conv", "ss2d_backward_proj_conv", "OP_FORWARD_PROJ_CONV", "OP_BACKWARD_PROJ_CONV",
    "ss2d_proj", "SS2DProjFunction",
    "ss2d_backward", "SS2DFunction", "ss2d", "workspace_bytes", "chunk_states_elems", "launch_count",
    "library_path", "CHUNK_LEN", "trace_events",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# SS2D_LIBRARY may point at another build of the same library (e.g. a tuning variant)
_LIB_PATH = os.environ.get("SS2D_LIBRARY") or os.path.join(_HERE, "libss2d.so")
_lock = threading.Lock()
_lib = None

CHUNK_LEN = 16  # SS2D_CHUNK_LEN
F32, BF16 = 0, 1
OP_SELECTIVE_SCAN_BWD, OP_FORWARD, OP_BACKWARD, OP_BIMAMBA_FORWARD, OP_BIMAMBA_BACKWARD = 1, 2, 3, 4, 5
OP_FORWARD_TABLE, OP_BACKWARD_TABLE, OP_FORWARD_PROJ, OP_BACKWARD_PROJ = 6, 7, 8, 9
OP_FORWARD_PROJ_CONV, OP_BACKWARD_PROJ_CONV = 10, 11
PATHS_CROSS, PATHS_DIAGONAL = 0, 1
_STATUS = {0: "SS2D_OK", 1: "SS2D_ERR_NULL", 2: "SS2D_ERR_SHAPE", 3: "SS2D_ERR_DTYPE", 4: "SS2D_ERR_ALIGN",
           5: "SS2D_ERR_WORKSPACE", 6: "SS2D_ERR_LAUNCH", 7: "SS2D_ERR_TIMEOUT", 8: "SS2D_ERR_DEVICE"}


class SS2DError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {_STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("height", ctypes.c_int64),
                ("width", ctypes.c_int64), ("d_state", ctypes.c_int64), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m selective_scan_crossscan_b200._build` (needs nvcc)")
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        D = ctypes.POINTER(Desc)
        i = ctypes.c_int
        sz = ctypes.c_size_t
        lib.ss2d_cross_scan.argtypes = [D, P, P, P]
        lib.ss2d_cross_merge.argtypes = [D, P, P, P]
        lib.ss2d_selective_scan_fwd.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P]
        lib.ss2d_selective_scan_bwd.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P, sz, P]
        lib.ss2d_selective_scan_fwd_ex.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, P]
        lib.ss2d_selective_scan_bwd_ex.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P,
                                                   P, sz, P]
        lib.ss2d_forward.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P, sz, P]
        lib.ss2d_bimamba_forward.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, sz, P]
        lib.ss2d_path_tables.argtypes = [D, i, P, P]
        lib.ss2d_forward_proj.argtypes = [D, i, P, P, P, P, P, P, i, P, P, P, P, sz, P]
        lib.ss2d_backward_proj.argtypes = [D, i, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P, sz, P]
        lib.ss2d_forward_proj_conv.argtypes = [D, i, i, P, P, P, P, P, P, P, P, i, P, P, P, P, sz, P]
        lib.ss2d_backward_proj_conv.argtypes = [D, i, i, P, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P,
                                                P, P, sz, P]
        lib.ss2d_cross_scan_table.argtypes = [D, P, P, P, P]
        lib.ss2d_cross_merge_table.argtypes = [D, P, P, P, P]
        lib.ss2d_forward_table.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, sz, P]
        lib.ss2d_backward_table.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P, sz, P]
        lib.ss2d_bimamba_backward.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P, P, sz,
                                              P]
        lib.ss2d_backward.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P, P, P, P, P, P, P, P, sz, P]
        for name in ("ss2d_cross_scan", "ss2d_cross_merge", "ss2d_selective_scan_fwd", "ss2d_selective_scan_bwd",
                     "ss2d_selective_scan_fwd_ex", "ss2d_selective_scan_bwd_ex", "ss2d_forward", "ss2d_backward",
                     "ss2d_bimamba_forward", "ss2d_bimamba_backward", "ss2d_path_tables", "ss2d_cross_scan_table",
                     "ss2d_cross_merge_table", "ss2d_forward_table", "ss2d_backward_table", "ss2d_forward_proj",
                     "ss2d_backward_proj", "ss2d_forward_proj_conv", "ss2d_backward_proj_conv"):
            getattr(lib, name).restype = ctypes.c_int
        lib.ss2d_workspace_bytes.argtypes = [D, i]
        lib.ss2d_workspace_bytes.restype = sz
        lib.ss2d_chunk_states_elems.argtypes = [D]
        lib.ss2d_chunk_states_elems.restype = sz
        lib.ss2d_status_string.argtypes = [i]
        lib.ss2d_status_string.restype = ctypes.c_char_p
        lib.ss2d_last_cuda_error.restype = ctypes.c_char_p
        lib.ss2d_launch_count.restype = ctypes.c_uint64
        lib.ss2d_version.restype = ctypes.c_int
        lib.ss2d_set_trace_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        lib.ss2d_set_trace_events.restype = None
        _lib = lib
        return lib


def _code(dtype) -> int:
    if dtype == torch.float32:
        return F32
    if dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {dtype}: float32 or bfloat16")


def _desc(batch, dim, height, width, d_state, in_dtype, out_dtype) -> Desc:
    return Desc(int(batch), int(dim), int(height), int(width), int(d_state), _code(in_dtype), _code(out_dtype))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _c(t, dtype=None):
    """contiguous CUDA tensor (optionally cast); None passes through"""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("ss2d: tensors must live on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        t = t.to(dtype)
    return t.contiguous()


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(status, where):
    if status != 0:
        detail = _load().ss2d_last_cuda_error().decode() if status == 6 else ""
        raise SS2DError(status, where, detail)


def launch_count() -> int:
    """Kernels libss2d has launched since it was loaded."""
    return int(_load().ss2d_launch_count())


class trace_events:
    """Context manager: record the given torch.cuda.Event objects after the library's next kernels.

    with ss.trace_events([e1, e2]):   # e1 after the 1st kernel, e2 after the 2nd
        ss.ss2d_forward(...)
    """

    def __init__(self, events):
        self._events = list(events)
        for e in self._events:
            if not e.cuda_event:  # torch creates the CUDA event lazily, on its first record
                e.record()
        self._arr = (ctypes.c_void_p * len(self._events))(*[e.cuda_event for e in self._events])

    def __enter__(self):
        _load().ss2d_set_trace_events(self._arr, len(self._events))
        return self

    def __exit__(self, *exc):
        _load().ss2d_set_trace_events(None, 0)
        return False


def workspace_bytes(batch, dim, height, width, d_state, op, in_dtype=torch.float32, out_dtype=None) -> int:
    d = _desc(batch, dim, height, width, d_state, in_dtype, out_dtype or in_dtype)
    return int(_load().ss2d_workspace_bytes(ctypes.byref(d), int(op)))


def chunk_states_elems(batch, dim, height, width, d_state) -> int:
    d = _desc(batch, dim, height, width, d_state, torch.float32, torch.float32)
    return int(_load().ss2d_chunk_states_elems(ctypes.byref(d)))


def _workspace(nbytes, device):
    if nbytes == 0:
        return None
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ steps --

def cross_scan(x, out=None):
    """x (B, D, H, W) -> xs (B, 4, D, H*W) in the same dtype."""
    x = _c(x)
    Bn, Dn, H, W = x.shape
    if out is None:
        out = torch.empty((Bn, 4, Dn, H * W), dtype=x.dtype, device=x.device)
    d = _desc(Bn, Dn, H, W, 1, x.dtype, x.dtype)
    _check(_load().ss2d_cross_scan(ctypes.byref(d), _p(x), _p(out), _stream(x)), "ss2d_cross_scan")
    return out


def cross_merge(ys, H, W, out=None, out_dtype=None):
    """ys (B, 4, D, H*W) -> y (B, D, H, W) = (y0 + y2) + (y1 + y3) per pixel, fp32 sum, one rounding."""
    ys = _c(ys)
    Bn, K, Dn, L = ys.shape
    if K != 4 or L != H * W:
        raise ValueError("cross_merge: ys must be (B, 4, D, H*W)")
    out_dtype = out_dtype or ys.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=ys.device)
    d = _desc(Bn, Dn, H, W, 1, ys.dtype, out.dtype)
    _check(_load().ss2d_cross_merge(ctypes.byref(d), _p(ys), _p(out), _stream(ys)), "ss2d_cross_merge")
    return out


def _params(A, D, delta_bias):
    return _c(A, torch.float32), _c(D, torch.float32), _c(delta_bias, torch.float32)


def selective_scan_fwd(u, delta, A, B, C, D=None, delta_bias=None, delta_softplus=False, out=None,
                       out_dtype=None, return_chunk_states=False, z=None, return_last_state=False):
    """S6 forward over the 4*dim sequences of an SS2D problem.

    u, delta (Bn, 4D, L); A (4D, N) fp32; B, C (Bn, 4, N, L); D, delta_bias (4D) fp32 or None;
    z (Bn, 4D, L) or None gates the output: out = (C.h + D u) * silu(z).
    Returns out (Bn, 4D, L), followed by last_state (Bn, 4D, N) fp32 if return_last_state and
    chunk_states (Bn, 4D, ceil(L / CHUNK_LEN), N) fp32 if return_chunk_states.
    """
    u = _c(u)
    delta, B, C, z = (_c(t, u.dtype) for t in (delta, B, C, z))
    A, D, delta_bias = _params(A, D, delta_bias)
    Bn, Ch, L = u.shape
    if Ch % 4 or B.shape[1] != 4:
        raise ValueError("selective_scan_fwd: u must be (B, 4*dim, L) and B/C (B, 4, N, L)")
    if z is not None and z.shape != u.shape:
        raise ValueError("selective_scan_fwd: z must have u's shape")
    N = A.shape[1]
    out_dtype = out_dtype or u.dtype
    if out is None:
        out = torch.empty((Bn, Ch, L), dtype=out_dtype, device=u.device)
    cs = None
    if return_chunk_states:
        cs = torch.empty((Bn, Ch, -(-L // CHUNK_LEN), N), dtype=torch.float32, device=u.device)
    last = torch.empty((Bn, Ch, N), dtype=torch.float32, device=u.device) if return_last_state else None
    d = _desc(Bn, Ch // 4, 1, L, N, u.dtype, out.dtype)
    st = _load().ss2d_selective_scan_fwd_ex(ctypes.byref(d), _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z),
                                            _p(delta_bias), int(bool(delta_softplus)), _p(out), _p(last), _p(cs),
                                            _stream(u))
    _check(st, "ss2d_selective_scan_fwd_ex")
    extra = ([last] if return_last_state else []) + ([cs] if return_chunk_states else [])
    return (out, *extra) if extra else out


def selective_scan_bwd(u, delta, A, B, C, D, delta_bias, delta_softplus, dout, chunk_states=None, z=None):
    """Gradients of selective_scan_fwd.  Returns dict du, ddelta, dA, dB, dC, dD, ddelta_bias, dz
    (dD, ddelta_bias, dz are None when D, delta_bias, z are)."""
    u = _c(u)
    delta, B, C, z = (_c(t, u.dtype) for t in (delta, B, C, z))
    A, D, delta_bias = _params(A, D, delta_bias)
    dout = _c(dout)
    chunk_states = _c(chunk_states, torch.float32)
    Bn, Ch, L = u.shape
    N = A.shape[1]
    dev = u.device
    du = torch.empty_like(u)
    ddelta = torch.empty_like(u)
    dA = torch.empty_like(A)
    dB = torch.empty_like(B)
    dC = torch.empty_like(C)
    dD = torch.empty_like(D) if D is not None else None
    dbias = torch.empty_like(delta_bias) if delta_bias is not None else None
    dz = torch.empty_like(u) if z is not None else None
    d = _desc(Bn, Ch // 4, 1, L, N, u.dtype, dout.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_SELECTIVE_SCAN_BWD))
    ws = _workspace(nbytes, dev)
    st = lib.ss2d_selective_scan_bwd_ex(ctypes.byref(d), _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z),
                                        _p(delta_bias), int(bool(delta_softplus)), _p(dout), _p(chunk_states),
                                        _p(du), _p(ddelta), _p(dA), _p(dB), _p(dC), _p(dD), _p(dbias), _p(dz),
                                        _p(ws), nbytes, _stream(u))
    _check(st, "ss2d_selective_scan_bwd_ex")
    return dict(du=du, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias, dz=dz)


class SelectiveScanFunction(torch.autograd.Function):
    """autograd wrapper of the scan with selective_scan_fn's arguments ("vision mamba-yolov8",
    section "2. Vmamba module code", SelectiveScanFn): the forward keeps the chunk states, the
    backward rebuilds the states from them; the last state carries no gradient."""

    @staticmethod
    def forward(ctx, u, delta, A, B, C, D, z, delta_bias, delta_softplus, return_last_state):
        out, last, cs = selective_scan_fwd(u, delta, A, B, C, D, delta_bias, delta_softplus, z=z,
                                           return_last_state=True, return_chunk_states=True)
        ctx.save_for_backward(u, delta, A, B, C, D, z, delta_bias, cs)
        ctx.delta_softplus = delta_softplus
        if not return_last_state:
            return out
        ctx.mark_non_differentiable(last)
        return out, last

    @staticmethod
    def backward(ctx, dout, *unused):
        u, delta, A, B, C, D, z, delta_bias, cs = ctx.saved_tensors
        g = selective_scan_bwd(u, delta, A, B, C, D, delta_bias, ctx.delta_softplus, dout.to(u.dtype),
                               chunk_states=cs, z=z)
        return (g["du"], g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"], None, None)


def selective_scan_fn(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
                      return_last_state=False):
    """Differentiable S6 scan over the (Bn, 4*dim, L) sequences of an SS2D problem, with the
    argument order of the pages' selective_scan_fn.  B and C carry the 4 path groups
    (Bn, 4, N, L).  Returns out, or (out, last_state) with last_state (Bn, 4*dim, N) fp32."""
    return SelectiveScanFunction.apply(u, delta, A, B, C, D, z, delta_bias, delta_softplus, return_last_state)


# ------------------------------------------------------------------ fused --

def ss2d_forward(x, delta, A, B, C, D=None, delta_bias=None, delta_softplus=True, out=None, out_dtype=None,
                 return_chunk_states=False, workspace=None, chunk_states_out=None):
    """Fused SS2D forward.  x (Bn, D, H, W), delta (Bn, 4D, H*W), A (4D, N), B/C (Bn, 4, N, H*W).

    Returns y (Bn, D, H, W) [, chunk_states].  ``workspace`` may be a preallocated uint8
    CUDA tensor of at least workspace_bytes(..., OP_FORWARD) bytes.
    """
    x = _c(x)
    delta, B, C = (_c(t, x.dtype) for t in (delta, B, C))
    A, D, delta_bias = _params(A, D, delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=x.device)
    cs = chunk_states_out
    if return_chunk_states and cs is None:
        cs = torch.empty((Bn, 4 * Dn, -(-(H * W) // CHUNK_LEN), N), dtype=torch.float32, device=x.device)
    d = _desc(Bn, Dn, H, W, N, x.dtype, out.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_FORWARD))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_forward(ctypes.byref(d), _p(x), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(delta_bias),
                          int(bool(delta_softplus)), _p(out), _p(cs), _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_forward")
    return (out, cs) if return_chunk_states else out


def ss2d_backward(x, delta, A, B, C, D, delta_bias, delta_softplus, dy, chunk_states=None, workspace=None):
    """Fused SS2D backward.  Returns dict dx, ddelta, dA, dB, dC, dD, ddelta_bias."""
    x = _c(x)
    delta, B, C = (_c(t, x.dtype) for t in (delta, B, C))
    A, D, delta_bias = _params(A, D, delta_bias)
    dy = _c(dy)
    chunk_states = _c(chunk_states, torch.float32)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    dev = x.device
    dx = torch.empty_like(x)
    ddelta = torch.empty_like(delta)
    dA = torch.empty_like(A)
    dB = torch.empty_like(B)
    dC = torch.empty_like(C)
    dD = torch.empty_like(D) if D is not None else None
    dbias = torch.empty_like(delta_bias) if delta_bias is not None else None
    d = _desc(Bn, Dn, H, W, N, x.dtype, dy.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BACKWARD))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, dev)
    st = lib.ss2d_backward(ctypes.byref(d), _p(x), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(delta_bias),
                           int(bool(delta_softplus)), _p(dy), _p(chunk_states), _p(dx), _p(ddelta), _p(dA), _p(dB),
                           _p(dC), _p(dD), _p(dbias), _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_backward")
    return dict(dx=dx, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias)


class SS2DFunction(torch.autograd.Function):
    """autograd wrapper: forward saves the chunk states, backward runs the fused backward.
    ``tables`` (from path_tables) selects another path set; None is the cross scan."""

    @staticmethod
    def forward(ctx, x, delta, A, B, C, D, delta_bias, delta_softplus, tables=None):
        if tables is None:
            y, cs = ss2d_forward(x, delta, A, B, C, D, delta_bias, delta_softplus, return_chunk_states=True)
        else:
            y, cs = ss2d_forward_table(x, delta, A, B, C, D, delta_bias, delta_softplus, tables,
                                       return_chunk_states=True)
        ctx.save_for_backward(x, delta, A, B, C, D, delta_bias, cs, tables)
        ctx.delta_softplus = delta_softplus
        return y

    @staticmethod
    def backward(ctx, dy):
        x, delta, A, B, C, D, delta_bias, cs, tables = ctx.saved_tensors
        if tables is None:
            g = ss2d_backward(x, delta, A, B, C, D, delta_bias, ctx.delta_softplus, dy.to(x.dtype), chunk_states=cs)
        else:
            g = ss2d_backward_table(x, delta, A, B, C, D, delta_bias, ctx.delta_softplus, dy.to(x.dtype), tables,
                                    chunk_states=cs)
        return g["dx"], g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["ddelta_bias"], None, None


def ss2d(x, delta, A, B, C, D=None, delta_bias=None, delta_softplus=True, tables=None):
    """Differentiable fused SS2D: y = CrossMerge(S6(CrossScan(x))) over the cross scan, or over
    the path set of ``tables`` (see path_tables)."""
    return SS2DFunction.apply(x, delta, A, B, C, D, delta_bias, delta_softplus, tables)


# ------------------------------------------------------------ bidirectional --

def _bidir_params(A, A_b, D, delta_bias):
    A2 = torch.stack([_c(A, torch.float32), _c(A_b, torch.float32)]).contiguous()  # (2, D, N)
    return A2, _c(D, torch.float32), _c(delta_bias, torch.float32)


def _bc3(t, dtype):
    """B or C as (Bn, N, L); a (Bn, 1, N, L) tensor is accepted too"""
    t = _c(t, dtype)
    return t[:, 0] if t.dim() == 4 else t


def bimamba_forward(x, delta, A, A_b, B, C, D=None, z=None, delta_bias=None, delta_softplus=True, out=None,
                    out_dtype=None, return_chunk_states=False, workspace=None):
    """Bidirectional scan of bimamba_inner_ref: S6 over the sequence with A plus S6 over the reversed
    sequence with A_b, reversed back; gated by silu(z) when z is given.

    x, delta, z (Bn, D, L); A, A_b (D, N) fp32; B, C (Bn, N, L); D, delta_bias (D) fp32 or None.
    Returns y (Bn, D, L) [, chunk_states (Bn, 2D, ceil(L / CHUNK_LEN), N)].
    """
    x = _c(x)
    delta, z = (_c(t, x.dtype) for t in (delta, z))
    B, C = _bc3(B, x.dtype), _bc3(C, x.dtype)
    A2, D, delta_bias = _bidir_params(A, A_b, D, delta_bias)
    Bn, Dn, L = x.shape
    N = A2.shape[2]
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty((Bn, Dn, L), dtype=out_dtype, device=x.device)
    cs = None
    if return_chunk_states:
        cs = torch.empty((Bn, 2 * Dn, -(-L // CHUNK_LEN), N), dtype=torch.float32, device=x.device)
    d = _desc(Bn, Dn, 1, L, N, x.dtype, out.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BIMAMBA_FORWARD))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_bimamba_forward(ctypes.byref(d), _p(x), _p(delta), _p(A2), _p(B), _p(C), _p(D), _p(z),
                                  _p(delta_bias), int(bool(delta_softplus)), _p(out), _p(cs), _p(workspace), nbytes,
                                  _stream(x))
    _check(st, "ss2d_bimamba_forward")
    return (out, cs) if return_chunk_states else out


def bimamba_backward(x, delta, A, A_b, B, C, D, z, delta_bias, delta_softplus, dy, chunk_states=None,
                     workspace=None):
    """Gradients of bimamba_forward.  Returns dict dx, ddelta, dA, dA_b, dB, dC, dD, ddelta_bias, dz
    (dB, dC as (Bn, N, L); None where the input is None)."""
    x = _c(x)
    delta, z = (_c(t, x.dtype) for t in (delta, z))
    B, C = _bc3(B, x.dtype), _bc3(C, x.dtype)
    A2, D, delta_bias = _bidir_params(A, A_b, D, delta_bias)
    dy = _c(dy)
    chunk_states = _c(chunk_states, torch.float32)
    Bn, Dn, L = x.shape
    N = A2.shape[2]
    dev = x.device
    dx = torch.empty_like(x)
    ddelta = torch.empty_like(delta)
    dA2 = torch.empty_like(A2)
    dB = torch.empty_like(B)
    dC = torch.empty_like(C)
    dD = torch.empty_like(D) if D is not None else None
    dbias = torch.empty_like(delta_bias) if delta_bias is not None else None
    dz = torch.empty_like(z) if z is not None else None
    d = _desc(Bn, Dn, 1, L, N, x.dtype, dy.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BIMAMBA_BACKWARD))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, dev)
    st = lib.ss2d_bimamba_backward(ctypes.byref(d), _p(x), _p(delta), _p(A2), _p(B), _p(C), _p(D), _p(z),
                                   _p(delta_bias), int(bool(delta_softplus)), _p(dy), _p(chunk_states), _p(dx),
                                   _p(ddelta), _p(dA2), _p(dB), _p(dC), _p(dD), _p(dbias), _p(dz), _p(workspace),
                                   nbytes, _stream(x))
    _check(st, "ss2d_bimamba_backward")
    return dict(dx=dx, ddelta=ddelta, dA=dA2[0], dA_b=dA2[1], dB=dB, dC=dC, dD=dD, ddelta_bias=dbias, dz=dz)


class BiMambaFunction(torch.autograd.Function):
    """autograd wrapper of the bidirectional scan: the forward keeps both directions' chunk states."""

    @staticmethod
    def forward(ctx, x, delta, A, A_b, B, C, D, z, delta_bias, delta_softplus):
        y, cs = bimamba_forward(x, delta, A, A_b, B, C, D, z, delta_bias, delta_softplus, return_chunk_states=True)
        ctx.save_for_backward(x, delta, A, A_b, B, C, D, z, delta_bias, cs)
        ctx.delta_softplus = delta_softplus
        ctx.bc4 = (B.dim() == 4, C.dim() == 4)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, delta, A, A_b, B, C, D, z, delta_bias, cs = ctx.saved_tensors
        g = bimamba_backward(x, delta, A, A_b, B, C, D, z, delta_bias, ctx.delta_softplus, dy.to(x.dtype),
                             chunk_states=cs)
        dB = g["dB"].unsqueeze(1) if ctx.bc4[0] else g["dB"]
        dC = g["dC"].unsqueeze(1) if ctx.bc4[1] else g["dC"]
        return g["dx"], g["ddelta"], g["dA"], g["dA_b"], dB, dC, g["dD"], g["dz"], g["ddelta_bias"], None


def bimamba_scan(x, delta, A, A_b, B, C, D=None, z=None, delta_bias=None, delta_softplus=True):
    """Differentiable bidirectional scan (the selective-scan part of bimamba_inner_ref)."""
    return BiMambaFunction.apply(x, delta, A, A_b, B, C, D, z, delta_bias, delta_softplus)


# ---------------------------------------------------------------- path sets --

def path_tables(H, W, paths=PATHS_DIAGONAL, device=None):
    """int32 (4, H*W) device table of a path set: rows 0, 1 the pixel at each step of paths 0
    and 1, rows 2, 3 the step at each pixel (paths 2, 3 are 0, 1 backwards).  paths is
    PATHS_CROSS (row-major, column-major) or PATHS_DIAGONAL (the two diagonal orders)."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    t = torch.empty((4, H * W), dtype=torch.int32, device=device)
    d = _desc(1, 1, H, W, 1, torch.float32, torch.float32)
    _check(_load().ss2d_path_tables(ctypes.byref(d), int(paths), _p(t), _stream(t)), "ss2d_path_tables")
    return t


def _tab(tables, L):
    t = _c(tables)
    if t.dtype != torch.int32 or t.shape != (4, L):
        raise ValueError(f"path tables must be int32 (4, {L})")
    return t


def cross_scan_table(x, tables, out=None):
    """x (B, D, H, W) -> xs (B, 4, D, H*W) along the path set of ``tables``."""
    x = _c(x)
    Bn, Dn, H, W = x.shape
    t = _tab(tables, H * W)
    if out is None:
        out = torch.empty((Bn, 4, Dn, H * W), dtype=x.dtype, device=x.device)
    d = _desc(Bn, Dn, H, W, 1, x.dtype, x.dtype)
    _check(_load().ss2d_cross_scan_table(ctypes.byref(d), _p(t), _p(x), _p(out), _stream(x)), "ss2d_cross_scan_table")
    return out


def cross_merge_table(ys, H, W, tables, out=None, out_dtype=None):
    """ys (B, 4, D, H*W) -> y (B, D, H, W): each path's value at each pixel, (t0 + t2) + (t1 + t3) in fp32."""
    ys = _c(ys)
    Bn, K, Dn, L = ys.shape
    if K != 4 or L != H * W:
        raise ValueError("cross_merge_table: ys must be (B, 4, D, H*W)")
    t = _tab(tables, L)
    out_dtype = out_dtype or ys.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=ys.device)
    d = _desc(Bn, Dn, H, W, 1, ys.dtype, out.dtype)
    _check(_load().ss2d_cross_merge_table(ctypes.byref(d), _p(t), _p(ys), _p(out), _stream(ys)),
           "ss2d_cross_merge_table")
    return out


def ss2d_forward_table(x, delta, A, B, C, D, delta_bias, delta_softplus, tables, out=None, out_dtype=None,
                       return_chunk_states=False, workspace=None):
    """Fused SS2D forward over the path set of ``tables``; arguments as ss2d_forward."""
    x = _c(x)
    delta, B, C = (_c(t, x.dtype) for t in (delta, B, C))
    A, D, delta_bias = _params(A, D, delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    t = _tab(tables, H * W)
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=x.device)
    cs = None
    if return_chunk_states:
        cs = torch.empty((Bn, 4 * Dn, -(-(H * W) // CHUNK_LEN), N), dtype=torch.float32, device=x.device)
    d = _desc(Bn, Dn, H, W, N, x.dtype, out.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_FORWARD_TABLE))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_forward_table(ctypes.byref(d), _p(t), _p(x), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(delta_bias),
                                int(bool(delta_softplus)), _p(out), _p(cs), _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_forward_table")
    return (out, cs) if return_chunk_states else out


def ss2d_backward_table(x, delta, A, B, C, D, delta_bias, delta_softplus, dy, tables, chunk_states=None,
                        workspace=None):
    """Fused SS2D backward over the path set of ``tables``.  Returns the dict of ss2d_backward."""
    x = _c(x)
    delta, B, C = (_c(t, x.dtype) for t in (delta, B, C))
    A, D, delta_bias = _params(A, D, delta_bias)
    dy = _c(dy)
    chunk_states = _c(chunk_states, torch.float32)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    t = _tab(tables, H * W)
    dev = x.device
    dx = torch.empty_like(x)
    ddelta = torch.empty_like(delta)
    dA = torch.empty_like(A)
    dB = torch.empty_like(B)
    dC = torch.empty_like(C)
    dD = torch.empty_like(D) if D is not None else None
    dbias = torch.empty_like(delta_bias) if delta_bias is not None else None
    d = _desc(Bn, Dn, H, W, N, x.dtype, dy.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BACKWARD_TABLE))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, dev)
    st = lib.ss2d_backward_table(ctypes.byref(d), _p(t), _p(x), _p(delta), _p(A), _p(B), _p(C), _p(D),
                                 _p(delta_bias), int(bool(delta_softplus)), _p(dy), _p(chunk_states), _p(dx),
                                 _p(ddelta), _p(dA), _p(dB), _p(dC), _p(dD), _p(dbias), _p(workspace), nbytes,
                                 _stream(x))
    _check(st, "ss2d_backward_table")
    return dict(dx=dx, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias)


# ---------------------------------------------------------------- producer --

def ss2d_forward_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D=None, delta_softplus=True, out=None,
                      out_dtype=None, return_x_dbl=False, return_chunk_states=False, workspace=None):
    """Fused SS2D forward with its per-path producer (MambaInnerFn.forward's x_proj and dt_proj):
    x (Bn, D, H, W); x_proj_weight (4, R+2N, D); dt_proj_weight (4, D, R); dt_proj_bias (4D).
    For dt ranks up to 8 delta is never materialised: the scan computes softplus(W_dt . x_dbl[:R] +
    bias) per step; larger ranks materialise delta in the workspace.
    Returns y [, x_dbl (Bn, 4, R+2N, L)] [, chunk_states]."""
    x = _c(x)
    Wx = _c(x_proj_weight, torch.float32)
    Wdt = _c(dt_proj_weight, torch.float32)
    A, D, bias = _params(A, D, dt_proj_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    R = Wdt.shape[2]
    if Wx.shape != (4, R + 2 * N, Dn) or Wdt.shape != (4, Dn, R):
        raise ValueError("ss2d_forward_proj: x_proj_weight must be (4, R+2N, D) and dt_proj_weight (4, D, R)")
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=x.device)
    x_dbl = torch.empty((Bn, 4, R + 2 * N, H * W), dtype=x.dtype, device=x.device)
    cs = None
    if return_chunk_states:
        cs = torch.empty((Bn, 4 * Dn, -(-(H * W) // CHUNK_LEN), N), dtype=torch.float32, device=x.device)
    d = _desc(Bn, Dn, H, W, N, x.dtype, out.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_FORWARD_PROJ))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_forward_proj(ctypes.byref(d), int(R), _p(x), _p(Wx), _p(Wdt), _p(bias), _p(A), _p(D),
                               int(bool(delta_softplus)), _p(out), _p(x_dbl), _p(cs), _p(workspace), nbytes,
                               _stream(x))
    _check(st, "ss2d_forward_proj")
    extra = ([x_dbl] if return_x_dbl else []) + ([cs] if return_chunk_states else [])
    return (out, *extra) if extra else out


def ss2d_backward_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, x_dbl, dy, delta_softplus=True,
                       chunk_states=None, workspace=None):
    """Backward of ss2d_forward_proj (MambaInnerFn.backward's path through the scan and the producer).
    x_dbl is the forward's (Bn, 4, R+2N, L) output; dy (Bn, D, H, W).  Returns a dict with dx,
    dx_proj_weight (4, R+2N, D), ddt_proj_weight (4, D, R), ddt_proj_bias (4D, or None without a bias),
    dA (4D, N) and dD (4D, or None without D); the weight, bias, A and D gradients are fp32."""
    x = _c(x)
    Wx = _c(x_proj_weight, torch.float32)
    Wdt = _c(dt_proj_weight, torch.float32)
    A, D, bias = _params(A, D, dt_proj_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    R = Wdt.shape[2]
    if Wx.shape != (4, R + 2 * N, Dn) or Wdt.shape != (4, Dn, R):
        raise ValueError("ss2d_backward_proj: x_proj_weight must be (4, R+2N, D) and dt_proj_weight (4, D, R)")
    x_dbl = _c(x_dbl, x.dtype)
    if x_dbl.shape != (Bn, 4, R + 2 * N, H * W):
        raise ValueError("ss2d_backward_proj: x_dbl must be (Bn, 4, R+2N, H*W) in x's dtype")
    dy = _c(dy)
    cs = _c(chunk_states, torch.float32) if chunk_states is not None else None
    f32 = dict(dtype=torch.float32, device=x.device)
    dx = torch.empty_like(x)
    dWx = torch.empty((4, R + 2 * N, Dn), **f32)
    dWdt = torch.empty((4, Dn, R), **f32)
    dbias = torch.empty((4 * Dn,), **f32) if bias is not None else None
    dA = torch.empty((4 * Dn, N), **f32)
    dD = torch.empty((4 * Dn,), **f32) if D is not None else None
    d = _desc(Bn, Dn, H, W, N, x.dtype, dy.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BACKWARD_PROJ))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_backward_proj(ctypes.byref(d), int(R), _p(x), _p(Wx), _p(Wdt), _p(bias), _p(A), _p(D),
                                int(bool(delta_softplus)), _p(x_dbl), _p(cs), _p(dy), _p(dx), _p(dWx), _p(dWdt),
                                _p(dbias), _p(dA), _p(dD), _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_backward_proj")
    return dict(dx=dx, dx_proj_weight=dWx, ddt_proj_weight=dWdt, ddt_proj_bias=dbias, dA=dA, dD=dD)


def _conv_args(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, what):
    x = _c(x)
    cw = _c(conv_weight, torch.float32)
    cb = _c(conv_bias, torch.float32) if conv_bias is not None else None
    Wx = _c(x_proj_weight, torch.float32)
    Wdt = _c(dt_proj_weight, torch.float32)
    A, D, bias = _params(A, D, dt_proj_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    R = Wdt.shape[2]
    if Wx.shape != (4, R + 2 * N, Dn) or Wdt.shape != (4, Dn, R):
        raise ValueError(f"{what}: x_proj_weight must be (4, R+2N, D) and dt_proj_weight (4, D, R)")
    if cw.dim() != 3 or cw.shape[:2] != (4, Dn) or (cb is not None and cb.shape != (4 * Dn,)):
        raise ValueError(f"{what}: conv_weight must be (4, D, d_conv) and conv_bias (4D)")
    return x, cw, cb, Wx, Wdt, A, D, bias, R, N


def ss2d_forward_proj_conv(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D=None,
                           delta_softplus=True, out=None, out_dtype=None, return_x_dbl=False,
                           return_chunk_states=False, workspace=None):
    """SS2D forward with the whole per-path producer of MambaInnerFn.forward: a causal depthwise
    conv of width d_conv with SiLU along every path (conv_weight (4, D, d_conv), conv_bias (4D)),
    then x_proj, dt_proj, the scan of every path and CrossMerge.  Returns y [, x_dbl] [, chunk_states]."""
    x, cw, cb, Wx, Wdt, A, D, bias, R, N = _conv_args(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight,
                                                      dt_proj_bias, A, D, "ss2d_forward_proj_conv")
    Bn, Dn, H, W = x.shape
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty((Bn, Dn, H, W), dtype=out_dtype, device=x.device)
    x_dbl = torch.empty((Bn, 4, R + 2 * N, H * W), dtype=x.dtype, device=x.device)
    cs = None
    if return_chunk_states:
        cs = torch.empty((Bn, 4 * Dn, -(-(H * W) // CHUNK_LEN), N), dtype=torch.float32, device=x.device)
    d = _desc(Bn, Dn, H, W, N, x.dtype, out.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_FORWARD_PROJ_CONV))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_forward_proj_conv(ctypes.byref(d), int(R), int(cw.shape[2]), _p(x), _p(cw), _p(cb), _p(Wx),
                                    _p(Wdt), _p(bias), _p(A), _p(D), int(bool(delta_softplus)), _p(out), _p(x_dbl),
                                    _p(cs), _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_forward_proj_conv")
    extra = ([x_dbl] if return_x_dbl else []) + ([cs] if return_chunk_states else [])
    return (out, *extra) if extra else out


def ss2d_backward_proj_conv(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, x_dbl,
                            dy, delta_softplus=True, chunk_states=None, workspace=None):
    """Backward of ss2d_forward_proj_conv.  Returns a dict with dx, dconv_weight (4, D, d_conv),
    dconv_bias (4D or None), dx_proj_weight, ddt_proj_weight, ddt_proj_bias, dA, dD (fp32 but dx)."""
    x, cw, cb, Wx, Wdt, A, D, bias, R, N = _conv_args(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight,
                                                      dt_proj_bias, A, D, "ss2d_backward_proj_conv")
    Bn, Dn, H, W = x.shape
    x_dbl = _c(x_dbl, x.dtype)
    if x_dbl.shape != (Bn, 4, R + 2 * N, H * W):
        raise ValueError("ss2d_backward_proj_conv: x_dbl must be (Bn, 4, R+2N, H*W) in x's dtype")
    dy = _c(dy)
    cs = _c(chunk_states, torch.float32) if chunk_states is not None else None
    f32 = dict(dtype=torch.float32, device=x.device)
    dx = torch.empty_like(x)
    dcw = torch.empty(tuple(cw.shape), **f32)
    dcb = torch.empty((4 * Dn,), **f32) if cb is not None else None
    dWx = torch.empty((4, R + 2 * N, Dn), **f32)
    dWdt = torch.empty((4, Dn, R), **f32)
    dbias = torch.empty((4 * Dn,), **f32) if bias is not None else None
    dA = torch.empty((4 * Dn, N), **f32)
    dD = torch.empty((4 * Dn,), **f32) if D is not None else None
    d = _desc(Bn, Dn, H, W, N, x.dtype, dy.dtype)
    lib = _load()
    nbytes = int(lib.ss2d_workspace_bytes(ctypes.byref(d), OP_BACKWARD_PROJ_CONV))
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    st = lib.ss2d_backward_proj_conv(ctypes.byref(d), int(R), int(cw.shape[2]), _p(x), _p(cw), _p(cb), _p(Wx),
                                     _p(Wdt), _p(bias), _p(A), _p(D), int(bool(delta_softplus)), _p(x_dbl), _p(cs),
                                     _p(dy), _p(dx), _p(dcw), _p(dcb), _p(dWx), _p(dWdt), _p(dbias), _p(dA), _p(dD),
                                     _p(workspace), nbytes, _stream(x))
    _check(st, "ss2d_backward_proj_conv")
    return dict(dx=dx, dconv_weight=dcw, dconv_bias=dcb, dx_proj_weight=dWx, ddt_proj_weight=dWdt,
                ddt_proj_bias=dbias, dA=dA, dD=dD)


class SS2DProjFunction(torch.autograd.Function):
    """autograd wrapper of the SS2D forward with its per-path producer (MambaInnerFn's x_proj and
    dt_proj, and with conv_weight its causal depthwise conv + SiLU): the forward keeps x_dbl and
    the chunk states, the backward runs ss2d_backward_proj(_conv)."""

    @staticmethod
    def forward(ctx, x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, conv_weight, conv_bias, delta_softplus):
        if conv_weight is None:
            y, xd, cs = ss2d_forward_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, delta_softplus,
                                          return_x_dbl=True, return_chunk_states=True)
        else:
            y, xd, cs = ss2d_forward_proj_conv(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight,
                                               dt_proj_bias, A, D, delta_softplus, return_x_dbl=True,
                                               return_chunk_states=True)
        ctx.save_for_backward(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, conv_weight, conv_bias, xd, cs)
        ctx.delta_softplus = delta_softplus
        return y

    @staticmethod
    def backward(ctx, dy):
        x, Wx, Wdt, bias, A, D, cw, cb, xd, cs = ctx.saved_tensors
        dy = dy.contiguous()
        if cw is None:
            g = ss2d_backward_proj(x, Wx, Wdt, bias, A, D, xd, dy, ctx.delta_softplus, chunk_states=cs)
            dcw = dcb = None
        else:
            g = ss2d_backward_proj_conv(x, cw, cb, Wx, Wdt, bias, A, D, xd, dy, ctx.delta_softplus, chunk_states=cs)
            dcw, dcb = g["dconv_weight"], g["dconv_bias"]
        return (g["dx"], g["dx_proj_weight"], g["ddt_proj_weight"], g["ddt_proj_bias"], g["dA"], g["dD"], dcw, dcb,
                None)


def ss2d_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D=None, conv_weight=None, conv_bias=None,
              delta_softplus=True):
    """Differentiable SS2D with its per-path producer: y = ss2d_forward_proj(...) or, with conv_weight
    (4, D, d_conv), ss2d_forward_proj_conv(...).  Gradients reach x, both projection weights, the
    dt_proj bias, A, D and the conv weight and bias."""
    return SS2DProjFunction.apply(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, conv_weight, conv_bias,
                                  delta_softplus)
