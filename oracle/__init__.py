"""fp64 CPU oracle for SS2D (CrossScan -> S6 selective scan -> CrossMerge).

TEST INFRASTRUCTURE ONLY.  This package is the checker that the CUDA library
is compared against.  It shares no code with the CUDA path; only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use it.

Sources of the arithmetic (restated, not copied):

* "VMamba: Visual State Space Model", section "2D Selective Scan (SS2D) for
  visual data" and Fig. 2: CrossScan unfolds the map along four paths, one S6
  block per path, CrossMerge sums the four results back into the map.
* "vision mamba-yolov8", section "2. Vmamba module code", ``selective_scan_ref``:
  the S6 recurrence with softplus step size and grouped B/C.

The numerical work lives in ``ss2d_oracle.c`` (plain loops, double precision);
this module compiles it with gcc on first use and marshals numpy arrays.
Inputs may be any real dtype; they are converted to float64 exactly
(bf16 / fp32 values are representable in fp64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss2d_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

K_PATHS = 4


def build(force: bool = False) -> str:
    """Compile ``ss2d_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.POINTER(ctypes.c_double)
            l = ctypes.c_long
            lib.oracle_path_pixel.argtypes = [ctypes.c_int, l, l, l]
            lib.oracle_path_pixel.restype = l
            lib.oracle_cross_scan.argtypes = [l, l, l, l, P, P]
            lib.oracle_cross_merge.argtypes = [l, l, l, l, P, P]
            lib.oracle_selective_scan_fwd.argtypes = [l, l, l, l, l, P, P, P, P, P, P, P,
                                                      ctypes.c_int, P, P, P]
            lib.oracle_selective_scan_bwd.argtypes = [l, l, l, l, l, P, P, P, P, P, P, P,
                                                      ctypes.c_int, P, P, P, P, P, P, P, P, P, P]
            lib.oracle_ss2d_forward.argtypes = [l, l, l, l, l, P, P, P, P, P, P, P, ctypes.c_int, P]
            lib.oracle_ss2d_backward.argtypes = [l, l, l, l, l, P, P, P, P, P, P, P, ctypes.c_int,
                                                 P, P, P, P, P, P, P, P]
            lib.oracle_num_threads.restype = ctypes.c_int
            LP = ctypes.POINTER(ctypes.c_long)
            lib.oracle_cross_scan_table.argtypes = [l, l, l, LP, P, P]
            lib.oracle_cross_merge_table.argtypes = [l, l, l, LP, P, P]
            lib.oracle_ss2d_forward_table.argtypes = [l, l, l, l, LP, P, P, P, P, P, P, P, ctypes.c_int, P]
            lib.oracle_ss2d_backward_table.argtypes = [l, l, l, l, LP, P, P, P, P, P, P, P, ctypes.c_int, P, P,
                                                       P, P, P, P, P, P]
            _lib = lib
    return _lib


def _f64(a):
    """Contiguous float64 copy of an array-like (torch tensors included)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: exact upcast on the host
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def path_pixel(k: int, l: int, H: int, W: int) -> int:
    """Pixel index h*W+w visited at step l of path k."""
    return int(_load().oracle_path_pixel(int(k), int(l), int(H), int(W)))


def cross_scan(x):
    """x (B, D, H, W) -> xs (B, 4, D, H*W)."""
    x = _f64(x)
    Bn, Dn, H, W = x.shape
    xs = np.empty((Bn, K_PATHS, Dn, H * W), dtype=np.float64)
    _load().oracle_cross_scan(Bn, Dn, H, W, _ptr(x), _ptr(xs))
    return xs


def cross_merge(ys, H: int, W: int):
    """ys (B, 4, D, H*W) -> y (B, D, H, W), summed as (y0 + y2) + (y1 + y3)."""
    ys = _f64(ys)
    Bn, K, Dn, L = ys.shape
    assert K == K_PATHS and L == H * W
    y = np.empty((Bn, Dn, H, W), dtype=np.float64)
    _load().oracle_cross_merge(Bn, Dn, H, W, _ptr(ys), _ptr(y))
    return y


def selective_scan_fwd(u, delta, A, B, C, D=None, delta_bias=None, delta_softplus=False,
                       return_last_state=False, z=None):
    """S6 forward.  u, delta (Bn, Ch, L); A (Ch, N); B, C (Bn, G, N, L); D, delta_bias (Ch);
    z (Bn, Ch, L) gates the output with silu(z)."""
    u, delta, A, B, C = (_f64(t) for t in (u, delta, A, B, C))
    D, delta_bias, z = _f64(D), _f64(delta_bias), _f64(z)
    Bn, Ch, L = u.shape
    N = A.shape[1]
    G = B.shape[1]
    assert delta.shape == u.shape and A.shape == (Ch, N) and B.shape == (Bn, G, N, L)
    assert C.shape == B.shape and Ch % G == 0
    assert z is None or z.shape == u.shape
    out = np.empty_like(u)
    last = np.empty((Bn, Ch, N), dtype=np.float64) if return_last_state else None
    _load().oracle_selective_scan_fwd(Bn, Ch, L, N, G, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                      _ptr(C), _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)),
                                      _ptr(z), _ptr(out), _ptr(last))
    return (out, last) if return_last_state else out


def selective_scan_bwd(u, delta, A, B, C, D, delta_bias, delta_softplus, dout, z=None):
    """S6 backward.  Returns dict du, ddelta, dA, dB, dC, dD, ddelta_bias, dz (None when absent)."""
    u, delta, A, B, C, dout = (_f64(t) for t in (u, delta, A, B, C, dout))
    D, delta_bias, z = _f64(D), _f64(delta_bias), _f64(z)
    Bn, Ch, L = u.shape
    N = A.shape[1]
    G = B.shape[1]
    du = np.empty_like(u)
    ddelta = np.empty_like(u)
    dA = np.empty_like(A)
    dB = np.empty_like(B)
    dC = np.empty_like(C)
    dD = np.empty(Ch, dtype=np.float64) if D is not None else None
    dbias = np.empty(Ch, dtype=np.float64) if delta_bias is not None else None
    dz = np.empty_like(u) if z is not None else None
    assert z is None or z.shape == u.shape
    _load().oracle_selective_scan_bwd(Bn, Ch, L, N, G, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                      _ptr(C), _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)),
                                      _ptr(z), _ptr(dout), _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB),
                                      _ptr(dC), _ptr(dD), _ptr(dbias), _ptr(dz))
    return dict(du=du, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias, dz=dz)


# ------------------------------------------------------- producer projections

def path_projections(x, x_proj_weight, dt_proj_weight):
    """The producer of the scan's inputs, per path, as in MambaInnerFn.forward ("vision
    mamba-yolov8", section 2): x_dbl = x_proj(u) with R + 2N outputs per token,
    delta = dt_proj.weight @ x_dbl[:R], B = x_dbl[R:R+N], C = x_dbl[R+N:].  SS2D gives every
    path k its own projections; u is x read along path k (CrossScan).

    x (Bn, D, H, W); x_proj_weight (4, R+2N, D); dt_proj_weight (4, D, R).
    Returns delta (Bn, 4D, L), B, C (Bn, 4, N, L), x_dbl (Bn, 4, R+2N, L)."""
    x, Wx, Wdt = _f64(x), _f64(x_proj_weight), _f64(dt_proj_weight)
    Bn, Dn, H, W = x.shape
    K, RN, _ = Wx.shape
    R = Wdt.shape[2]
    N = (RN - R) // 2
    xs = cross_scan(x)                                         # (Bn, 4, D, L)
    x_dbl = np.einsum("bkdl,kcd->bkcl", xs, Wx)                # (Bn, 4, R+2N, L)
    delta = np.einsum("kdr,bkrl->bkdl", Wdt, x_dbl[:, :, :R])  # (Bn, 4, D, L)
    Bm = np.ascontiguousarray(x_dbl[:, :, R:R + N])
    Cm = np.ascontiguousarray(x_dbl[:, :, R + N:])
    return delta.reshape(Bn, K * Dn, H * W), Bm, Cm, x_dbl


def ss2d_forward_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D=None, delta_softplus=True):
    """SS2D forward with its producer: path_projections, then the SS2D forward on those inputs
    with dt_proj's bias as delta_bias."""
    delta, Bm, Cm, _ = path_projections(x, x_proj_weight, dt_proj_weight)
    return ss2d_forward(x, delta, A, Bm, Cm, D, dt_proj_bias, delta_softplus)


def ss2d_backward_proj(x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, delta_softplus, dy):
    """Gradients of ss2d_forward_proj, per path as MambaInnerFn.backward ("vision mamba-yolov8",
    section 2) computes them: the scan's backward on the projected inputs, then
    dx_dbl[:R] = dt_proj.weight^T @ ddelta, dx_dbl[R:] = (dB, dC),
    d dt_proj.weight = ddelta @ x_dbl[:R]^T, d x_proj.weight = dx_dbl @ u^T and
    du += x_proj.weight^T @ dx_dbl, with u and du taken along each path (CrossScan / CrossMerge).
    Returns dict dx, dx_proj_weight, ddt_proj_weight, ddt_proj_bias, dA, dD."""
    x, Wx, Wdt, dy = _f64(x), _f64(x_proj_weight), _f64(dt_proj_weight), _f64(dy)
    D, bias, A = _f64(D), _f64(dt_proj_bias), _f64(A)
    Bn, Dn, H, W = x.shape
    R = Wdt.shape[2]
    N = (Wx.shape[1] - R) // 2
    L = H * W
    delta, Bm, Cm, x_dbl = path_projections(x, Wx, Wdt)
    g = ss2d_backward(x, delta, A, Bm, Cm, D, bias, delta_softplus, dy)
    ddelta = g["ddelta"].reshape(Bn, K_PATHS, Dn, L)
    dx_dbl = np.concatenate([np.einsum("kdr,bkdl->bkrl", Wdt, ddelta), g["dB"], g["dC"]], axis=2)
    ddt_proj_weight = np.einsum("bkdl,bkrl->kdr", ddelta, x_dbl[:, :, :R])
    xs = cross_scan(x)                                              # u along every path
    dx_proj_weight = np.einsum("bkcl,bkdl->kcd", dx_dbl, xs)
    dus = np.einsum("kcd,bkcl->bkdl", Wx, dx_dbl)                   # du along every path
    dx = g["dx"] + cross_merge(dus, H, W)
    return dict(dx=dx, dx_proj_weight=dx_proj_weight, ddt_proj_weight=ddt_proj_weight,
                ddt_proj_bias=g["ddelta_bias"], dA=g["dA"], dD=g["dD"])


# --------------------------------------------- causal depthwise conv per path

def path_conv(x, conv_weight, conv_bias=None):
    """The causal depthwise conv with SiLU that MambaInnerFn.forward ("vision mamba-yolov8",
    section 2) applies before x_proj (causal_conv1d_fwd(x, weight, bias, True)), taken along
    every SS2D path, each path with its own weights, as the SS2D of "Visual Mamba实战从零开始搭建
    图像分类模型附PyTorch代码" (section 3) runs one Mamba block per scan direction:
        pre_k[d, l] = bias[k, d] + sum_j w[k, d, j] * x_k[d, l - (W-1) + j]   (x_k = 0 before step 0)
        u_k[d, l]   = silu(pre_k[d, l]) = pre / (1 + exp(-pre))
    with x_k = x read along path k (CrossScan).  x (Bn, D, H, W); conv_weight (4, D, W);
    conv_bias (4D) or None.  Returns u (Bn, 4, D, L) and pre (Bn, 4, D, L)."""
    x, w, bias = _f64(x), _f64(conv_weight), _f64(conv_bias)
    Bn, Dn, H, W = x.shape
    Wc = w.shape[2]
    L = H * W
    xs = cross_scan(x)
    pre = np.zeros_like(xs)
    for j in range(Wc):
        s = Wc - 1 - j                                         # tap j reads s steps back
        pre[..., s:] += w[None, :, :, j, None] * xs[..., :L - s]
    if bias is not None:
        pre += bias.reshape(1, K_PATHS, Dn, 1)
    return pre / (1.0 + np.exp(-pre)), pre


def _seq_projections(us, Wx, Wdt):
    """x_proj and dt_proj of per-path sequences us (Bn, 4, D, L), as path_projections."""
    R = Wdt.shape[2]
    N = (Wx.shape[1] - R) // 2
    x_dbl = np.einsum("bkdl,kcd->bkcl", us, Wx)
    delta = np.einsum("kdr,bkrl->bkdl", Wdt, x_dbl[:, :, :R])
    return delta, np.ascontiguousarray(x_dbl[:, :, R:R + N]), np.ascontiguousarray(x_dbl[:, :, R + N:]), x_dbl


def ss2d_forward_proj_conv(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D=None,
                           delta_softplus=True):
    """SS2D forward with the whole per-path producer of MambaInnerFn.forward: u_k = path_conv,
    x_dbl = x_proj(u_k), delta = dt_proj.weight @ x_dbl[:R], B, C from x_dbl, the S6 scan of
    every path on u_k, and CrossMerge.  Returns y (Bn, D, H, W)."""
    x, Wx, Wdt = _f64(x), _f64(x_proj_weight), _f64(dt_proj_weight)
    Bn, Dn, H, W = x.shape
    L = H * W
    u, _ = path_conv(x, conv_weight, conv_bias)
    delta, Bm, Cm, _ = _seq_projections(u, Wx, Wdt)
    ys = selective_scan_fwd(u.reshape(Bn, K_PATHS * Dn, L), delta.reshape(Bn, K_PATHS * Dn, L), A, Bm, Cm, D,
                            dt_proj_bias, delta_softplus)
    return cross_merge(ys.reshape(Bn, K_PATHS, Dn, L), H, W)


def ss2d_backward_proj_conv(x, conv_weight, conv_bias, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D,
                            delta_softplus, dy):
    """Gradients of ss2d_forward_proj_conv, as MambaInnerFn.backward takes them: the scan's
    backward on (u, delta, B, C) with dout = dy along every path; the projections' gradients as
    ss2d_backward_proj; du_k = the scan's du + x_proj.weight^T dx_dbl; then the conv's backward
    (causal_conv1d_bwd with SiLU): dpre = du * silu'(pre), d conv_weight[k, d, j] = sum over batch
    and steps of dpre[l] x_k[l - (W-1) + j], d conv_bias = sum of dpre, and dx_k[m] =
    sum_j w[k, d, j] dpre[m + (W-1) - j], merged along the paths.
    Returns dict dx, dconv_weight, dconv_bias, dx_proj_weight, ddt_proj_weight, ddt_proj_bias, dA, dD."""
    x, w, Wx, Wdt, dy = _f64(x), _f64(conv_weight), _f64(x_proj_weight), _f64(dt_proj_weight), _f64(dy)
    Bn, Dn, H, W = x.shape
    L = H * W
    R = Wdt.shape[2]
    Wc = w.shape[2]
    u, pre = path_conv(x, conv_weight, conv_bias)
    delta, Bm, Cm, x_dbl = _seq_projections(u, Wx, Wdt)
    g = selective_scan_bwd(u.reshape(Bn, K_PATHS * Dn, L), delta.reshape(Bn, K_PATHS * Dn, L), A, Bm, Cm, D,
                           dt_proj_bias, delta_softplus, cross_scan(dy).reshape(Bn, K_PATHS * Dn, L))
    ddelta = g["ddelta"].reshape(Bn, K_PATHS, Dn, L)
    dx_dbl = np.concatenate([np.einsum("kdr,bkdl->bkrl", Wdt, ddelta), g["dB"], g["dC"]], axis=2)
    ddt_proj_weight = np.einsum("bkdl,bkrl->kdr", ddelta, x_dbl[:, :, :R])
    dx_proj_weight = np.einsum("bkcl,bkdl->kcd", dx_dbl, u)
    du = g["du"].reshape(Bn, K_PATHS, Dn, L) + np.einsum("kcd,bkcl->bkdl", Wx, dx_dbl)
    sig = 1.0 / (1.0 + np.exp(-pre))
    dpre = du * sig * (1.0 + pre * (1.0 - sig))                # silu'(p) = s (1 + p (1 - s))
    xs = cross_scan(x)
    dconv_weight = np.empty_like(w)
    dxs = np.zeros_like(xs)
    for j in range(Wc):
        s = Wc - 1 - j
        dconv_weight[:, :, j] = np.einsum("bkdl,bkdl->kd", dpre[..., s:], xs[..., :L - s])
        dxs[..., :L - s] += w[None, :, :, j, None] * dpre[..., s:]
    dconv_bias = dpre.sum(axis=(0, 3)).reshape(K_PATHS * Dn) if conv_bias is not None else None
    return dict(dx=cross_merge(dxs, H, W), dconv_weight=dconv_weight, dconv_bias=dconv_bias,
                dx_proj_weight=dx_proj_weight, ddt_proj_weight=ddt_proj_weight, ddt_proj_bias=g["ddelta_bias"],
                dA=g["dA"], dD=g["dD"])


# ---------------------------------------------------------------- path sets

def cross_paths(H: int, W: int):
    """(4, H*W) table of the VMamba page's cross scan: row-major, column-major, both reversed."""
    L = H * W
    return np.array([[path_pixel(k, l, H, W) for l in range(L)] for k in range(K_PATHS)], dtype=np.int64)


def diagonal_order(H: int, W: int, direction: int):
    """Pixel order of the diagonal scans of "Visual Mamba实战从零开始搭建图像分类模型附PyTorch代码"
    (section 3, SS2D._get_diagonal_indices): anti-diagonals s = 0 .. H+W-2 in turn, rows i ascending
    within each; column j = s - i for direction > 0, j = (W-1) - (s - i) otherwise."""
    order = []
    for s in range(H + W - 1):
        for i in range(max(0, s - W + 1), min(s + 1, H)):
            j = s - i if direction > 0 else (W - 1) - (s - i)
            order.append(i * W + j)
    return np.array(order, dtype=np.int64)


def diagonal_paths(H: int, W: int):
    """(4, H*W) table: the two diagonal orders, then each of them reversed (paths 2, 3), the same
    structure as the cross scan's path set."""
    d0, d1 = diagonal_order(H, W, 1), diagonal_order(H, W, -1)
    return np.stack([d0, d1, d0[::-1], d1[::-1]]).astype(np.int64)


def _table(table, L):
    t = np.ascontiguousarray(np.asarray(table, dtype=np.int64).reshape(K_PATHS, L))
    return t, t.ctypes.data_as(ctypes.POINTER(ctypes.c_long))


def cross_scan_table(x, table):
    """x (B, D, H, W) -> xs (B, 4, D, L) along the four paths of `table` (4, L)."""
    x = _f64(x)
    Bn, Dn, H, W = x.shape
    t, tp = _table(table, H * W)
    xs = np.empty((Bn, K_PATHS, Dn, H * W), dtype=np.float64)
    _load().oracle_cross_scan_table(Bn, Dn, H * W, tp, _ptr(x), _ptr(xs))
    return xs


def cross_merge_table(ys, H: int, W: int, table):
    ys = _f64(ys)
    Bn, K, Dn, L = ys.shape
    t, tp = _table(table, L)
    y = np.empty((Bn, Dn, H, W), dtype=np.float64)
    _load().oracle_cross_merge_table(Bn, Dn, L, tp, _ptr(ys), _ptr(y))
    return y


def ss2d_forward_table(x, delta, A, B, C, D, delta_bias, delta_softplus, table):
    """SS2D forward over the path set `table` (4, L)."""
    x, delta, A, B, C = (_f64(t) for t in (x, delta, A, B, C))
    D, delta_bias = _f64(D), _f64(delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    t, tp = _table(table, H * W)
    y = np.empty_like(x)
    _load().oracle_ss2d_forward_table(Bn, Dn, H * W, N, tp, _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                      _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y))
    return y


def ss2d_backward_table(x, delta, A, B, C, D, delta_bias, delta_softplus, dy, table):
    x, delta, A, B, C, dy = (_f64(t) for t in (x, delta, A, B, C, dy))
    D, delta_bias = _f64(D), _f64(delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    t, tp = _table(table, H * W)
    dx = np.empty_like(x)
    ddelta = np.empty_like(delta)
    dA = np.empty_like(A)
    dB = np.empty_like(B)
    dC = np.empty_like(C)
    dD = np.empty(K_PATHS * Dn, dtype=np.float64) if D is not None else None
    dbias = np.empty(K_PATHS * Dn, dtype=np.float64) if delta_bias is not None else None
    _load().oracle_ss2d_backward_table(Bn, Dn, H * W, N, tp, _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                       _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dy), _ptr(dx),
                                       _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dbias))
    return dict(dx=dx, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias)


def _flip(t):
    return None if t is None else np.ascontiguousarray(np.flip(t, -1))


def _group_axis(B):
    """B or C given as (Bn, N, L) -> (Bn, 1, N, L); 4-D passes through."""
    return None if B is None else (B[:, None] if B.ndim == 3 else B)


def bimamba_forward(x, delta, A, A_b, B, C, D=None, z=None, delta_bias=None, delta_softplus=True):
    """Bidirectional scan of bimamba_inner_ref ("vision mamba-yolov8", section "2. Vmamba module
    code"): one scan over the sequence with A, one over the flipped sequence with A_b (delta, B,
    C, z flipped too; D and delta_bias shared), the second output flipped back and added.

    x, delta, z (Bn, D, L); A, A_b (D, N); B, C (Bn, N, L) or (Bn, 1, N, L); D, delta_bias (D).
    """
    x, delta, A, A_b, B, C = (_f64(t) for t in (x, delta, A, A_b, B, C))
    D, delta_bias, z = _f64(D), _f64(delta_bias), _f64(z)
    B4, C4 = _group_axis(B), _group_axis(C)
    y = selective_scan_fwd(x, delta, A, B4, C4, D, delta_bias, delta_softplus, z=z)
    y_b = selective_scan_fwd(_flip(x), _flip(delta), A_b, _flip(B4), _flip(C4), D, delta_bias, delta_softplus,
                             z=_flip(z))
    return y + _flip(y_b)


def bimamba_backward(x, delta, A, A_b, B, C, D, z, delta_bias, delta_softplus, dy):
    """Gradients of bimamba_forward: the two scans' backward passes, the flipped one's gradients
    flipped back, shared inputs' gradients added.  Returns dict dx, ddelta, dA, dA_b, dB, dC, dD,
    ddelta_bias, dz (dB, dC in B's and C's shapes; None where an input is None)."""
    x, delta, A, A_b, B, C, dy = (_f64(t) for t in (x, delta, A, A_b, B, C, dy))
    D, delta_bias, z = _f64(D), _f64(delta_bias), _f64(z)
    B4, C4 = _group_axis(B), _group_axis(C)
    gf = selective_scan_bwd(x, delta, A, B4, C4, D, delta_bias, delta_softplus, dy, z=z)
    gb = selective_scan_bwd(_flip(x), _flip(delta), A_b, _flip(B4), _flip(C4), D, delta_bias, delta_softplus,
                            _flip(dy), z=_flip(z))

    def both(name):
        return None if gf[name] is None else gf[name] + _flip(gb[name])

    def total(name):
        return None if gf[name] is None else gf[name] + gb[name]

    dB, dC = both("dB"), both("dC")
    return dict(dx=both("du"), ddelta=both("ddelta"), dA=gf["dA"], dA_b=gb["dA"],
                dB=dB.reshape(B.shape), dC=dC.reshape(C.shape), dD=total("dD"),
                ddelta_bias=total("ddelta_bias"), dz=both("dz"))


def ss2d_forward(x, delta, A, B, C, D=None, delta_bias=None, delta_softplus=True):
    """Full SS2D forward.  x (Bn, D, H, W) -> y (Bn, D, H, W)."""
    x, delta, A, B, C = (_f64(t) for t in (x, delta, A, B, C))
    D, delta_bias = _f64(D), _f64(delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    assert delta.shape == (Bn, K_PATHS * Dn, H * W) and A.shape == (K_PATHS * Dn, N)
    assert B.shape == (Bn, K_PATHS, N, H * W) and C.shape == B.shape
    y = np.empty_like(x)
    _load().oracle_ss2d_forward(Bn, Dn, H, W, N, _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y))
    return y


def ss2d_backward(x, delta, A, B, C, D, delta_bias, delta_softplus, dy):
    """Full SS2D backward.  Returns dict dx, ddelta, dA, dB, dC, dD, ddelta_bias."""
    x, delta, A, B, C, dy = (_f64(t) for t in (x, delta, A, B, C, dy))
    D, delta_bias = _f64(D), _f64(delta_bias)
    Bn, Dn, H, W = x.shape
    N = A.shape[1]
    dx = np.empty_like(x)
    ddelta = np.empty_like(delta)
    dA = np.empty_like(A)
    dB = np.empty_like(B)
    dC = np.empty_like(C)
    dD = np.empty(K_PATHS * Dn, dtype=np.float64) if D is not None else None
    dbias = np.empty(K_PATHS * Dn, dtype=np.float64) if delta_bias is not None else None
    _load().oracle_ss2d_backward(Bn, Dn, H, W, N, _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                 _ptr(D), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dy),
                                 _ptr(dx), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD),
                                 _ptr(dbias))
    return dict(dx=dx, ddelta=ddelta, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias)
