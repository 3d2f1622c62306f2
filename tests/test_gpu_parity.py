"""GPU parity: the CUDA library (called through its C ABI via the binding) against the fp64 oracle.

Bars (element by element on the same seeded inputs):
  * CrossScan / CrossMerge index maps: bit-exact;
  * fp32 forward: |y - y_ref| <= 1e-4 * (1 + |y_ref|);
  * fp32 gradients: relative L2 error <= 1e-4;
  * bf16 inputs: relative L2 error <= 1e-2 against the oracle fed the same bf16-rounded values.
Full-size workloads are compared on sampled batch items (batch items are independent, so
the oracle on a batch slice is exact for those items).
"""
import numpy as np
import pytest
import torch

import oracle
import selective_scan_crossscan_b200 as ss
import ss2d_inputs

pytestmark = pytest.mark.gpu

FWD_TOL = 1e-4
GRAD_TOL = 1e-4
BF16_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from selective_scan_crossscan_b200 import _build
    _build.build()
    oracle.build()
    torch.cuda.set_device(0)


def _np(t):
    return t.detach().to("cpu").double().numpy()


def _dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def assert_fwd_close(y, ref, what=""):
    y = _np(y) if torch.is_tensor(y) else y
    err = np.abs(y - ref)
    bound = FWD_TOL * (1.0 + np.abs(ref))
    worst = np.max(err - bound)
    assert worst <= 0, f"{what}: max excess {worst:.3e}, max err {err.max():.3e}"


# Where the exact reference is identically zero (e.g. dA for L = 1, where no earlier state
# exists) the kernel returns fp32 rounding residue of terms that cancel; those are compared
# at an absolute floor of 1e-9 per element instead of relatively.
ABS_FLOOR = 1e-9


def rel_l2(a, ref):
    a = _np(a) if torch.is_tensor(a) else a
    floor = ABS_FLOOR * np.sqrt(ref.size)
    return float(np.linalg.norm((a - ref).ravel()) / max(np.linalg.norm(ref.ravel()), floor))


def assert_rel_l2(a, ref, tol, what=""):
    r = rel_l2(a, ref)
    assert r <= tol, f"{what}: rel L2 {r:.3e} > {tol}"


# ------------------------------------------------------------ cross scan/merge

SHAPES = [(1, 8, 8, 8), (2, 3, 5, 7), (2, 4, 33, 65), (1, 2, 1, 1), (3, 5, 14, 14), (1, 3, 1, 37), (1, 2, 40, 3)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES)
def test_cross_scan_bit_exact(shape, dtype):
    g = torch.Generator().manual_seed(1)
    x = torch.randn(shape, generator=g).to(dtype)
    xs = ss.cross_scan(x.cuda())
    ref = oracle.cross_scan(x)
    assert xs.dtype == dtype
    np.testing.assert_array_equal(_np(xs), ref)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES)
def test_merge_of_scan_is_exactly_four_x(shape, dtype):
    g = torch.Generator().manual_seed(2)
    x = torch.randn(shape, generator=g).to(dtype).cuda()
    y = ss.cross_merge(ss.cross_scan(x), shape[2], shape[3])
    assert torch.equal(y, 4 * x)


@pytest.mark.parametrize("shape", SHAPES)
def test_cross_merge_index_map_bit_exact(shape):
    # integer-valued tags keep every fp32 sum exact, so any misplaced element shows
    Bn, Dn, H, W = shape
    g = torch.Generator().manual_seed(3)
    ys = torch.randint(-1000, 1000, (Bn, 4, Dn, H * W), generator=g).float()
    y = ss.cross_merge(ys.cuda(), H, W)
    np.testing.assert_array_equal(_np(y), oracle.cross_merge(ys, H, W))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_cross_merge_random_values(out_dtype):
    Bn, Dn, H, W = 2, 3, 9, 11
    g = torch.Generator().manual_seed(4)
    ys = torch.randn((Bn, 4, Dn, H * W), generator=g)
    y = ss.cross_merge(ys.cuda(), H, W, out_dtype=out_dtype)
    ref = oracle.cross_merge(ys, H, W)
    tol = 1e-6 if out_dtype == torch.float32 else 8e-3
    np.testing.assert_allclose(_np(y), ref, rtol=tol, atol=tol)


# --------------------------------------------------------------- S6 forward

def _scan_case(Bn, Dn, H, W, N, dtype="f32", seed=0):
    w = ss2d_inputs.custom(Bn, Dn, H, W, N, dtype=dtype)
    return w, ss2d_inputs.make_scan_inputs(w, seed=seed, with_dout=True)


SCAN_CASES = [(1, 8, 8, 8, 4), (2, 70, 5, 7, 16), (1, 3, 1, 1, 3), (2, 16, 3, 45, 8), (1, 64, 9, 15, 1),
              (1, 5, 16, 20, 16), (3, 2, 2, 2, 5)]


@pytest.mark.parametrize("case", SCAN_CASES)
def test_selective_scan_fwd_parity(case):
    w, inp = _scan_case(*case)
    d = _dev(inp)
    y = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    ref = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True)
    assert_fwd_close(y, ref, str(case))


@pytest.mark.parametrize("opts", [dict(D=False, bias=True, sp=True), dict(D=True, bias=False, sp=True),
                                  dict(D=False, bias=False, sp=False)])
def test_selective_scan_fwd_optional_inputs(opts):
    w, inp = _scan_case(2, 8, 6, 6, 8, seed=5)
    if not opts["sp"]:
        inp["delta"] = inp["delta"].abs() * 0.5 + 0.01  # positive step sizes without softplus
    D = inp["D"] * 0.5 if opts["D"] else None
    bias = inp["delta_bias"] if opts["bias"] else None
    d = _dev(inp)
    y = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], None if D is None else D.cuda(),
                              None if bias is None else bias.cuda(), opts["sp"])
    ref = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D, bias, opts["sp"])
    assert_fwd_close(y, ref, str(opts))


def test_selective_scan_fwd_chunk_states():
    # chunk j holds h after step min(16 (j+1), L) - 1: the oracle's last state on the truncated sequence
    w, inp = _scan_case(1, 4, 10, 20, 16, seed=6)  # L = 200 -> 13 chunks, ragged last one
    d = _dev(inp)
    y, cs = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                  return_chunk_states=True)
    assert cs.shape == (1, 16, 13, 16)
    for j, end in [(0, 16), (5, 96), (11, 192), (12, 200)]:
        _, last = oracle.selective_scan_fwd(inp["u"][..., :end], inp["delta"][..., :end], inp["A"],
                                            inp["B"][..., :end], inp["C"][..., :end], inp["D"], inp["delta_bias"],
                                            True, return_last_state=True)
        assert_rel_l2(cs[:, :, j], last, 1e-5, f"chunk {j}")


def test_selective_scan_fwd_bf16():
    w, inp = _scan_case(2, 16, 7, 7, 16, dtype="bf16", seed=7)
    d = _dev(inp)
    y = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    assert y.dtype == torch.bfloat16
    ref = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True)
    assert_rel_l2(y, ref, BF16_TOL)


# -------------------------------------------------------------- S6 backward

BWD_NAMES = [("du", "du"), ("ddelta", "ddelta"), ("dA", "dA"), ("dB", "dB"), ("dC", "dC"), ("dD", "dD"),
             ("ddelta_bias", "ddelta_bias")]


@pytest.mark.parametrize("case", [(1, 8, 8, 8, 4), (2, 40, 5, 7, 16), (1, 3, 1, 1, 3), (1, 33, 4, 50, 8),
                                  (2, 4, 3, 43, 16)])
@pytest.mark.parametrize("with_states", [False, True])
def test_selective_scan_bwd_parity(case, with_states):
    w, inp = _scan_case(*case, seed=8)
    d = _dev(inp)
    cs = None
    if with_states:
        _, cs = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                      return_chunk_states=True)
    g = ss.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, d["dout"],
                              chunk_states=cs)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, inp["dout"])
    for name, rname in BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], GRAD_TOL, f"{case} {name}")


def test_selective_scan_bwd_without_optional():
    w, inp = _scan_case(1, 8, 6, 11, 8, seed=9)
    d = _dev(inp)
    g = ss.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], None, None, True, d["dout"])
    assert g["dD"] is None and g["ddelta_bias"] is None
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], None, None, True,
                                    inp["dout"])
    for name in ("du", "ddelta", "dA", "dB", "dC"):
        assert_rel_l2(g[name], ref[name], GRAD_TOL, name)


# ------------------------------------------- output gate and last state

def _gated_case(Bn, Dn, H, W, N, dtype="f32", seed=0):
    w = ss2d_inputs.custom(Bn, Dn, H, W, N, dtype=dtype)
    return w, ss2d_inputs.make_scan_inputs(w, seed=seed, with_dout=True, with_z=True)


GATED_CASES = [(1, 8, 8, 8, 4), (2, 40, 5, 7, 16), (1, 3, 1, 1, 3), (1, 33, 4, 50, 8), (2, 4, 3, 43, 16)]


@pytest.mark.parametrize("case", GATED_CASES)
def test_selective_scan_fwd_gate_and_last_state(case):
    w, inp = _gated_case(*case, seed=30)
    d = _dev(inp)
    out, last, cs = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                          z=d["z"], return_last_state=True, return_chunk_states=True)
    ref, ref_last = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                              inp["delta_bias"], True, return_last_state=True, z=inp["z"])
    assert_fwd_close(out, ref, f"{case} out")
    assert_fwd_close(last, ref_last, f"{case} last_state")
    # the last state is the final chunk state, bit for bit
    assert torch.equal(last, cs[:, :, -1, :])


def test_last_state_without_gate_and_gate_without_last_state():
    w, inp = _gated_case(2, 6, 7, 9, 16, seed=31)
    d = _dev(inp)
    plain = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    out, last = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                      return_last_state=True)
    assert torch.equal(out, plain)  # the last state changes nothing else
    _, ref_last = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                            inp["delta_bias"], True, return_last_state=True)
    assert_fwd_close(last, ref_last, "last_state")
    gated = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                  z=d["z"])
    ref = oracle.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, z=inp["z"])
    assert_fwd_close(gated, ref, "gated out")


def test_gate_extremes():
    # z = 0 gives exactly 0; very negative z gives (-)0, not NaN; large z passes the output through
    w, inp = _gated_case(1, 4, 4, 16, 8, seed=32)
    d = _dev(inp)
    args = (d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    plain = ss.selective_scan_fwd(*args)
    assert torch.all(ss.selective_scan_fwd(*args, z=torch.zeros_like(d["u"])) == 0)
    neg = ss.selective_scan_fwd(*args, z=torch.full_like(d["u"], -200.0))
    assert torch.all(neg == 0) and not torch.isnan(neg).any()
    big = ss.selective_scan_fwd(*args, z=torch.full_like(d["u"], 60.0))
    torch.testing.assert_close(big, 60.0 * plain, rtol=2e-6, atol=0)


GATED_BWD_NAMES = BWD_NAMES + [("dz", "dz")]


@pytest.mark.parametrize("case", GATED_CASES)
@pytest.mark.parametrize("with_states", [False, True])
def test_selective_scan_bwd_gated_parity(case, with_states):
    w, inp = _gated_case(*case, seed=33)
    d = _dev(inp)
    cs = None
    if with_states:
        _, cs = ss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                      z=d["z"], return_chunk_states=True)
    g = ss.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, d["dout"],
                              chunk_states=cs, z=d["z"])
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, inp["dout"], z=inp["z"])
    for name, rname in GATED_BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], GRAD_TOL, f"{case} {name}")


def test_gated_bwd_bf16():
    w, inp = _gated_case(2, 8, 6, 20, 16, dtype="bf16", seed=34)
    d = _dev(inp)
    g = ss.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, d["dout"],
                              z=d["z"])
    assert g["dz"].dtype == torch.bfloat16
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, inp["dout"], z=inp["z"])
    for name, rname in GATED_BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], BF16_TOL, name)


def test_selective_scan_fn_autograd():
    # the pages' selective_scan_fn call: gated output and last state; backward through autograd
    w, inp = _gated_case(2, 5, 6, 13, 16, seed=35)
    d = _dev(inp)
    leaves = {k: d[k].clone().requires_grad_(True) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    out, last = ss.selective_scan_fn(leaves["u"], leaves["delta"], leaves["A"], leaves["B"], leaves["C"],
                                     leaves["D"], z=leaves["z"], delta_bias=leaves["delta_bias"],
                                     delta_softplus=True, return_last_state=True)
    assert not last.requires_grad
    out.backward(d["dout"])
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, inp["dout"], z=inp["z"])
    names = dict(u="du", delta="ddelta", A="dA", B="dB", C="dC", D="dD", z="dz", delta_bias="ddelta_bias")
    for k, rname in names.items():
        assert_rel_l2(leaves[k].grad, ref[rname], GRAD_TOL, k)


# ------------------------------------------------------- bidirectional scan

def _bidir_case(Bn, Dn, L, N, dtype="f32", seed=0, with_z=True):
    w = ss2d_inputs.custom(Bn, Dn, 1, L, N, dtype=dtype, a_init="s4d_real", kind="bidir")
    return w, ss2d_inputs.make_bimamba_inputs(w, seed=seed, with_dy=True, with_z=with_z, distinct_a_b=True)


# L = 1, ragged L (scalar staging), several 16-step blocks and 64-channel tiles, N < 16
BIDIR_CASES = [(1, 8, 16, 4), (2, 40, 37, 16), (1, 3, 1, 3), (2, 70, 200, 16), (1, 5, 197, 8), (3, 33, 64, 16)]
BIDIR_BWD_NAMES = ["dx", "ddelta", "dA", "dA_b", "dB", "dC", "dD", "ddelta_bias", "dz"]


def _bidir_ref_fwd(inp, z=True):
    return oracle.bimamba_forward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], inp["D"],
                                  inp["z"] if z else None, inp["delta_bias"], True)


@pytest.mark.parametrize("case", BIDIR_CASES)
@pytest.mark.parametrize("gated", [True, False])
def test_bimamba_forward_parity(case, gated):
    w, inp = _bidir_case(*case, seed=40, with_z=gated)
    d = _dev(inp)
    y = ss.bimamba_forward(d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"], d["D"], d.get("z"),
                           d["delta_bias"], True)
    assert_fwd_close(y, _bidir_ref_fwd(inp, gated), f"{case} y")


@pytest.mark.parametrize("case", BIDIR_CASES)
@pytest.mark.parametrize("with_states", [False, True])
def test_bimamba_backward_parity(case, with_states):
    w, inp = _bidir_case(*case, seed=41)
    d = _dev(inp)
    args = (d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"], True)
    cs = None
    if with_states:
        _, cs = ss.bimamba_forward(*args, return_chunk_states=True)
    g = ss.bimamba_backward(*args, d["dy"], chunk_states=cs)
    ref = oracle.bimamba_backward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, inp["dy"])
    for name in BIDIR_BWD_NAMES:
        assert_rel_l2(g[name], ref[name], GRAD_TOL, f"{case} {name}")


def test_bimamba_without_optional_inputs():
    w, inp = _bidir_case(2, 12, 45, 16, seed=42, with_z=False)
    d = _dev(inp)
    y = ss.bimamba_forward(d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"])
    ref = oracle.bimamba_forward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"])
    assert_fwd_close(y, ref, "y")
    g = ss.bimamba_backward(d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"], None, None, None, True, d["dy"])
    assert g["dD"] is None and g["ddelta_bias"] is None and g["dz"] is None
    r = oracle.bimamba_backward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], None, None, None,
                                True, inp["dy"])
    for name in ("dx", "ddelta", "dA", "dA_b", "dB", "dC"):
        assert_rel_l2(g[name], r[name], GRAD_TOL, name)


def test_bimamba_bf16():
    w, inp = _bidir_case(2, 16, 60, 16, dtype="bf16", seed=43)
    d = _dev(inp)
    args = (d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"], True)
    y = ss.bimamba_forward(*args)
    assert y.dtype == torch.bfloat16
    assert_rel_l2(y, _bidir_ref_fwd(inp), BF16_TOL, "y")
    g = ss.bimamba_backward(*args, d["dy"])
    ref = oracle.bimamba_backward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, inp["dy"])
    for name in BIDIR_BWD_NAMES:
        assert_rel_l2(g[name], ref[name], BF16_TOL, name)


def test_bimamba_autograd():
    w, inp = _bidir_case(2, 6, 29, 16, seed=44)
    d = _dev(inp)
    names = ("x", "delta", "A", "A_b", "B", "C", "D", "z", "delta_bias")
    leaves = {k: d[k].clone().requires_grad_(True) for k in names}
    y = ss.bimamba_scan(leaves["x"], leaves["delta"], leaves["A"], leaves["A_b"], leaves["B"], leaves["C"],
                        leaves["D"], leaves["z"], leaves["delta_bias"], True)
    y.backward(d["dy"])
    ref = oracle.bimamba_backward(inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, inp["dy"])
    gmap = dict(x="dx", delta="ddelta", A="dA", A_b="dA_b", B="dB", C="dC", D="dD", z="dz",
                delta_bias="ddelta_bias")
    for k, rname in gmap.items():
        assert_rel_l2(leaves[k].grad, ref[rname], GRAD_TOL, k)


def test_bimamba_full_vim_workload_sampled():
    # the benchmark's bidirectional workload at full size, in the launch configuration bench.py
    # times; batch items checked one by one against the oracle
    w = ss2d_inputs.workload("vim_t_bidir_fp32")
    inp = ss2d_inputs.make_bimamba_inputs(w, seed=5, with_dy=True, with_z=True, distinct_a_b=True)
    d = _dev(inp)
    args = (d["x"], d["delta"], d["A"], d["A_b"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"], True)
    y, cs = ss.bimamba_forward(*args, return_chunk_states=True)
    g = ss.bimamba_backward(*args, d["dy"], chunk_states=cs)
    for bi in (0, 77, w.batch - 1):
        sl = ss2d_inputs.batch_slice(inp, [bi])
        ref_y = oracle.bimamba_forward(sl["x"], sl["delta"], sl["A"], sl["A_b"], sl["B"], sl["C"], sl["D"],
                                       sl["z"], sl["delta_bias"], True)
        assert_fwd_close(y[bi:bi + 1], ref_y, f"y[{bi}]")
        r = oracle.bimamba_backward(sl["x"], sl["delta"], sl["A"], sl["A_b"], sl["B"], sl["C"], sl["D"], sl["z"],
                                    sl["delta_bias"], True, sl["dy"])
        for name in ("dx", "ddelta", "dB", "dC", "dz"):
            assert_rel_l2(g[name][bi:bi + 1], r[name], GRAD_TOL, f"{name}[{bi}]")


# ---------------------------------------------------- path sets as tables

# ragged planes, one-row and one-column maps, a 14x14 plane, and a plane too large for the
# shared-memory merge (100 x 100)
TABLE_SHAPES = [(1, 2, 3, 4), (2, 3, 5, 7), (1, 2, 1, 9), (1, 3, 8, 1), (2, 4, 14, 14), (1, 2, 100, 100)]


@pytest.mark.parametrize("H,W", [(3, 4), (1, 7), (6, 1), (14, 14), (13, 37), (56, 56)])
@pytest.mark.parametrize("kind", ["cross", "diagonal"])
def test_path_tables_match_oracle(H, W, kind):
    t = ss.path_tables(H, W, ss.PATHS_DIAGONAL if kind == "diagonal" else ss.PATHS_CROSS)
    ref = oracle.diagonal_paths(H, W) if kind == "diagonal" else oracle.cross_paths(H, W)
    got = _np(t).astype(np.int64)
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[1], ref[1])
    L = H * W
    for k in range(2):  # rows 2, 3: inverse permutations
        np.testing.assert_array_equal(got[2 + k][ref[k]], np.arange(L))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", TABLE_SHAPES)
def test_cross_scan_table_bit_exact(shape, dtype):
    Bn, Dn, H, W = shape
    g = torch.Generator().manual_seed(11)
    x = torch.randn(shape, generator=g).to(dtype)
    t = ss.path_tables(H, W, ss.PATHS_DIAGONAL)
    xs = ss.cross_scan_table(x.cuda(), t)
    np.testing.assert_array_equal(_np(xs), oracle.cross_scan_table(x, oracle.diagonal_paths(H, W)))


@pytest.mark.parametrize("shape", TABLE_SHAPES)
def test_cross_merge_table_bit_exact(shape):
    Bn, Dn, H, W = shape
    g = torch.Generator().manual_seed(12)
    ys = torch.randint(-1000, 1000, (Bn, 4, Dn, H * W), generator=g).float()
    t = ss.path_tables(H, W, ss.PATHS_DIAGONAL)
    y = ss.cross_merge_table(ys.cuda(), H, W, t)
    np.testing.assert_array_equal(_np(y), oracle.cross_merge_table(ys, H, W, oracle.diagonal_paths(H, W)))
    x = torch.randn((Bn, Dn, H, W), generator=g).cuda()
    assert torch.equal(ss.cross_merge_table(ss.cross_scan_table(x, t), H, W, t), 4 * x)


def test_cross_table_equals_the_fixed_cross_path():
    # the table machinery over the cross set gives the fixed path's results bit for bit
    Bn, Dn, H, W, N = 2, 6, 9, 11, 16
    w = ss2d_inputs.custom(Bn, Dn, H, W, N)
    inp = ss2d_inputs.make_inputs(w, seed=13, with_dy=True)
    d = _dev(inp)
    t = ss.path_tables(H, W, ss.PATHS_CROSS)
    args = (d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    assert torch.equal(ss.cross_scan_table(d["x"], t), ss.cross_scan(d["x"]))
    assert torch.equal(ss.ss2d_forward_table(*args, t), ss.ss2d_forward(*args))
    g1 = ss.ss2d_backward_table(*args, d["dy"], t)
    g2 = ss.ss2d_backward(*args, d["dy"])
    for name in g1:
        assert torch.equal(g1[name], g2[name]), name


DIAG_CASES = [(1, 8, 8, 8, 4), (2, 6, 5, 9, 16), (1, 70, 12, 11, 16), (2, 3, 1, 1, 2), (1, 4, 3, 100, 8),
              (1, 2, 100, 100, 16)]


@pytest.mark.parametrize("case", DIAG_CASES)
def test_ss2d_forward_diagonal_parity(case):
    Bn, Dn, H, W, N = case
    w = ss2d_inputs.custom(Bn, Dn, H, W, N)
    inp = ss2d_inputs.make_inputs(w, seed=14)
    d = _dev(inp)
    t = ss.path_tables(H, W, ss.PATHS_DIAGONAL)
    y = ss.ss2d_forward_table(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, t)
    ref = oracle.ss2d_forward_table(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, oracle.diagonal_paths(H, W))
    assert_fwd_close(y, ref, f"{case} y")


@pytest.mark.parametrize("case", DIAG_CASES[:5])
@pytest.mark.parametrize("with_states", [False, True])
def test_ss2d_backward_diagonal_parity(case, with_states):
    Bn, Dn, H, W, N = case
    w = ss2d_inputs.custom(Bn, Dn, H, W, N)
    inp = ss2d_inputs.make_inputs(w, seed=15, with_dy=True)
    d = _dev(inp)
    t = ss.path_tables(H, W, ss.PATHS_DIAGONAL)
    args = (d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    cs = None
    if with_states:
        _, cs = ss.ss2d_forward_table(*args, t, return_chunk_states=True)
    g = ss.ss2d_backward_table(*args, d["dy"], t, chunk_states=cs)
    ref = oracle.ss2d_backward_table(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                     inp["delta_bias"], True, inp["dy"], oracle.diagonal_paths(H, W))
    for name, rname in SS2D_BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], GRAD_TOL, f"{case} {name}")


def test_ss2d_diagonal_bf16_and_autograd():
    w = ss2d_inputs.custom(1, 8, 12, 12, 16, dtype="bf16", a_init="s4d_real")
    inp = ss2d_inputs.make_inputs(w, seed=16, with_dy=True)
    d = _dev(inp)
    t = ss.path_tables(12, 12, ss.PATHS_DIAGONAL)
    tab = oracle.diagonal_paths(12, 12)
    y = ss.ss2d_forward_table(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, t)
    ref = oracle.ss2d_forward_table(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["delta_bias"], True, tab)
    assert_rel_l2(y, ref, BF16_TOL, "y bf16")
    # autograd through ss2d(..., tables=) in fp32
    w = ss2d_inputs.custom(1, 4, 6, 7, 8)
    inp = ss2d_inputs.make_inputs(w, seed=17, with_dy=True)
    d = _dev(inp)
    t = ss.path_tables(6, 7, ss.PATHS_DIAGONAL)
    names = ("x", "delta", "A", "B", "C", "D", "delta_bias")
    leaves = {k: d[k].clone().requires_grad_(True) for k in names}
    y = ss.ss2d(leaves["x"], leaves["delta"], leaves["A"], leaves["B"], leaves["C"], leaves["D"],
                leaves["delta_bias"], True, tables=t)
    y.backward(d["dy"])
    ref = oracle.ss2d_backward_table(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                     inp["delta_bias"], True, inp["dy"], oracle.diagonal_paths(6, 7))
    gmap = dict(x="dx", delta="ddelta", A="dA", B="dB", C="dC", D="dD", delta_bias="ddelta_bias")
    for k, rname in gmap.items():
        assert_rel_l2(leaves[k].grad, ref[rname], GRAD_TOL, k)


def test_ss2d_diagonal_full_stage1_sampled():
    # VMamba-T stage-1 shapes over the diagonal path set, batch items checked one by one
    w = ss2d_inputs.workload("vmamba_t_stage1_fp32")
    inp = ss2d_inputs.make_inputs(w, seed=18)
    d = _dev(inp)
    t = ss.path_tables(w.height, w.width, ss.PATHS_DIAGONAL)
    y = ss.ss2d_forward_table(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, t)
    tab = oracle.diagonal_paths(w.height, w.width)
    for bi in (0, 63, w.batch - 1):
        sl = ss2d_inputs.batch_slice(inp, [bi])
        ref = oracle.ss2d_forward_table(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], sl["D"], sl["delta_bias"],
                                        True, tab)
        assert_fwd_close(y[bi:bi + 1], ref, f"y[{bi}]")


# ----------------------------------------------------- producer projections

def _proj_case(Bn, Dn, H, W, N, dtype="f32", seed=0):
    w = ss2d_inputs.custom(Bn, Dn, H, W, N, dtype=dtype, a_init="s4d_real")
    return w, ss2d_inputs.make_proj_inputs(w, seed=seed)


# R = ceil(D / 32): D = 8 -> 1, 70 -> 3, 192 -> 6, 512 -> 8; ragged and one-pixel maps, N < 16
PROJ_CASES = [(1, 8, 8, 8, 4), (2, 70, 5, 9, 16), (1, 40, 12, 11, 8), (2, 6, 1, 1, 16), (1, 192, 14, 14, 16),
              (1, 512, 4, 6, 16)]


@pytest.mark.parametrize("case", PROJ_CASES)
def test_ss2d_forward_proj_parity(case):
    w, inp = _proj_case(*case, seed=50)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"],
                                    d["D"], True, return_x_dbl=True)
    _, _, _, ref_dbl = oracle.path_projections(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"])
    assert_fwd_close(x_dbl, ref_dbl, f"{case} x_dbl")
    ref = oracle.ss2d_forward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                   inp["A"], inp["D"], True)
    assert_fwd_close(y, ref, f"{case} y")


def test_ss2d_forward_proj_matches_materialised_delta():
    # the in-kernel dt projection against the plain fused forward fed the same projections
    w, inp = _proj_case(2, 24, 9, 10, 16, seed=51)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"],
                                    d["D"], True, return_x_dbl=True)
    R, N = inp["R"], w.d_state
    xd = x_dbl.double()
    delta = torch.einsum("kdr,bkrl->bkdl", d["dt_proj_weight"].double(), xd[:, :, :R]).reshape(2, 4 * 24, 90)
    y2 = ss.ss2d_forward(d["x"], delta.float(), d["A"], x_dbl[:, :, R:R + N].contiguous(),
                         x_dbl[:, :, R + N:].contiguous(), d["D"], d["dt_proj_bias"], True)
    torch.testing.assert_close(y, y2, rtol=1e-5, atol=1e-5)


def test_ss2d_forward_proj_bf16_and_full_stage1_sampled():
    w, inp = _proj_case(2, 16, 12, 12, 16, dtype="bf16", seed=52)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"])
    ref = oracle.ss2d_forward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                   inp["A"], inp["D"], True)
    assert_rel_l2(y, ref, BF16_TOL, "y bf16")
    # VMamba-T stage-1 shapes in the launch configuration bench.py times, sampled batch items
    w = ss2d_inputs.workload("vmamba_t_stage1_fp32")
    inp = ss2d_inputs.make_proj_inputs(w, seed=53)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"])
    for bi in (0, w.batch - 1):
        ref = oracle.ss2d_forward_proj(inp["x"][bi:bi + 1], inp["x_proj_weight"], inp["dt_proj_weight"],
                                       inp["dt_proj_bias"], inp["A"], inp["D"], True)
        assert_fwd_close(y[bi:bi + 1], ref, f"y[{bi}]")


PROJ_BWD_CASES = [(1, 8, 8, 8, 4), (2, 70, 5, 9, 16), (2, 6, 1, 1, 16), (1, 40, 33, 35, 8), (1, 192, 14, 14, 16),
                  (1, 512, 4, 6, 16)]


@pytest.mark.parametrize("case", PROJ_BWD_CASES)
def test_ss2d_backward_proj_parity(case):
    w, inp = _proj_case(*case, seed=54)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"],
                                    d["D"], True, return_x_dbl=True)
    g = torch.Generator().manual_seed(55)
    dy_np = torch.randn(tuple(y.shape), generator=g, dtype=torch.float32).double().numpy()
    got = ss.ss2d_backward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"],
                                x_dbl, torch.as_tensor(dy_np, dtype=torch.float32, device="cuda"), True)
    ref = oracle.ss2d_backward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                    inp["A"], inp["D"], True, dy_np)
    for name in ("dx", "dx_proj_weight", "ddt_proj_weight", "ddt_proj_bias", "dA", "dD"):
        assert_rel_l2(got[name], ref[name], GRAD_TOL, f"{case} {name}")


def test_ss2d_backward_proj_wide_rank_bf16_and_chunk_states():
    # dt rank 24 (d_model 384), more tokens than one weight-gradient chunk, forward chunk states reused
    w, inp = _proj_case(1, 768, 36, 30, 16, seed=56)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl, cs = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"],
                                        d["A"], d["D"], True, return_x_dbl=True, return_chunk_states=True)
    dy = torch.randn(y.shape, generator=torch.Generator(device="cuda").manual_seed(57), device="cuda")
    a = ss.ss2d_backward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"],
                              x_dbl, dy, True)
    b = ss.ss2d_backward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"],
                              x_dbl, dy, True, chunk_states=cs)
    for k in a:
        torch.testing.assert_close(a[k], b[k], rtol=1e-5, atol=1e-6)
    ref = oracle.ss2d_backward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                    inp["A"], inp["D"], True, dy.double().cpu().numpy())
    for name in ("dx", "dx_proj_weight", "ddt_proj_weight", "ddt_proj_bias", "dA", "dD"):
        assert_rel_l2(a[name], ref[name], GRAD_TOL, name)
    # bf16 activations: relative L2 against the oracle on the bf16-rounded inputs
    w, inp = _proj_case(2, 16, 12, 12, 16, dtype="bf16", seed=58)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"],
                                    d["D"], True, return_x_dbl=True)
    dy_np = torch.randn(tuple(y.shape), generator=torch.Generator().manual_seed(59), dtype=torch.float64)
    dy_np = dy_np.to(torch.bfloat16).double().numpy()
    got = ss.ss2d_backward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"],
                                x_dbl, torch.as_tensor(dy_np, device="cuda").to(torch.bfloat16), True)
    ref = oracle.ss2d_backward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                    inp["A"], inp["D"], True, dy_np)
    for name in ("dx", "dx_proj_weight", "ddt_proj_weight", "ddt_proj_bias", "dA", "dD"):
        assert_rel_l2(got[name], ref[name], BF16_TOL, f"{name} bf16")


def test_ss2d_backward_proj_deterministic():
    w, inp = _proj_case(2, 64, 20, 24, 16, seed=60)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"],
                                    d["D"], True, return_x_dbl=True)
    dy = torch.randn(y.shape, generator=torch.Generator(device="cuda").manual_seed(61), device="cuda")
    runs = [ss.ss2d_backward_proj(d["x"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"], d["A"], d["D"],
                                  x_dbl, dy, True) for _ in range(2)]
    for k in runs[0]:
        assert torch.equal(runs[0][k], runs[1][k]), k


# ---------------------------------------- producer with its causal conv per path

CONV_NAMES = ("dx", "dconv_weight", "dconv_bias", "dx_proj_weight", "ddt_proj_weight", "ddt_proj_bias", "dA", "dD")

# (Bn, D, H, W, N, d_conv): L % 4 != 0 (plain-load paths), one-pixel maps, every conv width, wide rank
CONV_CASES = [(1, 8, 8, 8, 4, 4), (2, 70, 5, 9, 16, 4), (2, 6, 1, 1, 16, 3), (1, 40, 12, 11, 8, 2),
              (1, 192, 14, 14, 16, 4), (1, 16, 6, 7, 16, 1), (1, 768, 6, 8, 16, 4)]


def _conv_case(Bn, Dn, H, W, N, d_conv, dtype="f32", seed=0):
    w = ss2d_inputs.custom(Bn, Dn, H, W, N, dtype=dtype, a_init="s4d_real")
    return w, ss2d_inputs.make_proj_inputs(w, seed=seed, d_conv=d_conv)


def _conv_call_args(d):
    return (d["x"], d["conv_weight"], d["conv_bias"], d["x_proj_weight"], d["dt_proj_weight"], d["dt_proj_bias"],
            d["A"], d["D"])


@pytest.mark.parametrize("case", CONV_CASES)
def test_ss2d_proj_conv_forward_backward_parity(case):
    w, inp = _conv_case(*case, seed=62)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj_conv(*_conv_call_args(d), True, return_x_dbl=True)
    ref = oracle.ss2d_forward_proj_conv(*_conv_call_args(inp), True)
    assert_fwd_close(y, ref, f"{case} y")
    u, _ = oracle.path_conv(inp["x"], inp["conv_weight"], inp["conv_bias"])
    ref_dbl = np.einsum("bkdl,kcd->bkcl", u, inp["x_proj_weight"].double().numpy())
    assert_fwd_close(x_dbl, ref_dbl, f"{case} x_dbl")
    dy_np = torch.randn(tuple(y.shape), generator=torch.Generator().manual_seed(63),
                        dtype=torch.float32).double().numpy()
    got = ss.ss2d_backward_proj_conv(*_conv_call_args(d), x_dbl, torch.as_tensor(dy_np, dtype=torch.float32,
                                                                                  device="cuda"), True)
    refg = oracle.ss2d_backward_proj_conv(*_conv_call_args(inp), True, dy_np)
    for name in CONV_NAMES:
        assert_rel_l2(got[name], refg[name], GRAD_TOL, f"{case} {name}")


def test_ss2d_proj_conv_without_bias_bf16_and_deterministic():
    w, inp = _conv_case(2, 24, 9, 10, 16, 4, seed=64)
    inp["conv_bias"] = None
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items() if k != "R"}
    y, x_dbl, cs = ss.ss2d_forward_proj_conv(*_conv_call_args(d), True, return_x_dbl=True, return_chunk_states=True)
    assert_fwd_close(y, oracle.ss2d_forward_proj_conv(*_conv_call_args(inp), True), "y without conv bias")
    dy = torch.randn(y.shape, generator=torch.Generator(device="cuda").manual_seed(65), device="cuda")
    runs = [ss.ss2d_backward_proj_conv(*_conv_call_args(d), x_dbl, dy, True, chunk_states=cs) for _ in range(2)]
    assert runs[0]["dconv_bias"] is None
    for k in runs[0]:
        if runs[0][k] is not None:
            assert torch.equal(runs[0][k], runs[1][k]), k
    refg = oracle.ss2d_backward_proj_conv(*_conv_call_args(inp), True, dy.double().cpu().numpy())
    for name in CONV_NAMES:
        if name != "dconv_bias":
            assert_rel_l2(runs[0][name], refg[name], GRAD_TOL, f"{name} without conv bias")
    # bf16 activations against the oracle on the bf16-rounded inputs
    w, inp = _conv_case(2, 16, 12, 12, 16, 4, dtype="bf16", seed=66)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y, x_dbl = ss.ss2d_forward_proj_conv(*_conv_call_args(d), True, return_x_dbl=True)
    assert_rel_l2(y, oracle.ss2d_forward_proj_conv(*_conv_call_args(inp), True), BF16_TOL, "y bf16")
    dy_np = torch.randn(tuple(y.shape), generator=torch.Generator().manual_seed(67), dtype=torch.float64)
    dy_np = dy_np.to(torch.bfloat16).double().numpy()
    got = ss.ss2d_backward_proj_conv(*_conv_call_args(d), x_dbl,
                                     torch.as_tensor(dy_np, device="cuda").to(torch.bfloat16), True)
    refg = oracle.ss2d_backward_proj_conv(*_conv_call_args(inp), True, dy_np)
    for name in CONV_NAMES:
        assert_rel_l2(got[name], refg[name], BF16_TOL, f"{name} bf16")


def test_ss2d_proj_conv_full_stage1_sampled():
    # VMamba-T stage-1 shapes in the launch configuration bench.py times, sampled batch items
    w = ss2d_inputs.workload("vmamba_t_stage1_fp32")
    inp = ss2d_inputs.make_proj_inputs(w, seed=68, d_conv=4)
    d = _dev({k: v for k, v in inp.items() if k != "R"})
    y = ss.ss2d_forward_proj_conv(*_conv_call_args(d), True)
    for bi in (0, w.batch - 1):
        sl = dict(inp, x=inp["x"][bi:bi + 1])
        assert_fwd_close(y[bi:bi + 1], oracle.ss2d_forward_proj_conv(*_conv_call_args(sl), True), f"y[{bi}]")


# ------------------------------------------------------------- fused SS2D

FUSED_CASES = [(1, 8, 8, 8, 4), (2, 6, 5, 9, 16), (1, 70, 12, 11, 16), (1, 8, 64, 64, 16), (2, 3, 1, 1, 2),
               (1, 4, 3, 100, 8)]


@pytest.mark.parametrize("case", FUSED_CASES)
def test_ss2d_forward_parity(case):
    Bn, Dn, H, W, N = case
    w = ss2d_inputs.custom(Bn, Dn, H, W, N)
    inp = ss2d_inputs.make_inputs(w, seed=10)
    d = _dev(inp)
    y = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    ref = oracle.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                              True)
    assert_fwd_close(y, ref, str(case))


def test_ss2d_forward_tiny_workload():
    w = ss2d_inputs.workload(0)
    inp = ss2d_inputs.make_inputs(w, seed=0)
    d = _dev(inp)
    y, cs = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                            return_chunk_states=True)
    ref = oracle.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                              True)
    assert_fwd_close(y, ref, "tiny")
    # the last chunk state is the final state of each of the 4*D path sequences
    xs = oracle.cross_scan(inp["x"]).reshape(1, 32, 64)
    _, last = oracle.selective_scan_fwd(xs, inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                                        True, return_last_state=True)
    assert_rel_l2(cs[:, :, -1], last, 1e-5, "last state")


def test_ss2d_forward_bf16():
    w = ss2d_inputs.custom(2, 16, 14, 14, 16, dtype="bf16", a_init="s4d_real")
    inp = ss2d_inputs.make_inputs(w, seed=11)
    d = _dev(inp)
    y = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    assert y.dtype == torch.bfloat16
    ref = oracle.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                              True)
    assert_rel_l2(y, ref, BF16_TOL)


@pytest.mark.parametrize("H,W", [(4, 8), (7, 9)])
def test_unfused_pipeline_equals_fused(H, W):
    # single pass on both sides (L <= 32): bit-identical; longer sequences of a small problem are
    # split into segments by the fused forward, whose carries round differently: within 1e-5
    w = ss2d_inputs.custom(2, 8, H, W, 16)
    L = H * W
    d = _dev(ss2d_inputs.make_inputs(w, seed=12))
    y = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    xs = ss.cross_scan(d["x"]).reshape(2, 32, L)
    ys = ss.selective_scan_fwd(xs, d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    y2 = ss.cross_merge(ys.reshape(2, 4, 8, L), H, W)
    if L <= 32:
        assert torch.equal(y, y2)
    else:
        torch.testing.assert_close(y, y2, rtol=1e-5, atol=1e-5)


def test_forward_is_deterministic():
    w = ss2d_inputs.custom(2, 20, 16, 16, 16)
    d = _dev(ss2d_inputs.make_inputs(w, seed=13))
    y1 = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    y2 = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    assert torch.equal(y1, y2)


SS2D_BWD_NAMES = [("dx", "dx"), ("ddelta", "ddelta"), ("dA", "dA"), ("dB", "dB"), ("dC", "dC"), ("dD", "dD"),
                  ("ddelta_bias", "ddelta_bias")]


@pytest.mark.parametrize("case", [(1, 8, 8, 8, 4), (2, 6, 5, 9, 16), (1, 40, 9, 10, 16), (1, 3, 1, 1, 2),
                                  (1, 4, 10, 20, 8)])
@pytest.mark.parametrize("with_states", [False, True])
def test_ss2d_backward_parity(case, with_states):
    Bn, Dn, H, W, N = case
    w = ss2d_inputs.custom(Bn, Dn, H, W, N)
    inp = ss2d_inputs.make_inputs(w, seed=14, with_dy=True)
    d = _dev(inp)
    cs = None
    if with_states:
        _, cs = ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True,
                                return_chunk_states=True)
    g = ss.ss2d_backward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, d["dy"],
                         chunk_states=cs)
    ref = oracle.ss2d_backward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                               True, inp["dy"])
    for name, rname in SS2D_BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], GRAD_TOL, f"{case} {name}")


def test_ss2d_backward_bf16():
    w = ss2d_inputs.custom(1, 8, 12, 12, 16, dtype="bf16", a_init="s4d_real")
    inp = ss2d_inputs.make_inputs(w, seed=15, with_dy=True)
    d = _dev(inp)
    g = ss.ss2d_backward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True, d["dy"])
    ref = oracle.ss2d_backward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                               True, inp["dy"])
    for name, rname in SS2D_BWD_NAMES:
        assert_rel_l2(g[name], ref[rname], BF16_TOL, name)


def test_autograd_function_matches_backward():
    w = ss2d_inputs.custom(1, 4, 6, 7, 8)
    inp = ss2d_inputs.make_inputs(w, seed=16, with_dy=True)
    d = _dev(inp)
    leaves = {k: d[k].clone().requires_grad_(True) for k in ("x", "delta", "A", "B", "C", "D", "delta_bias")}
    y = ss.ss2d(leaves["x"], leaves["delta"], leaves["A"], leaves["B"], leaves["C"], leaves["D"],
                leaves["delta_bias"], True)
    y.backward(d["dy"])
    ref = oracle.ss2d_backward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                               True, inp["dy"])
    for k, rname in (("x", "dx"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("D", "dD"),
                     ("delta_bias", "ddelta_bias")):
        assert_rel_l2(leaves[k].grad, ref[rname], GRAD_TOL, k)


def test_launch_counter_counts_fused_forward():
    w = ss2d_inputs.custom(1, 8, 8, 8, 4)
    d = _dev(ss2d_inputs.make_inputs(w, seed=17))
    before = ss.launch_count()
    ss.ss2d_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["delta_bias"], True)
    torch.cuda.synchronize()
    assert ss.launch_count() - before >= 2


# ---------------------------------------------------- full-size workloads

def _full_forward_check(index, items):
    w = ss2d_inputs.workload(index)
    inp = ss2d_inputs.make_inputs(w, seed=index, device="cuda", with_dy=False)
    y = ss.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"], True)
    torch.cuda.synchronize()
    sl = ss2d_inputs.batch_slice(inp, items)
    ref = oracle.ss2d_forward(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], sl["D"], sl["delta_bias"], True)
    got = y[items]
    if w.dtype == "f32":
        assert_fwd_close(got, ref, w.name)
    else:
        assert_rel_l2(got, ref, BF16_TOL, w.name)


def test_full_size_vmamba_t_stage1_fp32():
    _full_forward_check(1, [0, 64, 127])


def test_full_size_vmamba_stage3_bf16():
    _full_forward_check(2, [0, 64, 127])


def test_full_size_highres_bf16():
    _full_forward_check(3, [0, 4, 7])


def test_full_size_fwd_bwd_fp32():
    w = ss2d_inputs.workload(4)
    inp = ss2d_inputs.make_inputs(w, seed=4, device="cuda", with_dy=True)
    y, cs = ss.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"], True,
                            return_chunk_states=True)
    g = ss.ss2d_backward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"], True,
                         inp["dy"], chunk_states=cs)
    torch.cuda.synchronize()
    items = [0, 16, 31]
    sl = ss2d_inputs.batch_slice(inp, items)
    ref_y = oracle.ss2d_forward(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], sl["D"], sl["delta_bias"], True)
    assert_fwd_close(y[items], ref_y, "c4 fwd")
    ref = oracle.ss2d_backward(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], sl["D"], sl["delta_bias"], True,
                               sl["dy"])
    # per-item gradients compare directly; dA, dD, ddelta_bias sum over the whole batch, so they are
    # checked on the full batch through the identity with per-item sums below
    for name in ("dx", "ddelta", "dB", "dC"):
        assert_rel_l2(g[name][items], ref[name], GRAD_TOL, f"c4 {name}")
    # batch-summed parameter gradients: oracle over the whole batch would cost minutes; instead
    # check them on the three items with a separate GPU call restricted to those items
    g3 = ss.ss2d_backward(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], sl["D"], sl["delta_bias"], True, sl["dy"])
    for name in ("dA", "dD", "ddelta_bias"):
        assert_rel_l2(g3[name], ref[name], GRAD_TOL, f"c4 items {name}")


@pytest.mark.parametrize("d_conv", [0, 4])
def test_ss2d_proj_autograd(d_conv):
    # the differentiable producer path against the oracle's gradients, with and without the conv
    w, inp = _conv_case(1, 24, 6, 8, 16, 4, seed=70)
    names = ("x", "x_proj_weight", "dt_proj_weight", "dt_proj_bias", "A", "D", "conv_weight", "conv_bias")
    lv = {k: inp[k].cuda().requires_grad_(True) for k in names}
    cw, cb = (lv["conv_weight"], lv["conv_bias"]) if d_conv else (None, None)
    y = ss.ss2d_proj(lv["x"], lv["x_proj_weight"], lv["dt_proj_weight"], lv["dt_proj_bias"], lv["A"], lv["D"], cw, cb)
    dy = torch.randn(y.shape, generator=torch.Generator(device="cuda").manual_seed(71), device="cuda")
    y.backward(dy)
    dy_np = dy.double().cpu().numpy()
    if d_conv:
        ref = oracle.ss2d_backward_proj_conv(*_conv_call_args(inp), True, dy_np)
        pairs = dict(x="dx", conv_weight="dconv_weight", conv_bias="dconv_bias", x_proj_weight="dx_proj_weight",
                     dt_proj_weight="ddt_proj_weight", dt_proj_bias="ddt_proj_bias", A="dA", D="dD")
    else:
        ref = oracle.ss2d_backward_proj(inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"],
                                        inp["A"], inp["D"], True, dy_np)
        pairs = dict(x="dx", x_proj_weight="dx_proj_weight", dt_proj_weight="ddt_proj_weight",
                     dt_proj_bias="ddt_proj_bias", A="dA", D="dD")
    for leaf, rname in pairs.items():
        assert_rel_l2(lv[leaf].grad, ref[rname], GRAD_TOL, f"{leaf} (d_conv {d_conv})")
