"""Pins for the fp64 oracle: each test checks it against something other than itself.

Sources: "VMamba: Visual State Space Model" (section "2D Selective Scan (SS2D)
for visual data", Fig. 2) for the paths and the merge; "vision mamba-yolov8"
(section "2. Vmamba module code", selective_scan_ref) for the S6 recurrence.

Pins used: hand-tabulated traversal orders and hand-worked S6 values
(tests/golden/), the closed-form geometric series, the dense L x L form of the
recurrence evaluated by brute force, special cases that reduce to library
routines (cumulative sum, elementwise product), linearity, permutation and
adjoint identities of the index maps, central finite differences and exact
dot-product identities for the backward.  The bidirectional scan
(bimamba_inner_ref) is pinned by its mirror symmetry and by the SS2D oracle on a
one-row image, whose row-major paths are the sequence and its reverse.  Path
sets given as tables (the diagonal scans of the mooersco page, section 3) are
pinned by hand-tabulated diagonal orders (tests/golden/diagonal_paths.txt), the
horizontal-flip identity between the two diagonal families, equality with the
fixed cross-scan functions for the cross table, merge-of-scan = 4x, adjointness
and central differences.  The producer projections (MambaInnerFn.forward) are
pinned by per-token loops, by the B/C scale invariance of the output, and by
the special cases dt_proj = 0 and x_proj's C rows = 0.  The output gate (out times silu(z),
the last lines of selective_scan_ref) is pinned by its special values, by
scipy's logistic function and by central differences; the last state by
reading it back through a one-hot C.
"""
import json
import math
import os

import numpy as np
import pytest

import ss2d_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 1234


def _rng(seed=rng_seed):
    return np.random.default_rng(seed)


def _random_problem(rng, Bn, Ch, L, N, G, softplus=True, with_d=True, with_bias=True):
    u = rng.standard_normal((Bn, Ch, L))
    delta = 0.3 * rng.standard_normal((Bn, Ch, L))
    A = -rng.uniform(0.2, 3.0, size=(Ch, N))
    B = rng.standard_normal((Bn, G, N, L))
    C = rng.standard_normal((Bn, G, N, L))
    D = rng.standard_normal(Ch) if with_d else None
    bias = rng.uniform(-4.0, 0.0, size=Ch) if with_bias else None
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=D, delta_bias=bias, delta_softplus=softplus)


# ----------------------------------------------------------------- index maps

def _golden_paths():
    rows = []
    with open(os.path.join(GOLDEN, "crossscan_paths.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, seq = line.split(":")
            H, W, k = (int(t) for t in head.split())
            rows.append((H, W, k, [int(t) for t in seq.split()]))
    return rows


def test_paths_match_hand_tabulated_orders(oracle):
    rows = _golden_paths()
    assert len(rows) == 20
    for H, W, k, seq in rows:
        got = [oracle.path_pixel(k, l, H, W) for l in range(H * W)]
        assert got == seq, (H, W, k)


def test_cross_scan_matches_golden_gather(oracle):
    # the golden orders applied to a labelled image give CrossScan's output
    for H, W, k, seq in _golden_paths():
        x = np.arange(2 * 3 * H * W, dtype=np.float64).reshape(2, 3, H, W)
        xs = oracle.cross_scan(x)
        flat = x.reshape(2, 3, H * W)
        np.testing.assert_array_equal(xs[:, k], flat[:, :, seq])


@pytest.mark.parametrize("H,W", [(1, 1), (1, 9), (9, 1), (3, 5), (5, 3), (8, 8), (7, 2), (14, 14), (6, 11)])
def test_paths_are_bijections_and_reverses(oracle, H, W):
    L = H * W
    maps = [[oracle.path_pixel(k, l, H, W) for l in range(L)] for k in range(4)]
    for k in range(4):
        assert sorted(maps[k]) == list(range(L))
    assert maps[2] == maps[0][::-1]
    assert maps[3] == maps[1][::-1]
    assert maps[0] == list(range(L))


def test_column_path_is_row_path_of_transpose(oracle):
    rng = _rng()
    for H, W in [(4, 4), (3, 7), (6, 2)]:
        x = rng.standard_normal((2, 3, H, W))
        xs = oracle.cross_scan(x)
        xt = np.ascontiguousarray(np.swapaxes(x, 2, 3))  # (B, D, W, H)
        np.testing.assert_array_equal(xs[:, 1], xt.reshape(2, 3, H * W))
        np.testing.assert_array_equal(xs[:, 3], xt.reshape(2, 3, H * W)[:, :, ::-1])


def test_merge_of_scan_is_four_x(oracle):
    rng = _rng()
    for H, W in [(1, 1), (3, 5), (8, 8), (13, 6)]:
        x = rng.standard_normal((2, 5, H, W))
        y = oracle.cross_merge(oracle.cross_scan(x), H, W)
        np.testing.assert_array_equal(y, 4.0 * x)


def test_merge_is_adjoint_of_scan(oracle):
    rng = _rng(7)
    for H, W in [(3, 5), (8, 8), (2, 9)]:
        x = rng.standard_normal((2, 4, H, W))
        ys = rng.standard_normal((2, 4, 4, H * W))
        lhs = float(np.sum(oracle.cross_merge(ys, H, W) * x))
        rhs = float(np.sum(ys * oracle.cross_scan(x)))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_merge_sums_each_path_at_its_own_pixel(oracle):
    # tag each path with a distinct power of two so that a swapped path shows
    H, W = 3, 5
    rows = {(k): seq for h, w, k, seq in _golden_paths() if (h, w) == (H, W)}
    ys = np.zeros((1, 4, 1, H * W))
    for k in range(4):
        ys[0, k, 0, :] = (2.0 ** (4 * k)) * (np.arange(H * W) + 1)
    y = oracle.cross_merge(ys, H, W).reshape(H * W)
    expect = np.zeros(H * W)
    for k in range(4):
        for l, p in enumerate(rows[k]):
            expect[p] += (2.0 ** (4 * k)) * (l + 1)
    np.testing.assert_array_equal(y, expect)


# -------------------------------------------------------- S6 forward pins

def test_hand_worked_examples(oracle):
    with open(os.path.join(GOLDEN, "s6_hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        arr = {k: (None if case[k] is None else np.array(case[k], dtype=np.float64))
               for k in ("u", "delta", "A", "B", "C", "D", "delta_bias")}
        y, last = oracle.selective_scan_fwd(arr["u"], arr["delta"], arr["A"], arr["B"], arr["C"],
                                            arr["D"], arr["delta_bias"], case["delta_softplus"],
                                            return_last_state=True)
        np.testing.assert_allclose(y, np.array(case["y"]), rtol=1e-15, atol=1e-15, err_msg=case["name"])
        np.testing.assert_allclose(last, np.array(case["last_state"]), rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("L", [64, 4096])
def test_closed_form_geometric_series(oracle, L):
    # constant dt and A, B = C = u = 1, D = 0:  h_l = dt (1 - a^(l+1)) / (1 - a),  y_l = sum_n h_l,n
    N, Ch = 4, 3
    dts = np.array([0.013, 0.05, 0.0021])
    A = -np.array([[0.5, 1.0, 2.0, 7.0], [1.0, 2.0, 3.0, 4.0], [0.1, 0.2, 16.0, 0.01]])
    u = np.ones((1, Ch, L))
    delta = np.broadcast_to(dts[None, :, None], (1, Ch, L)).copy()
    B = np.ones((1, 1, N, L))
    C = np.ones((1, 1, N, L))
    y = oracle.selective_scan_fwd(u, delta, A, B, C, None, None, False)
    l = np.arange(L)
    for c in range(Ch):
        a = np.exp(dts[c] * A[c])
        expect = sum(dts[c] * (1.0 - a[n] ** (l + 1)) / (1.0 - a[n]) for n in range(N))
        np.testing.assert_allclose(y[0, c], expect, rtol=1e-12, atol=0)


def _dense_reference(p):
    """y_i = sum_{j<=i} sum_n C[n,i] (prod_{k=j+1..i} a[k,n]) dt_j B[n,j] u_j + D u_i, by brute force."""
    u, delta, A, B, C = p["u"], p["delta"], p["A"], p["B"], p["C"]
    Bn, Ch, L = u.shape
    N = A.shape[1]
    G = B.shape[1]
    t = delta + (p["delta_bias"][None, :, None] if p["delta_bias"] is not None else 0.0)
    dt = np.logaddexp(0.0, t) if p["delta_softplus"] else t
    y = np.zeros_like(u)
    for b in range(Bn):
        for c in range(Ch):
            g = c // (Ch // G)
            a = np.exp(dt[b, c][:, None] * A[c][None, :])  # (L, N)
            for i in range(L):
                acc = 0.0
                for j in range(i + 1):
                    decay = np.prod(a[j + 1:i + 1], axis=0)  # empty product = 1
                    acc += np.sum(C[b, g, :, i] * decay * dt[b, c, j] * B[b, g, :, j] * u[b, c, j])
                if p["D"] is not None:
                    acc += p["D"][c] * u[b, c, i]
                y[b, c, i] = acc
    return y


@pytest.mark.parametrize("shape", [(1, 4, 9, 3, 1), (2, 8, 17, 4, 4), (1, 6, 33, 2, 2), (1, 2, 1, 5, 1)])
def test_dense_form_brute_force(oracle, shape):
    Bn, Ch, L, N, G = shape
    p = _random_problem(_rng(L), Bn, Ch, L, N, G)
    y = oracle.selective_scan_fwd(**p)
    np.testing.assert_allclose(y, _dense_reference(p), rtol=1e-11, atol=1e-12)


def test_dense_form_on_tiny_workload(oracle):
    # the tiny SS2D workload's own values (B=1, D=8, H=W=8, N=4), per path
    w = ss2d_inputs.workload(0)
    inp = ss2d_inputs.make_inputs(w, seed=0)
    xs = oracle.cross_scan(inp["x"])
    p = dict(u=xs.reshape(1, 32, 64), delta=inp["delta"].double().numpy(), A=inp["A"].double().numpy(),
             B=inp["B"].double().numpy(), C=inp["C"].double().numpy(), D=inp["D"].double().numpy(),
             delta_bias=inp["delta_bias"].double().numpy(), delta_softplus=True)
    y = oracle.selective_scan_fwd(**p)
    np.testing.assert_allclose(y, _dense_reference(p), rtol=1e-11, atol=1e-12)


def test_zero_A_is_prefix_sum(oracle):
    rng = _rng(3)
    Bn, Ch, L, N = 2, 4, 50, 3
    p = _random_problem(rng, Bn, Ch, L, N, 2, softplus=False, with_d=False, with_bias=False)
    p["A"] = np.zeros((Ch, N))
    y = oracle.selective_scan_fwd(**p)
    for b in range(Bn):
        for c in range(Ch):
            g = c // 2
            terms = p["delta"][b, c][None, :] * p["B"][b, g] * p["u"][b, c][None, :]  # (N, L)
            expect = np.sum(p["C"][b, g] * np.cumsum(terms, axis=1), axis=0)
            np.testing.assert_allclose(y[b, c], expect, rtol=1e-12, atol=1e-12)


def test_zero_C_gives_skip_only(oracle):
    p = _random_problem(_rng(4), 2, 4, 20, 3, 4)
    p["C"] = np.zeros_like(p["C"])
    y = oracle.selective_scan_fwd(**p)
    np.testing.assert_array_equal(y, p["D"][None, :, None] * p["u"])


def test_single_step(oracle):
    p = _random_problem(_rng(5), 3, 4, 1, 5, 2)
    y = oracle.selective_scan_fwd(**p)
    dt = np.logaddexp(0.0, p["delta"][:, :, 0] + p["delta_bias"][None, :])
    for c in range(4):
        g = c // 2
        expect = np.sum(p["C"][:, g, :, 0] * dt[:, c:c + 1] * p["B"][:, g, :, 0], axis=1) * p["u"][:, c, 0]
        expect += p["D"][c] * p["u"][:, c, 0]
        np.testing.assert_allclose(y[:, c, 0], expect, rtol=1e-13)


def test_softplus_switch(oracle):
    # softplus on with bias b equals softplus off with delta replaced by log(1 + e^(delta + b))
    p = _random_problem(_rng(6), 1, 4, 30, 4, 4)
    y_on = oracle.selective_scan_fwd(**p)
    q = dict(p)
    q["delta"] = np.log1p(np.exp(p["delta"] + p["delta_bias"][None, :, None]))
    q["delta_bias"] = None
    q["delta_softplus"] = False
    np.testing.assert_allclose(oracle.selective_scan_fwd(**q), y_on, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("which", ["u", "B", "C"])
def test_linearity(oracle, which):
    rng = _rng(8)
    p = _random_problem(rng, 2, 4, 40, 4, 2, with_d=(which == "u"))
    v1 = rng.standard_normal(p[which].shape)
    v2 = rng.standard_normal(p[which].shape)
    alpha, beta = 0.7, -1.3

    def f(v):
        q = dict(p)
        q[which] = v
        return oracle.selective_scan_fwd(**q)

    np.testing.assert_allclose(f(alpha * v1 + beta * v2), alpha * f(v1) + beta * f(v2),
                               rtol=1e-11, atol=1e-11)


def test_reverse_path_is_flipped_forward_scan(oracle):
    # path 2 is path 0 walked backwards: scanning flipped path-0 inputs with path-2 parameters
    # and flipping back gives the merged contribution of path 2 at each pixel
    rng = _rng(9)
    Bn, Dn, H, W, N = 1, 3, 4, 5, 3
    L = H * W
    x = rng.standard_normal((Bn, Dn, H, W))
    delta = 0.2 * rng.standard_normal((Bn, 4 * Dn, L))
    A = -rng.uniform(0.5, 2.0, (4 * Dn, N))
    B = rng.standard_normal((Bn, 4, N, L))
    C = rng.standard_normal((Bn, 4, N, L))
    xs = oracle.cross_scan(x)
    ys = oracle.selective_scan_fwd(xs.reshape(Bn, 4 * Dn, L), delta, A, B, C, None, None, True)
    ys = ys.reshape(Bn, 4, Dn, L)
    flat = x.reshape(Bn, Dn, L)
    sl = slice(2 * Dn, 3 * Dn)
    y_rev = oracle.selective_scan_fwd(flat[:, :, ::-1], delta[:, sl], A[sl], B[:, 2:3], C[:, 2:3],
                                      None, None, True)
    np.testing.assert_allclose(ys[:, 2], y_rev, rtol=1e-13, atol=1e-14)
    # and in image order, path 2's output at pixel p sits at step L-1-p
    np.testing.assert_allclose(ys[:, 2, :, ::-1], ys[:, 2][:, :, ::-1], rtol=0, atol=0)


def test_ss2d_forward_is_scan_fwd_merge(oracle):
    # the full forward equals its three steps run separately (and differs if a path is dropped)
    w = ss2d_inputs.workload(0)
    inp = {k: v.double().numpy() for k, v in ss2d_inputs.make_inputs(w, seed=0).items()}
    y = oracle.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                            inp["delta_bias"], True)
    xs = oracle.cross_scan(inp["x"]).reshape(1, 32, 64)
    ys = oracle.selective_scan_fwd(xs, inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                   inp["delta_bias"], True)
    y2 = oracle.cross_merge(ys.reshape(1, 4, 8, 64), 8, 8)
    np.testing.assert_allclose(y, y2, rtol=0, atol=1e-15)
    assert np.all(np.isfinite(y)) and np.abs(y).max() > 0.1


# -------------------------------------------------------------- backward pins

def _ss2d_problem(seed, Bn=1, Dn=2, H=3, W=4, N=3):
    rng = _rng(seed)
    L = H * W
    return dict(x=rng.standard_normal((Bn, Dn, H, W)), delta=0.3 * rng.standard_normal((Bn, 4 * Dn, L)),
                A=-rng.uniform(0.3, 2.5, (4 * Dn, N)), B=rng.standard_normal((Bn, 4, N, L)),
                C=rng.standard_normal((Bn, 4, N, L)), D=rng.standard_normal(4 * Dn),
                delta_bias=rng.uniform(-3.0, 0.5, 4 * Dn))


def _loss(oracle, p, dy, softplus=True):
    y = oracle.ss2d_forward(p["x"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"], softplus)
    return float(np.sum(y * dy))


@pytest.mark.parametrize("softplus", [True, False])
def test_backward_central_differences(oracle, softplus):
    p = _ss2d_problem(11)
    if not softplus:
        p["delta_bias"] = np.abs(p["delta_bias"]) * 0.05 + 0.01
        p["delta"] = np.abs(p["delta"]) * 0.1
    rng = _rng(12)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.ss2d_backward(p["x"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"],
                             softplus, dy)
    names = dict(x="dx", delta="ddelta", A="dA", B="dB", C="dC", D="dD", delta_bias="ddelta_bias")
    for name, gname in names.items():
        flat = p[name].reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 12), replace=False)
        for i in idx:
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = _loss(oracle, p, dy, softplus)
            flat[i] = theta - h
            lm = _loss(oracle, p, dy, softplus)
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


def test_backward_dot_product_identities(oracle):
    # the forward is linear in x, in B and in C separately: <dy, f(v)> == <grad, v> exactly up to rounding
    p = _ss2d_problem(21, Bn=2, Dn=3, H=4, W=3, N=4)
    p["D"] = None  # keeps f(B) and f(C) linear (the skip term does not involve them)
    rng = _rng(22)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.ss2d_backward(p["x"], p["delta"], p["A"], p["B"], p["C"], None, p["delta_bias"], True, dy)
    for name, gname in (("x", "dx"), ("B", "dB"), ("C", "dC")):
        v = rng.standard_normal(p[name].shape)
        q = dict(p)
        q[name] = v
        lhs = _loss(oracle, q, dy)
        rhs = float(np.sum(g[gname] * v))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), (name, lhs, rhs)


def test_backward_of_scan_alone_matches_central_differences(oracle):
    # the 1-D S6 backward with G=2 groups (dB, dC summed over the channels of a group)
    rng = _rng(31)
    p = _random_problem(rng, 2, 4, 7, 3, 2)
    dout = rng.standard_normal(p["u"].shape)
    g = oracle.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"],
                                  True, dout)

    def loss():
        return float(np.sum(oracle.selective_scan_fwd(**p) * dout))

    for name, gname in (("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                        ("D", "dD"), ("delta_bias", "ddelta_bias")):
        flat = p[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


# ------------------------------------------------------- gate and last state

def test_gate_special_values(oracle):
    # silu(0) = 0: a zero gate zeroes every output; silu(z) -> z as z grows (sigmoid(40) = 1 - 4e-18)
    rng = _rng(41)
    p = _random_problem(rng, 2, 3, 9, 4, 1)
    plain = oracle.selective_scan_fwd(**p)
    zero = oracle.selective_scan_fwd(**p, z=np.zeros_like(p["u"]))
    assert np.all(zero == 0.0)
    big = oracle.selective_scan_fwd(**p, z=np.full_like(p["u"], 40.0))
    np.testing.assert_allclose(big, 40.0 * plain, rtol=1e-15, atol=0)


def test_gate_matches_logistic_times_output(oracle):
    # gated = ungated (including the D*u term) times z * expit(z), elementwise at the same (b, c, l)
    from scipy.special import expit

    rng = _rng(42)
    p = _random_problem(rng, 2, 4, 11, 3, 2)
    z = 2.0 * rng.standard_normal(p["u"].shape)
    plain = oracle.selective_scan_fwd(**p)
    gated = oracle.selective_scan_fwd(**p, z=z)
    np.testing.assert_allclose(gated, plain * z * expit(z), rtol=1e-13, atol=1e-15)


def test_gated_backward_matches_central_differences(oracle):
    rng = _rng(43)
    p = _random_problem(rng, 2, 4, 7, 3, 2)
    z = 1.5 * rng.standard_normal(p["u"].shape)
    dout = rng.standard_normal(p["u"].shape)
    g = oracle.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"],
                                  True, dout, z=z)
    q = dict(p, z=z)

    def loss():
        return float(np.sum(oracle.selective_scan_fwd(**q) * dout))

    for name, gname in (("z", "dz"), ("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"),
                        ("C", "dC"), ("D", "dD"), ("delta_bias", "ddelta_bias")):
        flat = q[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


def test_gate_at_zero_halves_the_output_gradient(oracle):
    # silu'(0) = 1/2 and silu(0) = 0: dz = dout * o / 2 and nothing reaches the scan
    rng = _rng(44)
    p = _random_problem(rng, 1, 3, 6, 2, 1)
    dout = rng.standard_normal(p["u"].shape)
    g = oracle.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"],
                                  True, dout, z=np.zeros_like(p["u"]))
    o = oracle.selective_scan_fwd(**p)
    np.testing.assert_allclose(g["dz"], 0.5 * dout * o, rtol=1e-14, atol=1e-15)
    assert np.all(g["du"] == 0.0) and np.all(g["dA"] == 0.0) and np.all(g["dB"] == 0.0)


def test_last_state_read_back_through_one_hot_c(oracle):
    # with D absent and C[., n, L-1] = e_m, the last output is h_{L-1}[m]
    rng = _rng(45)
    Bn, Ch, L, N, G = 2, 4, 13, 5, 2
    p = _random_problem(rng, Bn, Ch, L, N, G, with_d=False)
    _, last = oracle.selective_scan_fwd(**p, return_last_state=True)
    assert last.shape == (Bn, Ch, N)
    for m in range(N):
        q = dict(p)
        q["C"] = p["C"].copy()
        q["C"][:, :, :, L - 1] = 0.0
        q["C"][:, :, m, L - 1] = 1.0
        y = oracle.selective_scan_fwd(**q)
        np.testing.assert_array_equal(y[:, :, L - 1], last[:, :, m])


def test_last_state_unaffected_by_gate(oracle):
    rng = _rng(46)
    p = _random_problem(rng, 1, 2, 8, 3, 1)
    _, a = oracle.selective_scan_fwd(**p, return_last_state=True)
    _, b = oracle.selective_scan_fwd(**p, return_last_state=True, z=rng.standard_normal(p["u"].shape))
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------- bidirectional scan

def _bimamba_problem(rng, Bn=2, Dn=3, L=9, N=4):
    return dict(x=rng.standard_normal((Bn, Dn, L)), delta=0.3 * rng.standard_normal((Bn, Dn, L)),
                A=-rng.uniform(0.2, 3.0, (Dn, N)), A_b=-rng.uniform(0.2, 3.0, (Dn, N)),
                B=rng.standard_normal((Bn, N, L)), C=rng.standard_normal((Bn, N, L)),
                D=rng.standard_normal(Dn), delta_bias=rng.uniform(-4.0, 0.0, Dn))


def test_bimamba_mirror_symmetry(oracle):
    # with A_b = A and mirror-symmetric inputs the two directions see the same sequence, so the
    # output is mirror-symmetric; with A_b != A it is not
    rng = _rng(51)
    p = _bimamba_problem(rng)
    for k in ("x", "delta", "B", "C"):
        p[k] = p[k] + np.flip(p[k], -1)
    z = rng.standard_normal(p["x"].shape)
    z = z + np.flip(z, -1)
    y = oracle.bimamba_forward(**dict(p, A_b=p["A"]), z=z)
    np.testing.assert_allclose(y, np.flip(y, -1), rtol=1e-13, atol=1e-13)
    y2 = oracle.bimamba_forward(**p, z=z)
    assert np.abs(y2 - np.flip(y2, -1)).max() > 1e-3


def test_bimamba_is_half_of_ss2d_on_one_row(oracle):
    # a 1 x L image: SS2D's paths 0 and 1 are the sequence itself, 2 and 3 its reverse.  Give the
    # reversed paths A_b and the reversed delta/B/C, and SS2D sums each direction twice.
    rng = _rng(52)
    Bn, Dn, L, N = 2, 3, 11, 4
    p = _bimamba_problem(rng, Bn, Dn, L, N)
    y = oracle.bimamba_forward(**p)
    fl = lambda t: np.flip(t, -1)
    delta4 = np.concatenate([p["delta"], p["delta"], fl(p["delta"]), fl(p["delta"])], axis=1)
    A4 = np.concatenate([p["A"], p["A"], p["A_b"], p["A_b"]], axis=0)
    B4 = np.stack([p["B"], p["B"], fl(p["B"]), fl(p["B"])], axis=1)
    C4 = np.stack([p["C"], p["C"], fl(p["C"]), fl(p["C"])], axis=1)
    y_img = oracle.ss2d_forward(p["x"].reshape(Bn, Dn, 1, L), delta4, A4, B4, C4, np.tile(p["D"], 4),
                                np.tile(p["delta_bias"], 4), True)
    np.testing.assert_allclose(y_img.reshape(Bn, Dn, L), 2.0 * y, rtol=1e-12, atol=1e-12)


def test_bimamba_backward_matches_central_differences(oracle):
    rng = _rng(53)
    p = _bimamba_problem(rng, 2, 3, 7, 3)
    p["z"] = 1.5 * rng.standard_normal(p["x"].shape)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.bimamba_backward(p["x"], p["delta"], p["A"], p["A_b"], p["B"], p["C"], p["D"], p["z"],
                                p["delta_bias"], True, dy)

    def loss():
        return float(np.sum(oracle.bimamba_forward(**p) * dy))

    names = dict(x="dx", delta="ddelta", A="dA", A_b="dA_b", B="dB", C="dC", D="dD", delta_bias="ddelta_bias",
                 z="dz")
    for name, gname in names.items():
        flat = p[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


def test_projection_backward_matches_central_differences(oracle):
    p = _proj_problem(74, Bn=1, Dn=3, H=3, W=4, N=3, R=2)
    rng = _rng(75)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.ss2d_backward_proj(p["x"], p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"], True, dy)

    def loss():
        return float(np.sum(oracle.ss2d_forward_proj(p["x"], p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"]) * dy))

    names = dict(x="dx", Wx="dx_proj_weight", Wdt="ddt_proj_weight", bias="ddt_proj_bias", A="dA", D="dD")
    for name, gname in names.items():
        flat = p[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


# ------------------------------------------------------------ path tables

def _golden_diagonals():
    rows = []
    with open(os.path.join(GOLDEN, "diagonal_paths.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, seq = line.split(":")
            H, W, direction = (int(t) for t in head.split())
            rows.append((H, W, direction, [int(t) for t in seq.split()]))
    return rows


def test_diagonal_orders_match_hand_tabulated(oracle):
    rows = _golden_diagonals()
    assert len(rows) == 8
    for H, W, direction, seq in rows:
        assert oracle.diagonal_order(H, W, direction).tolist() == seq, (H, W, direction)


@pytest.mark.parametrize("H,W", [(1, 1), (1, 6), (5, 1), (3, 7), (8, 8), (6, 4)])
def test_diagonal_paths_are_permutations_and_mirror_images(oracle, H, W):
    t = oracle.diagonal_paths(H, W)
    L = H * W
    for k in range(4):
        assert sorted(t[k].tolist()) == list(range(L))
    assert t[2].tolist() == t[0][::-1].tolist() and t[3].tolist() == t[1][::-1].tolist()
    # direction -1 is direction +1 on the horizontally flipped image: pixel (i, j) <-> (i, W-1-j)
    i, j = t[0] // W, t[0] % W
    assert t[1].tolist() == (i * W + (W - 1 - j)).tolist()
    if H == 1:  # one row: the diagonal order is the row order, the other family its reverse
        assert t[0].tolist() == list(range(L)) and t[1].tolist() == list(range(L))[::-1]


def test_cross_table_reproduces_the_fixed_paths(oracle):
    rng = _rng(61)
    Bn, Dn, H, W, N = 2, 3, 4, 5, 3
    x = rng.standard_normal((Bn, Dn, H, W))
    t = oracle.cross_paths(H, W)
    np.testing.assert_array_equal(oracle.cross_scan_table(x, t), oracle.cross_scan(x))
    ys = rng.standard_normal((Bn, 4, Dn, H * W))
    np.testing.assert_array_equal(oracle.cross_merge_table(ys, H, W, t), oracle.cross_merge(ys, H, W))
    p = _ss2d_problem(62, Bn, Dn, H, W, N)
    args = (p["x"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"], True)
    np.testing.assert_array_equal(oracle.ss2d_forward_table(*args, t), oracle.ss2d_forward(*args))
    dy = rng.standard_normal(x.shape)
    g1 = oracle.ss2d_backward_table(*args, dy, t)
    g2 = oracle.ss2d_backward(*args, dy)
    for name in g1:
        np.testing.assert_array_equal(g1[name], g2[name])


def test_diagonal_merge_of_scan_and_adjointness(oracle):
    rng = _rng(63)
    Bn, Dn, H, W = 2, 3, 5, 7
    t = oracle.diagonal_paths(H, W)
    x = rng.standard_normal((Bn, Dn, H, W))
    np.testing.assert_array_equal(oracle.cross_merge_table(oracle.cross_scan_table(x, t), H, W, t), 4.0 * x)
    ys = rng.standard_normal((Bn, 4, Dn, H * W))
    lhs = float(np.sum(oracle.cross_merge_table(ys, H, W, t) * x))
    rhs = float(np.sum(ys * oracle.cross_scan_table(x, t)))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))
    # the diagonal set is not the cross set: the scans differ
    assert np.abs(oracle.cross_scan_table(x, t) - oracle.cross_scan(x)).max() > 0.1


def test_diagonal_backward_matches_central_differences(oracle):
    p = _ss2d_problem(64, Bn=1, Dn=2, H=3, W=4, N=3)
    t = oracle.diagonal_paths(3, 4)
    rng = _rng(65)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.ss2d_backward_table(p["x"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"], True, dy, t)

    def loss():
        y = oracle.ss2d_forward_table(p["x"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["delta_bias"], True, t)
        return float(np.sum(y * dy))

    for name, gname in (("x", "dx"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC")):
        flat = p[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)


# ------------------------------------------------------ producer projections

def _proj_problem(seed, Bn=2, Dn=3, H=3, W=4, N=3, R=2):
    rng = _rng(seed)
    return dict(x=rng.standard_normal((Bn, Dn, H, W)), Wx=rng.standard_normal((4, R + 2 * N, Dn)) / np.sqrt(Dn),
                Wdt=rng.uniform(-1, 1, (4, Dn, R)) / np.sqrt(R), bias=rng.uniform(-4.0, -2.0, 4 * Dn),
                A=-rng.uniform(0.3, 2.5, (4 * Dn, N)), D=rng.standard_normal(4 * Dn))


def test_projections_match_per_token_loops(oracle):
    p = _proj_problem(71)
    x, Wx, Wdt = p["x"], p["Wx"], p["Wdt"]
    Bn, Dn, H, W = x.shape
    R, N = Wdt.shape[2], (Wx.shape[1] - Wdt.shape[2]) // 2
    delta, Bm, Cm, _ = oracle.path_projections(x, Wx, Wdt)
    for b in range(Bn):
        for k in range(4):
            for l in range(H * W):
                pix = oracle.path_pixel(k, l, H, W)
                u = [x[b, d, pix // W, pix % W] for d in range(Dn)]
                row = [sum(Wx[k, c, d] * u[d] for d in range(Dn)) for c in range(R + 2 * N)]
                for d in range(Dn):
                    want = sum(Wdt[k, d, r] * row[r] for r in range(R))
                    assert abs(delta[b, k * Dn + d, l] - want) <= 1e-12
                for n in range(N):
                    assert abs(Bm[b, k, n, l] - row[R + n]) <= 1e-12
                    assert abs(Cm[b, k, n, l] - row[R + N + n]) <= 1e-12


def test_projection_output_invariant_to_b_c_scaling(oracle):
    # h is linear in B and y = C.h: scaling x_proj's B rows by s and its C rows by 1/s leaves y unchanged
    p = _proj_problem(72)
    R, N = p["Wdt"].shape[2], (p["Wx"].shape[1] - p["Wdt"].shape[2]) // 2
    y = oracle.ss2d_forward_proj(p["x"], p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"])
    Wx2 = p["Wx"].copy()
    Wx2[:, R:R + N] *= 4.0
    Wx2[:, R + N:] /= 4.0
    y2 = oracle.ss2d_forward_proj(p["x"], Wx2, p["Wdt"], p["bias"], p["A"], p["D"])
    np.testing.assert_allclose(y2, y, rtol=1e-12, atol=1e-12)
    Wx3 = p["Wx"].copy()
    Wx3[:, R:R + N] *= 4.0  # B alone scaled: the state path scales, the skip term does not
    y3 = oracle.ss2d_forward_proj(p["x"], Wx3, p["Wdt"], p["bias"], p["A"], None)
    y0 = oracle.ss2d_forward_proj(p["x"], p["Wx"], p["Wdt"], p["bias"], p["A"], None)
    np.testing.assert_allclose(y3, 4.0 * y0, rtol=1e-12, atol=1e-12)


def test_projection_special_cases(oracle):
    p = _proj_problem(73)
    R, N = p["Wdt"].shape[2], (p["Wx"].shape[1] - p["Wdt"].shape[2]) // 2
    Bn, Dn, H, W = p["x"].shape
    # dt_proj = 0: delta = 0 and dt = softplus(bias)
    y = oracle.ss2d_forward_proj(p["x"], p["Wx"], np.zeros_like(p["Wdt"]), p["bias"], p["A"], p["D"])
    _, Bm, Cm, _ = oracle.path_projections(p["x"], p["Wx"], p["Wdt"])
    ref = oracle.ss2d_forward(p["x"], np.zeros((Bn, 4 * Dn, H * W)), p["A"], Bm, Cm, p["D"], p["bias"], True)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)
    # C rows = 0: only the skip term remains, 4 D u summed over the paths
    Wx = p["Wx"].copy()
    Wx[:, R + N:] = 0.0
    y = oracle.ss2d_forward_proj(p["x"], Wx, p["Wdt"], p["bias"], p["A"], p["D"])
    Dk = p["D"].reshape(4, Dn)
    np.testing.assert_allclose(y, Dk.sum(0)[None, :, None, None] * p["x"], rtol=1e-13, atol=1e-13)


# --------------------------------------------------------- input generator

def test_input_recipe_statistics():
    w = ss2d_inputs.workload(0)
    inp = ss2d_inputs.make_inputs(w, seed=0, with_dy=True)
    assert inp["x"].shape == (1, 8, 8, 8)
    assert inp["delta"].shape == (1, 32, 64)
    assert inp["B"].shape == (1, 4, 4, 64)
    assert inp["A"].shape == (32, 4)
    np.testing.assert_array_equal(inp["A"][0].numpy(), -np.arange(1, 5, dtype=np.float32))
    dt = np.logaddexp(0.0, inp["delta_bias"].double().numpy())
    assert dt.min() >= 1e-3 * (1 - 1e-5) and dt.max() <= 1e-1 * (1 + 1e-5)
    assert float(inp["D"].min()) == 1.0 and float(inp["D"].max()) == 1.0
    # bf16 workloads round u, delta, B, C only
    wb = ss2d_inputs.custom(1, 4, 3, 5, 4, dtype="bf16", a_init="s4d_real")
    ib = ss2d_inputs.make_inputs(wb, seed=1)
    import torch
    assert ib["x"].dtype == torch.bfloat16 and ib["A"].dtype == torch.float32
    # determinism
    again = ss2d_inputs.make_inputs(w, seed=0, with_dy=True)
    for k in inp:
        assert torch.equal(inp[k], again[k])


# ------------------------------------------- causal depthwise conv per path

def _conv_problem(seed, Bn=1, Dn=3, H=3, W=4, N=3, R=2, Wc=4):
    p = _proj_problem(seed, Bn=Bn, Dn=Dn, H=H, W=W, N=N, R=R)
    rng = _rng(seed + 1000)
    p["cw"] = rng.standard_normal((4, Dn, Wc)) / np.sqrt(Wc)
    p["cb"] = 0.3 * rng.standard_normal(4 * Dn)
    return p


def test_path_conv_matches_numpy_convolve(oracle):
    from scipy.special import expit
    p = _conv_problem(80, Bn=2, Dn=3, H=4, W=5)
    u, pre = oracle.path_conv(p["x"], p["cw"], p["cb"])
    xs = oracle.cross_scan(p["x"])
    L = xs.shape[-1]
    for b in range(2):
        for k in range(4):
            for d in range(3):
                # causal cross-correlation = convolution with the reversed taps, first L outputs
                ref = np.convolve(xs[b, k, d], p["cw"][k, d, ::-1])[:L] + p["cb"][k * 3 + d]
                np.testing.assert_allclose(pre[b, k, d], ref, rtol=1e-13, atol=1e-13)
                np.testing.assert_allclose(u[b, k, d], ref * expit(ref), rtol=1e-13, atol=1e-13)


def test_path_conv_is_causal_along_each_path(oracle):
    p = _conv_problem(81, Dn=2, H=3, W=5, Wc=3)
    u0, _ = oracle.path_conv(p["x"], p["cw"], p["cb"])
    H, W, L = 3, 5, 15
    for pix in (0, 7, 14):
        x = p["x"].copy()
        x[0, 1, pix // W, pix % W] += 1.0
        u1, _ = oracle.path_conv(x, p["cw"], p["cb"])
        for k in range(4):
            step = [oracle.path_pixel(k, l, H, W) for l in range(L)].index(pix)
            changed = np.nonzero(np.abs(u1[0, k, 1] - u0[0, k, 1]) > 0)[0]
            assert set(changed) <= set(range(step, min(L, step + 3))) and step in set(changed)
            assert np.array_equal(u1[0, k, 0], u0[0, k, 0])  # other channels untouched


def test_forward_proj_conv_with_last_tap_is_forward_proj_of_silu(oracle):
    # one-hot weight on the newest tap and no bias: u_k = silu(x) read along path k
    p = _conv_problem(82, Bn=2, Dn=3, H=3, W=4)
    w = np.zeros_like(p["cw"])
    w[:, :, -1] = 1.0
    y = oracle.ss2d_forward_proj_conv(p["x"], w, None, p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"], True)
    xs = p["x"] / (1.0 + np.exp(-p["x"]))
    ref = oracle.ss2d_forward_proj(xs, p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"], True)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_projection_conv_backward_matches_central_differences(oracle):
    p = _conv_problem(83, Bn=1, Dn=2, H=3, W=3, N=2, R=2, Wc=3)
    rng = _rng(84)
    dy = rng.standard_normal(p["x"].shape)
    g = oracle.ss2d_backward_proj_conv(p["x"], p["cw"], p["cb"], p["Wx"], p["Wdt"], p["bias"], p["A"], p["D"], True,
                                       dy)

    def loss():
        return float(np.sum(oracle.ss2d_forward_proj_conv(p["x"], p["cw"], p["cb"], p["Wx"], p["Wdt"], p["bias"],
                                                          p["A"], p["D"]) * dy))

    names = dict(x="dx", cw="dconv_weight", cb="dconv_bias", Wx="dx_proj_weight", Wdt="ddt_proj_weight",
                 bias="ddt_proj_bias", A="dA", D="dD")
    for name, gname in names.items():
        flat = p[name].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 8), replace=False):
            theta = flat[i]
            h = 1e-6 * max(1.0, abs(theta))
            flat[i] = theta + h
            lp = loss()
            flat[i] = theta - h
            lm = loss()
            flat[i] = theta
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)
