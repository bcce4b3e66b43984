"""Pins of the fp64 oracle against facts the method and the mathematics fix (CPU only).

Each test pins one part of the oracle to something other than the oracle itself: an unrolled
(matrix) form of the recurrence, a textbook IIR filter from scipy, a geometric-series closed
form, an exact sympy expansion, a hand-derived worked example, limits (Delta -> 0), symmetries
(axis transpose, direction flip) and invariants (constancy along the pooled axis, masked ==
dense when every token is kept).  A plausible slip in any step (a dropped term, a wrong sign,
an off-by-one in the scan, a transposed weight, a wrong divisor or axis) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.signal
import scipy.special

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_params(rng, nd, E, N, R, dt_range=(0.05, 0.6)):
    """Small random parameter set with step sizes in a range where every term matters."""
    A_log = rng.uniform(-1.0, 1.0, size=(nd, E, N)).astype(np.float32)
    D = rng.uniform(0.5, 1.5, size=(nd, E)).astype(np.float32)
    W_x = rng.uniform(-1.0, 1.0, size=(nd, R + 2 * N, E)).astype(np.float32)
    W_dt = rng.uniform(-0.5, 0.5, size=(nd, E, R)).astype(np.float32)
    d0 = rng.uniform(*dt_range, size=(nd, E))
    b_dt = np.log(np.expm1(d0)).astype(np.float32)
    return A_log, D, W_x, W_dt, b_dt


# ---------------------------------------------------------------------------------------------
# p1: the scan equals its unrolled (convolution / matrix) form, brute force on short sequences.
# ---------------------------------------------------------------------------------------------
def _unrolled_scan(xbar, delta, u, A_log, R, N, dir_flags):
    """y_t = sum_s C_t . (prod of Abar between s and t) Bbar_s x_s, each product taken as one
    exp of a summed exponent, i.e. a different computation from the step recurrence."""
    B, T, E = xbar.shape
    ys = np.zeros((B, T, E))
    dirs = [d for d in (1, 2) if dir_flags & d]
    for k, d in enumerate(dirs):
        A = -np.exp(A_log[k].astype(np.float64))  # [E, N]
        for b in range(B):
            dt = delta[k, b]  # [T, E]
            Bm = u[k, b, :, R:R + N]  # [T, N]
            Cm = u[k, b, :, R + N:]
            for t in range(T):
                for s in range(T):
                    if d == 1 and s > t:
                        continue
                    if d == 2 and s < t:
                        continue
                    if d == 1:
                        span = dt[s + 1:t + 1].sum(axis=0)  # Abar_{s+1} ... Abar_t
                    else:
                        span = dt[t:s].sum(axis=0)  # Abar_t ... Abar_{s-1}
                    decay = np.exp(span[:, None] * A)  # [E, N]
                    contrib = Cm[t][None, :] * decay * (dt[s][:, None] * Bm[s][None, :]) * xbar[b, s][:, None]
                    ys[b, t] += contrib.sum(axis=1)
    return ys


@pytest.mark.parametrize("dir_flags", [1, 2, 3])
@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_p1_scan_equals_unrolled_form(oracle_mod, dir_flags, T):
    rng = np.random.default_rng(100 + 10 * T + dir_flags)
    B, E, N, R = 2, 3, 4, 2
    nd = oracle_mod.nd_of(dir_flags)
    A_log = rng.uniform(-1, 1, size=(nd, E, N)).astype(np.float32)
    xbar = rng.standard_normal((B, T, E))
    delta = rng.uniform(0.01, 0.8, size=(nd, B, T, E))
    u = rng.standard_normal((nd, B, T, R + 2 * N))
    ys = oracle_mod.scan(xbar, delta, u, A_log, R, N, dir_flags)
    ref = _unrolled_scan(xbar, delta, u, A_log, R, N, dir_flags)
    np.testing.assert_allclose(ys, ref, rtol=1e-12, atol=1e-12)


def test_p1_scan_lti_matches_scipy_lfilter(oracle_mod):
    """Constant Delta and B make each state a first-order IIR filter: h = lfilter([b], [1, -a], x)."""
    rng = np.random.default_rng(7)
    B, T, E, N, R = 1, 40, 2, 3, 1
    A_log = rng.uniform(-1, 1, size=(1, E, N)).astype(np.float32)
    xbar = rng.standard_normal((B, T, E))
    dval = rng.uniform(0.05, 0.5, size=E)
    delta = np.broadcast_to(dval[None, None, None, :], (1, B, T, E)).copy()
    Bn = rng.standard_normal(N)
    Cn = rng.standard_normal((T, N))  # C may vary in t: it only reads the state
    u = np.zeros((1, B, T, R + 2 * N))
    u[0, 0, :, R:R + N] = Bn[None, :]
    u[0, 0, :, R + N:] = Cn
    for dir_flags in (1, 2):
        ys = oracle_mod.scan(xbar, delta, u, A_log, R, N, dir_flags)
        ref = np.zeros((T, E))
        for e in range(E):
            for n in range(N):
                a = math.exp(-dval[e] * math.exp(float(A_log[0, e, n])))
                seq = xbar[0, :, e] * dval[e] * Bn[n]
                if dir_flags == 2:
                    seq = seq[::-1]
                hs = scipy.signal.lfilter([1.0], [1.0, -a], seq)
                if dir_flags == 2:
                    hs = hs[::-1]
                ref[:, e] += Cn[:, n] * hs
        np.testing.assert_allclose(ys[0], ref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# p2: constant grid -> geometric-series closed form (pins pooling divisor, W_x column selection,
#     softplus, ZOH, both scan directions, repeat, skip and gate in one go).
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
def test_p2_constant_grid_closed_form(oracle_mod, pool_axis, dir_flags):
    rng = np.random.default_rng(200 + 3 * pool_axis + dir_flags)
    B, h, w, E, N, R = 2, 5, 7, 4, 3, 2
    nd = oracle_mod.nd_of(dir_flags)
    A_log, D, W_x, _, b_dt = _rand_params(rng, nd, E, N, R)
    W_dt = np.zeros((nd, E, R), np.float32)  # Delta = softplus(b_dt), independent of x
    c, alpha = 2, np.float32(1.75)
    x = np.zeros((B, h, w, E), np.float32)
    x[..., c] = alpha  # every token equals alpha * e_c, so the pooled token is alpha * e_c
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, dir_flags)

    T = h if pool_axis == 0 else w
    dirs = [d for d in (1, 2) if dir_flags & d]
    ys_c = np.zeros(T)
    for k, d in enumerate(dirs):
        dt = np.logaddexp(0.0, float(b_dt[k, c]))  # softplus via numpy
        Bn = W_x[k, R:R + N, c].astype(np.float64) * alpha  # one-hot token selects column c
        Cn = W_x[k, R + N:, c].astype(np.float64) * alpha
        a = np.exp(-dt * np.exp(A_log[k, c].astype(np.float64)))
        t = np.arange(T)
        steps = t + 1 if d == 1 else T - t  # number of inputs the state has absorbed
        hs = (dt * Bn * alpha)[None, :] * (1 - a[None, :] ** steps[:, None]) / (1 - a[None, :])
        ys_c += hs @ Cn
    Dsum = D.astype(np.float64).sum(axis=0)
    sig = scipy.special.expit(z.astype(np.float64))
    skip = Dsum[None, None, None, :] * x.astype(np.float64)
    pooled = np.zeros((B, h, w, E))
    if pool_axis == 0:
        pooled[..., c] = ys_c[None, :, None]
    else:
        pooled[..., c] = ys_c[None, None, :]
    ref = z * sig * (pooled + skip)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-13)


def test_p2_projection_is_a_matrix_product(oracle_mod):
    """u = W_x xbar (numpy matmul) and Delta selects dt_low through a one-hot W_dt."""
    rng = np.random.default_rng(21)
    B, T, E, N, R, nd = 2, 3, 6, 2, 4, 2
    xbar = rng.standard_normal((B, T, E))
    W_x = rng.standard_normal((nd, R + 2 * N, E)).astype(np.float32)
    W_dt = np.zeros((nd, E, R), np.float32)
    beta = rng.uniform(0.5, 2.0, size=(nd, E)).astype(np.float32)
    for e in range(E):
        W_dt[:, e, e % R] = beta[:, e]
    b_dt = rng.standard_normal((nd, E)).astype(np.float32)
    u, delta = oracle_mod.proj(xbar, W_x, W_dt, b_dt, R, N)
    ref_u = np.einsum("kje,bte->kbtj", W_x.astype(np.float64), xbar)
    np.testing.assert_allclose(u, ref_u, rtol=1e-12, atol=1e-12)
    pre = beta[:, None, None, :] * ref_u[..., np.arange(E) % R] + b_dt[:, None, None, :]
    np.testing.assert_allclose(delta, np.logaddexp(0.0, pre), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# p3: Delta -> 0 leaves only the skip: y = SiLU(z) (sum_k D_k) x.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
def test_p3_small_step_limit(oracle_mod, dir_flags):
    rng = np.random.default_rng(300 + dir_flags)
    B, h, w, E, N, R = 2, 4, 6, 5, 4, 2
    nd = oracle_mod.nd_of(dir_flags)
    A_log, D, W_x, _, _ = _rand_params(rng, nd, E, N, R)
    W_dt = np.zeros((nd, E, R), np.float32)
    b_dt = np.full((nd, E), -30.0, np.float32)  # Delta = softplus(-30) ~ 9e-14
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, 0, dir_flags)
    ref = scipy.special.expit(z.astype(np.float64)) * z * (D.astype(np.float64).sum(0) * x)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# p4: after the repeat, y is constant along the pooled axis when the skip is off and z constant.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p4_repeat_constant_along_pooled_axis(oracle_mod, pool_axis):
    rng = np.random.default_rng(400 + pool_axis)
    B, h, w, E, N, R, nd = 2, 5, 6, 4, 3, 2, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    D[:] = 0
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = np.full((B, h, w, E), 0.7, np.float32)
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)
    pooled_axis = 2 if pool_axis == 0 else 1
    first = np.take(y, [0], axis=pooled_axis)
    assert np.array_equal(y, np.broadcast_to(first, y.shape))
    # and it does vary along the scanned axis (the pooled tokens differ)
    scanned_axis = 1 if pool_axis == 0 else 2
    assert np.ptp(y, axis=scanned_axis).max() > 1e-3


# ---------------------------------------------------------------------------------------------
# p5: pooling then scanning equals scanning an explicitly averaged grid.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p5_pool_equals_explicit_mean(oracle_mod, pool_axis):
    rng = np.random.default_rng(500 + pool_axis)
    B, h, w, E, N, R, nd = 2, 6, 3, 5, 4, 2, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    D[:] = 0  # the skip reads full-resolution x; without it only the pooled token matters
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    ax = 2 if pool_axis == 0 else 1  # the pooled-over axis
    inter = oracle_mod.forward_intermediates(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)
    np.testing.assert_allclose(inter["xbar"], x.mean(axis=ax, dtype=np.float64), rtol=1e-13, atol=1e-15)
    # a grid whose pooled lines are replaced by their (fp32-rounded) numpy means
    xm = np.broadcast_to(x.mean(axis=ax, keepdims=True, dtype=np.float64), x.shape).astype(np.float32)
    y2 = oracle_mod.forward(xm, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)
    np.testing.assert_allclose(inter["y"], y2, rtol=1e-6, atol=1e-7 * np.abs(y2).max())
    y1 = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)
    np.testing.assert_array_equal(y1, inter["y"])


# ---------------------------------------------------------------------------------------------
# p6: symmetries -- axis transpose and direction flip.
# ---------------------------------------------------------------------------------------------
def test_p6_pool_axis_is_a_transpose(oracle_mod):
    rng = np.random.default_rng(600)
    B, h, w, E, N, R, nd = 2, 4, 7, 3, 4, 2, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    yh = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, 1, 3)
    xt = np.ascontiguousarray(x.transpose(0, 2, 1, 3))
    zt = np.ascontiguousarray(z.transpose(0, 2, 1, 3))
    yw = oracle_mod.forward(xt, zt, A_log, D, W_x, W_dt, b_dt, 0, 3)
    np.testing.assert_allclose(yh, yw.transpose(0, 2, 1, 3), rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p6_backward_is_flipped_forward(oracle_mod, pool_axis):
    rng = np.random.default_rng(610 + pool_axis)
    B, h, w, E, N, R = 2, 5, 4, 3, 4, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, 1, E, N, R)
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    ax = 1 if pool_axis == 0 else 2  # the scanned axis
    yb = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 2)
    xf = np.ascontiguousarray(np.flip(x, axis=ax))
    zf = np.ascontiguousarray(np.flip(z, axis=ax))
    yf = oracle_mod.forward(xf, zf, A_log, D, W_x, W_dt, b_dt, pool_axis, 1)
    np.testing.assert_allclose(yb, np.flip(yf, axis=ax), rtol=1e-14, atol=1e-15)
    # and the bidirectional layer is the sum of both one-directional layers minus one skip
    P2 = tuple(np.concatenate([a, a]) for a in (A_log, D, W_x, W_dt, b_dt))
    ybi = oracle_mod.forward(x, z, *P2, pool_axis, 3)
    yfw = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 1)
    skip = scipy.special.expit(z.astype(np.float64)) * z * (D[0].astype(np.float64) * x)
    np.testing.assert_allclose(ybi, yb + yfw, rtol=1e-12, atol=1e-13)
    assert np.abs(ybi - (yb + yfw - skip)).max() > 1e-3  # the skip is added once per direction


# ---------------------------------------------------------------------------------------------
# p7: tiny grids against an exact sympy expansion of the definitions.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("shape,pool_axis", [((2, 2), 0), ((2, 2), 1), ((1, 3), 0), ((1, 3), 1)])
def test_p7_tiny_grid_exact_sympy(oracle_mod, shape, pool_axis):
    import sympy as sp

    h, w = shape
    B, E, N, R, nd = 1, 2, 2, 1, 2
    rng = np.random.default_rng(700 + h * 10 + w + pool_axis)

    def q(size, lo=-8, hi=8, den=4):  # small dyadic rationals, exact in fp32
        return (rng.integers(lo, hi + 1, size=size) / den).astype(np.float32)

    x, z = q((B, h, w, E)), q((B, h, w, E))
    A_log, D, W_x, W_dt, b_dt = q((nd, E, N)), q((nd, E)), q((nd, R + 2 * N, E)), q((nd, E, R)), q((nd, E))
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)

    R_ = sp.Rational

    def r(v):
        return R_(str(float(v)))

    T = h if pool_axis == 0 else w
    S = w if pool_axis == 0 else h
    xb = [[sum(r(x[0, (t if pool_axis == 0 else s), (s if pool_axis == 0 else t), e]) for s in range(S)) / S
           for e in range(E)] for t in range(T)]
    ys = [[0 for _ in range(E)] for _ in range(T)]
    for k in range(nd):
        uu = [[sum(r(W_x[k, j, e]) * xb[t][e] for e in range(E)) for j in range(R + 2 * N)] for t in range(T)]
        dl = [[sp.log(1 + sp.exp(sum(r(W_dt[k, e, rr]) * uu[t][rr] for rr in range(R)) + r(b_dt[k, e])))
               for e in range(E)] for t in range(T)]
        for e in range(E):
            for n in range(N):
                A = -sp.exp(r(A_log[k, e, n]))
                for t in range(T):
                    srcs = range(0, t + 1) if k == 0 else range(t, T)
                    for s in srcs:
                        mid = range(s + 1, t + 1) if k == 0 else range(t, s)
                        decay = sp.exp(A * sum(dl[m][e] for m in mid)) if len(mid) else 1
                        ys[t][e] += uu[t][R + N + n] * decay * dl[s][e] * uu[s][R + n] * xb[s][e]
    for i in range(h):
        for j in range(w):
            t = i if pool_axis == 0 else j
            for e in range(E):
                zz = r(z[0, i, j, e])
                val = zz / (1 + sp.exp(-zz)) * (ys[t][e] + (r(D[0, e]) + r(D[1, e])) * r(x[0, i, j, e]))
                assert abs(float(sp.N(val, 30)) - y[0, i, j, e]) <= 1e-13 * max(1.0, abs(y[0, i, j, e]))


# ---------------------------------------------------------------------------------------------
# Hand-derived worked example (tests/golden/tiny_2x2_hand.json).
# ---------------------------------------------------------------------------------------------
def test_golden_hand_worked_example(oracle_mod):
    with open(os.path.join(GOLDEN, "tiny_2x2_hand.json")) as f:
        g = json.load(f)
    inp = {k: np.array(v, np.float32) for k, v in g["inputs"].items()}
    inter = oracle_mod.forward_intermediates(inp["x"], inp["z"], inp["A_log"], inp["D"], inp["W_x"],
                                             inp["W_dt"], inp["b_dt"], g["pool_axis"], g["dir_flags"])
    ln2 = math.log(2.0)
    np.testing.assert_allclose(inter["xbar"].ravel(), g["expected"]["xbar"], rtol=0, atol=0)
    np.testing.assert_allclose(inter["delta"].ravel(), ln2, rtol=1e-15)
    ys = np.array(g["expected"]["ys_over_ln2"]) * ln2
    np.testing.assert_allclose(inter["ys"].ravel(), ys, rtol=1e-14)
    x = inp["x"].astype(np.float64)
    z = inp["z"].astype(np.float64)
    t_of = np.array([[0, 0], [1, 1]]) if g["pool_axis"] == 0 else np.array([[0, 1], [0, 1]])
    y = z / (1 + np.exp(-z)) * (ys[t_of][None, ..., None] + g["expected"]["Dsum"] * x)
    np.testing.assert_allclose(inter["y"], y, rtol=1e-14)


# ---------------------------------------------------------------------------------------------
# Exact-ZOH input term and pooling scale (variants of the discretisation and pooling steps).
# ---------------------------------------------------------------------------------------------
def test_zoh_exact_closed_form_and_limit(oracle_mod):
    rng = np.random.default_rng(800)
    B, T, E, N, R = 1, 6, 2, 3, 1
    A_log = rng.uniform(-1, 1, size=(1, E, N)).astype(np.float32)
    xbar = np.ones((B, T, E))
    dval = np.array([0.3, 0.05])
    delta = np.broadcast_to(dval[None, None, None, :], (1, B, T, E)).copy()
    u = np.zeros((1, B, T, R + 2 * N))
    u[..., R:R + N] = 1.0
    u[..., R + N:] = 1.0
    ys = oracle_mod.scan(xbar, delta, u, A_log, R, N, 1, zoh_exact=True)
    A = -np.exp(A_log[0].astype(np.float64))  # [E, N]
    a = np.exp(dval[:, None] * A)
    bbar = (a - 1) / A  # exact ZOH of the input matrix with B = 1
    t = np.arange(T)
    ref = (bbar[None] * (1 - a[None] ** (t[:, None, None] + 1)) / (1 - a[None])).sum(-1)
    np.testing.assert_allclose(ys[0], ref, rtol=1e-12)
    # for small steps exact ZOH and the Euler input term agree to first order
    small = delta * 1e-6
    ye = oracle_mod.scan(xbar, small, u, A_log, R, N, 1, zoh_exact=True)
    yd = oracle_mod.scan(xbar, small, u, A_log, R, N, 1, zoh_exact=False)
    np.testing.assert_allclose(ye, yd, rtol=1e-5)


def test_pool_scale_scales_only_the_pooled_branch(oracle_mod):
    rng = np.random.default_rng(810)
    B, h, w, E, N, R, nd = 2, 4, 4, 4, 2, 2, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    i1 = oracle_mod.forward_intermediates(x, z, A_log, D, W_x, W_dt, b_dt, 0, 3, pool_scale=0.25)
    i2 = oracle_mod.forward_intermediates(x, z, A_log, D, W_x, W_dt, b_dt, 0, 3)
    np.testing.assert_allclose(i1["xbar"], 0.25 * i2["xbar"], rtol=1e-15)


# ---------------------------------------------------------------------------------------------
# p8: the masked layer.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p8_all_kept_in_grid_order_equals_dense(oracle_mod, pool_axis):
    rng = np.random.default_rng(900 + pool_axis)
    B, h, w, E, N, R, nd = 2, 4, 5, 3, 4, 2, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    yd = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3)
    idx = np.tile(np.arange(h * w, dtype=np.int32), (B, 1))
    ym = oracle_mod.forward(x.reshape(B, h * w, E), z.reshape(B, h * w, E), A_log, D, W_x, W_dt, b_dt,
                            pool_axis, 3, keep_idx=idx, h=h, w=w)
    np.testing.assert_allclose(ym, yd.reshape(B, h * w, E), rtol=1e-14, atol=1e-15)


def test_p8_permuted_indices_permute_outputs(oracle_mod):
    rng = np.random.default_rng(910)
    B, h, w, E, N, R, nd, K = 2, 6, 6, 3, 4, 2, 2, 9
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    idx = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
    x = rng.standard_normal((B, K, E)).astype(np.float32)
    z = rng.standard_normal((B, K, E)).astype(np.float32)
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, 0, 3, keep_idx=idx, h=h, w=w)
    p = rng.permutation(K)
    yp = oracle_mod.forward(x[:, p], z[:, p], A_log, D, W_x, W_dt, b_dt, 0, 3, keep_idx=idx[:, p], h=h, w=w)
    np.testing.assert_allclose(yp, y[:, p], rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p8_rows_match_numpy_bucketing(oracle_mod, pool_axis):
    rng = np.random.default_rng(920 + pool_axis)
    B, h, w, K = 3, 8, 5, 17
    idx = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
    st, row_of, row_off, row_tok = oracle_mod.mask_rows(idx, h, w, pool_axis)
    assert st == 0
    T = h if pool_axis == 0 else w
    ref_row = idx // w if pool_axis == 0 else idx % w
    assert np.array_equal(row_of, ref_row)
    for b in range(B):
        counts = np.bincount(ref_row[b], minlength=T)
        assert np.array_equal(row_off[b], np.concatenate([[0], np.cumsum(counts)]))
        assert np.array_equal(row_tok[b], np.argsort(ref_row[b], kind="stable"))


def test_p8_masked_pool_divides_by_fixed_width(oracle_mod):
    rng = np.random.default_rng(930)
    B, h, w, E, K = 2, 4, 6, 3, 7
    idx = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
    x = rng.standard_normal((B, K, E)).astype(np.float32)
    st, row_of, row_off, row_tok = oracle_mod.mask_rows(idx, h, w, 0)
    xbar = oracle_mod.pool_masked(x, row_off, row_tok, w)
    ref = np.zeros((B, h, E))
    for b in range(B):
        np.add.at(ref[b], idx[b] // w, x[b].astype(np.float64))
    np.testing.assert_allclose(xbar, ref / w, rtol=1e-14, atol=1e-15)
    assert (ref == 0).all(axis=2).any()  # some rows are empty and pool to zero


@pytest.mark.parametrize("bad", ["dup", "neg", "big"])
def test_p8_bad_indices_are_reported(oracle_mod, bad):
    h, w, K = 4, 4, 5
    idx = np.array([[0, 5, 9, 3, 12], [1, 2, 3, 4, 6]], np.int32)
    if bad == "dup":
        idx[1, 4] = 2
    elif bad == "neg":
        idx[0, 2] = -1
    else:
        idx[0, 0] = h * w
    st, row_of, _, _ = oracle_mod.mask_rows(idx, h, w, 0)
    assert st == oracle_mod.FVO_BAD_INDEX
    assert (row_of < 0).sum() == 1


# ---------------------------------------------------------------------------------------------
# p9: the post-SSM LayerNorm (after the repeat and the skip, before the gate).
# ---------------------------------------------------------------------------------------------
def _silu(z):
    return z * scipy.special.expit(z)


def _ln_case(rng, masked, pool_axis):
    B, h, w, E, N, R, nd = 2, 3, 5, 7, 4, 3, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    shp = (B, 6, E) if masked else (B, h, w, E)
    x = rng.standard_normal(shp).astype(np.float32)
    # |SiLU(z)| >= 0.27 everywhere, so the pre-gate value can be recovered by division
    z = (np.sign(rng.standard_normal(shp)) * (1.0 + np.abs(rng.standard_normal(shp)))).astype(np.float32)
    idx = np.stack([rng.permutation(h * w)[:6] for _ in range(B)]).astype(np.int32) if masked else None
    gamma = rng.uniform(0.5, 1.5, E).astype(np.float32)
    beta = (0.3 * rng.standard_normal(E)).astype(np.float32)
    return dict(x=x, z=z, A_log=A_log, D=D, W_x=W_x, W_dt=W_dt, b_dt=b_dt, pool_axis=pool_axis, dir_flags=3,
                keep_idx=idx, h=h, w=w), gamma, beta


@pytest.mark.parametrize("masked,pool_axis", [(False, 0), (False, 1), (True, 0), (True, 1)])
def test_p9_layernorm_is_torch_layer_norm_of_the_pre_gate_value(oracle_mod, masked, pool_axis):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(950 + 2 * pool_axis + masked)
    a, gamma, beta = _ln_case(rng, masked, pool_axis)
    eps = 0.05  # large enough that its placement under the root matters
    y0 = oracle_mod.forward(**a)
    y1 = oracle_mod.forward(**a, ln_gamma=gamma, ln_beta=beta, ln_eps=eps)
    s = _silu(a["z"].astype(np.float64))
    pre = y0 / s  # the pre-gate value ys[t] + (sum D) x, pinned by p2-p8
    ln = torch.nn.functional.layer_norm(torch.from_numpy(pre), (pre.shape[-1],),
                                        torch.from_numpy(gamma.astype(np.float64)),
                                        torch.from_numpy(beta.astype(np.float64)), eps).numpy()
    np.testing.assert_allclose(y1, s * ln, rtol=1e-11, atol=1e-13)


def test_p9_layernorm_standardises_each_token(oracle_mod):
    rng = np.random.default_rng(960)
    a, gamma, beta = _ln_case(rng, False, 0)
    E = gamma.shape[0]
    y = oracle_mod.forward(**a, ln_gamma=np.ones(E, np.float32), ln_beta=np.zeros(E, np.float32), ln_eps=0.0)
    v = y / _silu(a["z"].astype(np.float64))
    np.testing.assert_allclose(v.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((v * v).mean(axis=-1), 1.0, rtol=1e-12)
    # gamma scales and beta shifts the normalised value channel by channel
    y2 = oracle_mod.forward(**a, ln_gamma=gamma, ln_beta=beta, ln_eps=0.0)
    v2 = y2 / _silu(a["z"].astype(np.float64))
    np.testing.assert_allclose(v2, gamma.astype(np.float64) * v + beta.astype(np.float64), rtol=1e-12, atol=1e-13)


def test_p9_layernorm_arguments(oracle_mod):
    rng = np.random.default_rng(970)
    a, gamma, beta = _ln_case(rng, False, 1)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(**a, ln_gamma=gamma, ln_beta=None)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(**a, ln_gamma=gamma, ln_beta=beta, ln_eps=-1.0)


# ---------------------------------------------------------------------------------------------
# p10: the block's Conv1D in front of the layer (per-direction depthwise filters along the
# block's sequence, which runs line by line along the pooled-over axis).
# ---------------------------------------------------------------------------------------------
def _seq(x, pool_axis):
    """Grid [B,h,w,E] -> the block's sequence [B,L,E]: lines t in order, tokens s along each line."""
    return (x if pool_axis == 0 else x.transpose(0, 2, 1, 3)).reshape(x.shape[0], -1, x.shape[-1])


def _unseq(s, h, w, pool_axis):
    B, L, E = s.shape
    return s.reshape(B, h, w, E) if pool_axis == 0 else s.reshape(B, w, h, E).transpose(0, 2, 1, 3)


def _torch_conv(x, conv_w, conv_b, pool_axis, dir_flags, silu):
    """Reference Conv1D through torch.nn.functional.conv1d (fp64, groups = E, zero padding, the
    first L outputs: causal); the backward slot runs the same filter on the reversed sequence."""
    torch = pytest.importorskip("torch")
    B, h, w, E = x.shape
    dc = conv_w.shape[2]
    seq = torch.from_numpy(_seq(x.astype(np.float64), pool_axis)).permute(0, 2, 1)  # [B,E,L]
    outs = []
    dirs = [d for d in (1, 2) if dir_flags & d]
    for k, d in enumerate(dirs):
        wt = torch.from_numpy(conv_w[k].astype(np.float64))[:, None, :]
        bt = torch.from_numpy(conv_b[k].astype(np.float64))
        inp = seq if d == 1 else seq.flip(-1)
        o = torch.nn.functional.conv1d(inp, wt, bt, padding=dc - 1, groups=E)[..., :h * w]
        if d == 2:
            o = o.flip(-1)
        if silu:
            o = torch.nn.functional.silu(o)
        outs.append(_unseq(o.permute(0, 2, 1).numpy(), h, w, pool_axis))
    return np.stack(outs)


def _conv_case(rng, B=2, h=3, w=5, E=6, dc=4, nd=2):
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    cw = rng.uniform(-1, 1, size=(nd, E, dc)).astype(np.float32)
    cb = rng.uniform(-0.5, 0.5, size=(nd, E)).astype(np.float32)
    return x, cw, cb


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dc,silu", [(1, False), (2, False), (4, False), (4, True), (3, True)])
def test_p10_conv_matches_torch_conv1d(oracle_mod, pool_axis, dc, silu):
    rng = np.random.default_rng(1000 + 10 * dc + 2 * pool_axis + silu)
    x, cw, cb = _conv_case(rng, dc=dc)
    got = oracle_mod.conv(x, cw, cb, pool_axis, 3, silu)
    ref = _torch_conv(x, cw, cb, pool_axis, 3, silu)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    # one direction alone takes its own filter slot 0
    got_b = oracle_mod.conv(x, cw[1:], cb[1:], pool_axis, 2, silu)
    np.testing.assert_allclose(got_b[0], ref[1], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p10_conv_identity_and_one_step_shift(oracle_mod, pool_axis):
    rng = np.random.default_rng(1100 + pool_axis)
    B, h, w, E, dc = 2, 4, 3, 5, 4
    x, _, _ = _conv_case(rng, B, h, w, E, dc)
    zero_b = np.zeros((2, E), np.float32)
    ident = np.zeros((2, E, dc), np.float32)
    ident[..., dc - 1] = 1.0
    np.testing.assert_array_equal(oracle_mod.conv(x, ident, zero_b, pool_axis, 3), np.stack([x, x]).astype(np.float64))
    shift = np.zeros((2, E, dc), np.float32)
    shift[..., dc - 2] = 1.0
    xc = oracle_mod.conv(x, shift, zero_b, pool_axis, 3)
    s = _seq(x.astype(np.float64), pool_axis)
    prev = np.concatenate([np.zeros_like(s[:, :1]), s[:, :-1]], axis=1)  # forward: the token one step back
    nxt = np.concatenate([s[:, 1:], np.zeros_like(s[:, :1])], axis=1)    # backward: one step ahead
    np.testing.assert_array_equal(xc[0], _unseq(prev, h, w, pool_axis))
    np.testing.assert_array_equal(xc[1], _unseq(nxt, h, w, pool_axis))
    # bias only: a constant (SiLU of it) everywhere
    xb = oracle_mod.conv(np.zeros_like(x), shift, np.full((2, E), 0.75, np.float32), pool_axis, 3, True)
    np.testing.assert_allclose(xb, 0.75 / (1 + math.exp(-0.75)), rtol=1e-15)


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
def test_p10_identity_conv_layer_is_the_plain_layer(oracle_mod, pool_axis, dir_flags):
    rng = np.random.default_rng(1200 + 3 * pool_axis + dir_flags)
    B, h, w, E, N, R = 2, 3, 4, 5, 3, 2
    nd = oracle_mod.nd_of(dir_flags)
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, nd, E, N, R)
    x = rng.standard_normal((B, h, w, E)).astype(np.float32)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    ident = np.zeros((nd, E, 4), np.float32)
    ident[..., 3] = 1.0
    plain = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, dir_flags)
    conv = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, dir_flags, conv_w=ident,
                              conv_b=np.zeros((nd, E), np.float32))
    np.testing.assert_allclose(conv, plain, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("d", [1, 2])
def test_p10_one_direction_pools_scans_and_skips_its_own_convolved_input(oracle_mod, pool_axis, d):
    """With one direction the layer is the plain layer of that direction's convolved tokens: their
    explicit numpy mean pooled, the pinned projection and scan, and the skip D * xc."""
    rng = np.random.default_rng(1300 + 2 * pool_axis + d)
    B, h, w, E, N, R = 2, 4, 3, 5, 3, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, 1, E, N, R)
    x, cw, cb = _conv_case(rng, B, h, w, E, 3, 1)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    y = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, d, conv_w=cw, conv_b=cb, conv_silu=True)
    xc = _torch_conv(x, cw, cb, pool_axis, d, True)[0]
    xbar = xc.mean(axis=2 if pool_axis == 0 else 1)
    u, delta = oracle_mod.proj(xbar, W_x, W_dt, b_dt, R, N)
    ys = oracle_mod.scan(xbar, delta, u, A_log, R, N, d)
    rep = ys[:, :, None, :] if pool_axis == 0 else ys[:, None, :, :]
    ref = _silu(z.astype(np.float64)) * (rep + D[0].astype(np.float64) * xc)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("pool_axis", [0, 1])
def test_p10_two_directions_add(oracle_mod, pool_axis):
    """The gate is linear in the summed directions, so the two-direction layer equals the sum of
    the single-direction layers built from each slot's own filter and parameters."""
    rng = np.random.default_rng(1400 + pool_axis)
    B, h, w, E, N, R = 2, 3, 4, 5, 3, 2
    A_log, D, W_x, W_dt, b_dt = _rand_params(rng, 2, E, N, R)
    x, cw, cb = _conv_case(rng, B, h, w, E, 4, 2)
    z = rng.standard_normal((B, h, w, E)).astype(np.float32)
    both = oracle_mod.forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, 3, conv_w=cw, conv_b=cb)
    parts = 0.0
    for k, d in enumerate((1, 2)):
        sl = slice(k, k + 1)
        parts = parts + oracle_mod.forward(x, z, A_log[sl], D[sl], W_x[sl], W_dt[sl], b_dt[sl], pool_axis, d,
                                           conv_w=cw[sl], conv_b=cb[sl])
    np.testing.assert_allclose(both, parts, rtol=1e-12, atol=1e-13)


def test_p10_golden_hand_worked_conv_example(oracle_mod):
    with open(os.path.join(GOLDEN, "conv_1x3_hand.json")) as f:
        g = json.load(f)
    inp = {k: np.array(v, np.float32) for k, v in g["inputs"].items()}
    ln2 = math.log(2.0)
    for x, axis in ((inp["x"], g["pool_axis"]), (inp["x"].transpose(0, 2, 1, 3), 0)):  # and its 3x1 transpose
        inter = oracle_mod.forward_intermediates(x, inp["z"].reshape(x.shape), inp["A_log"], inp["D"], inp["W_x"],
                                                 inp["W_dt"], inp["b_dt"], axis, g["dir_flags"],
                                                 conv_w=inp["conv_w"], conv_b=inp["conv_b"])
        np.testing.assert_array_equal(inter["xc"][0].ravel(), g["expected"]["xc_fwd"])
        np.testing.assert_array_equal(inter["xc"][1].ravel(), g["expected"]["xc_bwd"])
        ys = np.array(g["expected"]["ys_over_ln2"]) * ln2
        np.testing.assert_allclose(inter["ys"].ravel(), ys, rtol=1e-14)
        z = inp["z"].astype(np.float64).ravel()
        y = z / (1 + np.exp(-z)) * (ys + np.array(g["expected"]["skip"]))
        np.testing.assert_allclose(inter["y"].ravel(), y, rtol=1e-14)
        full = oracle_mod.forward(x, inp["z"].reshape(x.shape), inp["A_log"], inp["D"], inp["W_x"], inp["W_dt"],
                                  inp["b_dt"], axis, g["dir_flags"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
        np.testing.assert_allclose(full.ravel(), y, rtol=1e-14)


# ---------------------------------------------------------------------------------------------
# p11: the scans' states (what a training forward keeps for the gradient), pinned to the scan
#      output the pins above fix and to scipy's first-order filter.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
@pytest.mark.parametrize("T", [4, 9])
def test_p11_states_read_out_by_C_give_the_scan_output(oracle_mod, dir_flags, T):
    """ys[t] = sum over directions of C_t . (the state after the direction's step at t), and the
    state after step s is the one entering step s + 1."""
    rng = np.random.default_rng(300 + 10 * T + dir_flags)
    B, E, N, R = 2, 3, 4, 2
    nd = oracle_mod.nd_of(dir_flags)
    A_log = rng.uniform(-1, 1, size=(nd, E, N)).astype(np.float32)
    xbar = rng.standard_normal((B, T, E))
    delta = rng.uniform(0.01, 0.8, size=(nd, B, T, E))
    u = rng.standard_normal((nd, B, T, R + 2 * N))
    for zoh in (False, True):
        ys = oracle_mod.scan(xbar, delta, u, A_log, R, N, dir_flags, zoh)
        hin = oracle_mod.scan_states(xbar, delta, u, A_log, R, N, dir_flags, zoh)
        assert hin.shape == (nd, B, T, E, N) and not hin[:, :, 0].any()
        fwd = [k == 0 if nd == 2 else dir_flags == 1 for k in range(nd)]
        checked = 0
        for t in range(T):
            steps = [t if fwd[k] else T - 1 - t for k in range(nd)]
            if max(steps) + 1 >= T:
                continue  # the state after a scan's last step is not stored
            for b in range(B):
                read = sum(np.einsum("en,n->e", hin[k, b, steps[k] + 1], u[k, b, t, R + N:]) for k in range(nd))
                np.testing.assert_allclose(read, ys[b, t], rtol=1e-12, atol=1e-12)
                checked += 1
        assert checked > 0


def test_p11_states_lti_match_scipy_lfilter(oracle_mod):
    """Constant Delta and B: each state is a first-order IIR filter of the input in scan order,
    h_after = lfilter([1], [1, -a], Delta B x), and the stored state is the one before the step."""
    rng = np.random.default_rng(11)
    B, T, E, N, R = 1, 23, 2, 3, 1
    A_log = rng.uniform(-1, 1, size=(1, E, N)).astype(np.float32)
    xbar = rng.standard_normal((B, T, E))
    dval = rng.uniform(0.05, 0.5, size=E)
    delta = np.broadcast_to(dval[None, None, None, :], (1, B, T, E)).copy()
    Bn = rng.standard_normal(N)
    u = rng.standard_normal((1, B, T, R + 2 * N))
    u[0, 0, :, R:R + N] = Bn[None, :]
    for dir_flags in (1, 2):
        hin = oracle_mod.scan_states(xbar, delta, u, A_log, R, N, dir_flags)
        for e in range(E):
            for n in range(N):
                a = math.exp(-dval[e] * math.exp(float(A_log[0, e, n])))
                seq = xbar[0, :, e] * dval[e] * Bn[n]
                if dir_flags == 2:
                    seq = seq[::-1]  # scan order
                after = scipy.signal.lfilter([1.0], [1.0, -a], seq)
                ref = np.concatenate([[0.0], after[:-1]])
                np.testing.assert_allclose(hin[0, 0, :, e, n], ref, rtol=1e-11, atol=1e-12)
