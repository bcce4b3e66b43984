"""Pins of the fp64 gradient oracle (CPU only).

The gradient oracle is pinned to the forward oracle, itself pinned by ``test_oracle_pins.py``:
for the scalar loss L = sum(dy * y), every gradient it returns must equal the central finite
difference of L, taken through the forward oracle with steps of 2^-12 that fp32 represents
exactly.  The truncation error of that difference is O(step^2), about 1e-7 of the gradient, and
the loss is fp64, so the agreement asked for (1e-6 of the largest gradient of each array) leaves
no room for a dropped term, a wrong sign or a transposed index.  Two invariants besides: a
masked call that keeps every token in grid order has the dense call's gradient, and a rejected
id gets no gradient.
"""
import numpy as np
import pytest

STEP = 2.0 ** -12
PARAMS = ("A_log", "D", "W_x", "W_dt", "b_dt")


def _params(rng, nd, E, N, R):
    return {
        "A_log": rng.uniform(-1.0, 1.0, (nd, E, N)).astype(np.float32),
        "D": rng.uniform(0.5, 1.5, (nd, E)).astype(np.float32),
        "W_x": rng.uniform(-1.0, 1.0, (nd, R + 2 * N, E)).astype(np.float32),
        "W_dt": rng.uniform(-0.5, 0.5, (nd, E, R)).astype(np.float32),
        "b_dt": np.log(np.expm1(rng.uniform(0.05, 0.6, (nd, E)))).astype(np.float32),
    }


def _case(rng, masked, B=2, h=3, w=4, E=4, N=3, R=2, K=7, nd=2):
    P = _params(rng, nd, E, N, R)
    if masked:
        idx = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
        shape, kw = (B, K, E), {"keep_idx": idx, "h": h, "w": w}
    else:
        shape, kw = (B, h, w, E), {}
    x = rng.standard_normal(shape).astype(np.float32)
    z = rng.standard_normal(shape).astype(np.float32)
    dy = rng.standard_normal(shape).astype(np.float32)
    return x, z, dy, P, kw


def _fd_check(oracle_mod, rng, x, z, dy, P, kw, pool_axis, dir_flags, zoh, scale, per_array=6, ln=None):
    """ln: None, or (gamma, beta, eps) for the post-SSM LayerNorm (then its gradients are checked too)."""
    lnkw = {} if ln is None else {"ln_gamma": ln[0], "ln_beta": ln[1], "ln_eps": ln[2]}
    g = oracle_mod.backward(x, z, P["A_log"], P["D"], P["W_x"], P["W_dt"], P["b_dt"], dy, pool_axis, dir_flags,
                            pool_scale=scale, zoh_exact=zoh, **kw, **lnkw)
    dy64 = dy.astype(np.float64)

    def loss(**over):
        a = {"x": x, "z": z, **P, **lnkw, **over}
        extra = {} if ln is None else {"ln_gamma": a["ln_gamma"], "ln_beta": a["ln_beta"], "ln_eps": a["ln_eps"]}
        y = oracle_mod.forward(a["x"], a["z"], a["A_log"], a["D"], a["W_x"], a["W_dt"], a["b_dt"], pool_axis,
                               dir_flags, pool_scale=scale, zoh_exact=zoh, **kw, **extra)
        return float(np.sum(dy64 * y))

    arrays = [("x", x), ("z", z)] + [(k, P[k]) for k in PARAMS]
    if ln is not None:
        arrays += [("ln_gamma", ln[0]), ("ln_beta", ln[1])]
    for name, arr in arrays:
        grad = g["d" + name]
        assert grad.shape == arr.shape
        scale_ref = np.abs(grad).max()
        assert scale_ref > 0, name
        for flat in rng.choice(arr.size, size=min(per_array, arr.size), replace=False):
            ap, am = arr.copy(), arr.copy()
            ap.flat[flat] += np.float32(STEP)
            am.flat[flat] -= np.float32(STEP)
            fd = (loss(**{name: ap}) - loss(**{name: am})) / (float(ap.flat[flat]) - float(am.flat[flat]))
            assert abs(fd - grad.flat[flat]) <= 1e-6 * scale_ref, (name, flat, fd, grad.flat[flat])
    return g


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
@pytest.mark.parametrize("zoh", [False, True])
def test_dense_gradient_equals_finite_differences(pool_axis, dir_flags, zoh, oracle_mod=None):
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(100 + 10 * pool_axis + 2 * dir_flags + zoh)
    nd = bin(dir_flags).count("1")
    x, z, dy, P, kw = _case(rng, False, nd=nd)
    _fd_check(oracle_mod, rng, x, z, dy, P, kw, pool_axis, dir_flags, zoh, 0.7)


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("zoh", [False, True])
def test_masked_gradient_equals_finite_differences(pool_axis, zoh, oracle_mod=None):
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(200 + pool_axis + 2 * zoh)
    x, z, dy, P, kw = _case(rng, True)
    _fd_check(oracle_mod, rng, x, z, dy, P, kw, pool_axis, 3, zoh, 1.0)


@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("pool_axis", [0, 1])
def test_layernorm_gradient_equals_finite_differences(masked, pool_axis, oracle_mod=None):
    """With the post-SSM LayerNorm: every gradient, dgamma and dbeta included (E = 6 channels, so
    the normalisation's mean and projection terms are far from negligible)."""
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(600 + 2 * masked + pool_axis)
    x, z, dy, P, kw = _case(rng, masked, E=6)
    gamma = rng.uniform(0.5, 1.5, 6).astype(np.float32)
    beta = rng.uniform(-0.5, 0.5, 6).astype(np.float32)
    _fd_check(oracle_mod, rng, x, z, dy, P, kw, pool_axis, 3, False, 1.0, ln=(gamma, beta, 1e-5))


def test_longer_sequence_gradient_equals_finite_differences(oracle_mod=None):
    """T = 9 with N = 5 and R = 3: the adjoint recurrence runs long enough for an off-by-one
    in its step order to show."""
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(300)
    x, z, dy, P, kw = _case(rng, False, B=1, h=9, w=2, E=3, N=5, R=3)
    _fd_check(oracle_mod, rng, x, z, dy, P, kw, 0, 3, False, 1.0, per_array=10)


def test_masked_all_kept_equals_dense(oracle_mod=None):
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(400)
    B, h, w, E = 2, 3, 4, 4
    x, z, dy, P, _ = _case(rng, False, B=B, h=h, w=w, E=E)
    args = (P["A_log"], P["D"], P["W_x"], P["W_dt"], P["b_dt"])
    for axis in (0, 1):
        gd = oracle_mod.backward(x, z, *args, dy, axis, 3)
        idx = np.tile(np.arange(h * w, dtype=np.int32), (B, 1))
        flat = lambda a: a.reshape(B, h * w, E)  # noqa: E731
        gm = oracle_mod.backward(flat(x), flat(z), *args, flat(dy), axis, 3, keep_idx=idx, h=h, w=w)
        np.testing.assert_allclose(gm["dx"], flat(gd["dx"]), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(gm["dz"], flat(gd["dz"]), rtol=1e-12, atol=1e-12)
        for k in PARAMS:
            np.testing.assert_allclose(gm["d" + k], gd["d" + k], rtol=1e-11, atol=1e-12)


def test_rejected_id_gets_no_gradient(oracle_mod=None):
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(500)
    x, z, dy, P, kw = _case(rng, True, B=1)
    kw["keep_idx"] = kw["keep_idx"].copy()
    kw["keep_idx"][0, 3] = kw["keep_idx"][0, 1]  # a duplicate id: the second copy is rejected
    g = oracle_mod.backward(x, z, P["A_log"], P["D"], P["W_x"], P["W_dt"], P["b_dt"], dy, 0, 3,
                            allow_bad_index=True, **kw)
    assert g["status"] == oracle_mod.FVO_BAD_INDEX
    assert not g["dx"][0, 3].any() and not g["dz"][0, 3].any()
    assert g["dx"][0, 1].any() and g["dz"][0, 1].any()


def test_gradient_axis_and_direction_symmetries(oracle_mod=None):
    """Pooling over h is pooling over w of the transposed grid, and a backward-only scan is a
    forward-only scan of the sequence read in reverse: the gradients must map the same way."""
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(700)
    B, h, w, E, N, R = 2, 3, 5, 4, 3, 2
    x, z, dy, P, _ = _case(rng, False, B=B, h=h, w=w, E=E, N=N, R=R)
    args = (P["A_log"], P["D"], P["W_x"], P["W_dt"], P["b_dt"])
    tr = lambda a: np.ascontiguousarray(a.transpose(0, 2, 1, 3))  # noqa: E731
    gh = oracle_mod.backward(x, z, *args, dy, 1, 3)
    gw = oracle_mod.backward(tr(x), tr(z), *args, tr(dy), 0, 3)
    np.testing.assert_allclose(gh["dx"], tr(gw["dx"]), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gh["dz"], tr(gw["dz"]), rtol=1e-12, atol=1e-13)
    for k in PARAMS:
        np.testing.assert_allclose(gh["d" + k], gw["d" + k], rtol=1e-11, atol=1e-13)
    # backward-only on x == forward-only on x flipped along the scan axis (POOL_W: axis h)
    one = {k: v[:1].copy() for k, v in P.items()}
    a1 = (one["A_log"], one["D"], one["W_x"], one["W_dt"], one["b_dt"])
    fl = lambda a: np.ascontiguousarray(a[:, ::-1])  # noqa: E731
    gb = oracle_mod.backward(x, z, *a1, dy, 0, 2)
    gf = oracle_mod.backward(fl(x), fl(z), *a1, fl(dy), 0, 1)
    np.testing.assert_allclose(gb["dx"], fl(gf["dx"]), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gb["dz"], fl(gf["dz"]), rtol=1e-12, atol=1e-13)
    for k in PARAMS:
        np.testing.assert_allclose(gb["d" + k], gf["d" + k], rtol=1e-11, atol=1e-13)


def test_masked_gradient_follows_a_permutation_of_the_kept_ids(oracle_mod=None):
    """Listing the kept tokens in another order permutes dx and dz the same way and leaves the
    parameter gradients unchanged."""
    import oracle
    oracle_mod = oracle_mod or oracle
    rng = np.random.default_rng(800)
    x, z, dy, P, kw = _case(rng, True)
    args = (P["A_log"], P["D"], P["W_x"], P["W_dt"], P["b_dt"])
    g0 = oracle_mod.backward(x, z, *args, dy, 0, 3, **kw)
    perm = rng.permutation(x.shape[1])
    kw2 = dict(kw, keep_idx=np.ascontiguousarray(kw["keep_idx"][:, perm]))
    g1 = oracle_mod.backward(np.ascontiguousarray(x[:, perm]), np.ascontiguousarray(z[:, perm]), *args,
                             np.ascontiguousarray(dy[:, perm]), 0, 3, **kw2)
    np.testing.assert_allclose(g1["dx"], g0["dx"][:, perm], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1["dz"], g0["dz"][:, perm], rtol=1e-12, atol=1e-13)
    for k in PARAMS:
        np.testing.assert_allclose(g1["d" + k], g0["d" + k], rtol=1e-11, atol=1e-13)
