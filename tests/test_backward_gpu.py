"""Parity of the layer's gradient (CUDA, through the C ABI) with the fp64 gradient oracle.

Each case runs the forward call, then the gradient call on its workspace, with every workspace
and output poisoned beforehand (NaN bytes), and compares dx, dz and the five parameter gradients
element by element: dx and dz at the layer's tolerance, the batch-summed parameter gradients at
the gradient tolerance (fv_testlib).  Shapes cover ragged channel blocks (E not a multiple of
64), partial state groups (N < 16), pooled lengths below, at and across the 16-step checkpoint
chunks, one or two directions, exact ZOH, pool_scale, the fused forward's workspace, masked
layers with empty rows and a rejected id, and the empty batch."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import GRAD_PARAM_ABS_RMS, assert_close  # noqa: E402
from pooled_selective_scan_b200 import _native as nat, inputs, ssm  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PARAMS = ("A_log", "D", "W_x", "W_dt", "b_dt")


def make_inputs(seed, B, h, w, E, N, R, nd, K=0, drop_row=None, pool_axis=0):
    d = inputs.params(E, N, R, nd, seed)
    rng = np.random.default_rng([seed, 99])
    # spread A and D so that every parameter gradient has structure to check
    d["A_log"] = (d["A_log"] + rng.uniform(-0.3, 0.3, d["A_log"].shape)).astype(np.float32)
    d["D"] = rng.uniform(0.5, 1.5, d["D"].shape).astype(np.float32)
    shp = (K, E) if K else (h, w, E)
    d["x"] = np.stack([inputs.image_x(seed, b, shp) for b in range(B)]) if B else np.empty((0,) + shp, np.float32)
    d["z"] = np.stack([inputs.image_z(seed, b, shp) for b in range(B)]) if B else np.empty((0,) + shp, np.float32)
    d["dy"] = np.stack([inputs.image_dy(seed, b, shp) for b in range(B)]) if B else np.empty((0,) + shp, np.float32)
    if K:
        ids = []
        for b in range(B):
            pool = np.arange(h * w)
            if drop_row is not None:  # leave one pooled row (grid row, or column under POOL_H) empty
                pool = pool[(pool // w if pool_axis == 0 else pool % w) != drop_row]
            ids.append(np.random.default_rng([seed, 3, b]).permutation(pool)[:K])
        d["keep_idx"] = np.stack(ids).astype(np.int32)
    return d


def gpu_grads(d, pool_axis, dir_flags, h, w, pool_scale=1.0, zoh_exact=False, path="auto", ln_eps=1e-5,
              keep_states=False, out=None):
    """d may hold ln_gamma and ln_beta: then the layer has the post-SSM LayerNorm.  out (a dict),
    if given, receives y and both workspaces."""
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in d.items()}
    keep = t.get("keep_idx")
    ln = "ln_gamma" in t
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, dir_flags, keep, h, w, pool_scale, zoh_exact,
                            path, ln, ln_eps, keep_states=keep_states)
    lnkw = dict(ln_gamma=t.get("ln_gamma"), ln_beta=t.get("ln_beta"), ln_eps=ln_eps, keep_states=keep_states)
    fws = ssm.alloc_workspace(shape, dev)
    fws.fill_(0xFF)
    y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], pool_axis, dir_flags,
                    keep_idx=keep, h=h, w=w, pool_scale=pool_scale, zoh_exact=zoh_exact, workspace=fws, path=path,
                    **lnkw)
    fstatus = ssm.device_status(fws)
    bws = torch.full((max(ssm.backward_workspace_size(shape), 256),), 0xFF, dtype=torch.uint8, device=dev)
    grads = {"dx": torch.full_like(t["x"], float("nan")), "dz": torch.full_like(t["z"], float("nan"))}
    for name in PARAMS + (("ln_gamma", "ln_beta") if ln else ()):
        grads["d" + name] = torch.full_like(t[name], float("nan"))
    ssm.backward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], t["dy"], fws, pool_axis,
                 dir_flags, keep_idx=keep, h=h, w=w, pool_scale=pool_scale, zoh_exact=zoh_exact, path=path,
                 grads=grads, workspace=bws, **lnkw)
    torch.cuda.synchronize()
    if out is not None:
        out.update(y=y.cpu().numpy(), fws=fws, bws=bws, shape=shape)
    return {k: v.cpu().numpy() for k, v in grads.items()}, fstatus, ssm.backward_launch_names(shape)


def oracle_grads(d, pool_axis, dir_flags, h, w, pool_scale=1.0, zoh_exact=False, allow_bad_index=False, ln_eps=1e-5):
    return oracle.backward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], d["dy"], pool_axis,
                           dir_flags, keep_idx=d.get("keep_idx"), h=h, w=w, pool_scale=pool_scale, zoh_exact=zoh_exact,
                           nthreads=8, allow_bad_index=allow_bad_index, ln_gamma=d.get("ln_gamma"),
                           ln_beta=d.get("ln_beta"), ln_eps=ln_eps)


def compare(got, ref, what):
    reps = {}
    for k in ("dx", "dz"):
        reps[k] = assert_close(got[k], ref[k], f"{what} {k}")
    for name in PARAMS + (("ln_gamma", "ln_beta") if "dln_gamma" in ref else ()):
        reps["d" + name] = assert_close(got["d" + name], ref["d" + name], f"{what} d{name}", GRAD_PARAM_ABS_RMS)
    print(what, {k: (round(v["max_abs_over_rms"], 9), round(v["max_err_over_bound"], 4)) for k, v in reps.items()})
    return reps


DENSE = [
    # B, h, w, E, N, R, pool_axis, dir_flags, zoh_exact, pool_scale, path
    (2, 14, 14, 384, 16, 12, 0, 3, False, 1.0, "auto"),
    (2, 14, 14, 384, 16, 12, 1, 3, False, 1.0, "auto"),
    (3, 13, 7, 68, 5, 3, 0, 1, False, 1.0, "staged"),
    (3, 13, 7, 68, 5, 3, 1, 2, True, 0.25, "staged"),
    (2, 40, 3, 132, 16, 7, 0, 3, False, 1.0, "staged"),
    (2, 5, 37, 64, 16, 4, 1, 3, True, 1.0, "staged"),
    (2, 16, 9, 256, 16, 16, 0, 3, False, 1.0, "staged"),
    (1, 1, 1, 4, 1, 1, 0, 3, False, 1.0, "staged"),
    (1, 6, 5, 2048, 16, 8, 1, 3, False, 1.0, "staged"),
    (2, 64, 64, 1024, 16, 64, 0, 3, False, 1.0, "fused"),
    (2, 64, 64, 1024, 16, 64, 0, 3, False, 1.0, "staged"),
]


@pytest.mark.parametrize("case", DENSE, ids=lambda c: "x".join(map(str, c[:6])) + f"-a{c[6]}d{c[7]}z{int(c[8])}{c[10]}")
def test_dense_gradient(case):
    B, h, w, E, N, R, axis, dirs, zoh, scale, path = case
    nd = bin(dirs).count("1")
    d = make_inputs(7, B, h, w, E, N, R, nd)
    got, fst, names = gpu_grads(d, axis, dirs, h, w, scale, zoh, path)
    assert fst == 0
    # the step sizes come from the forward workspace when its staged path wrote them (dt_rank >= 32)
    fwd_delta = R >= 32 and path == "staged"
    assert names[0] == "bwd_gate_dense_kernel" and len(names) == (7 if fwd_delta else 8)
    assert (names[1] == "dt_proj_kernel") == (not fwd_delta)
    ref = oracle_grads(d, axis, dirs, h, w, scale, zoh)
    compare(got, ref, f"dense {case}")


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("zoh", [False, True])
def test_masked_gradient_with_an_empty_row(pool_axis, zoh):
    h, w, E, N, R, K = 16, 16, 132, 16, 8, 100
    d = make_inputs(11, 2, h, w, E, N, R, 2, K=K, drop_row=3, pool_axis=pool_axis)
    got, fst, names = gpu_grads(d, pool_axis, 3, h, w, 1.0, zoh)
    assert fst == 0 and names[0] == "bwd_gate_masked_kernel"
    ref = oracle_grads(d, pool_axis, 3, h, w, 1.0, zoh)
    compare(got, ref, f"masked axis {pool_axis} zoh {zoh}")


def test_masked_gradient_rejected_id():
    """A repeated id: one copy is rejected (the forward reports FV_ERR_INDEX) and gets zero
    gradients.  Both copies carry the same x, z and dy, so the result is the same whichever copy
    the device keeps; compare the pair as a set and everything else element by element."""
    h, w, E, N, R, K = 8, 8, 64, 16, 4, 20
    d = make_inputs(13, 2, h, w, E, N, R, 2, K=K)
    k1, k2 = 2, 9
    d["keep_idx"][0, k2] = d["keep_idx"][0, k1]
    for key in ("x", "z", "dy"):
        d[key][0, k2] = d[key][0, k1]
    got, fst, _ = gpu_grads(d, 0, 3, h, w)
    assert fst == 4  # FV_ERR_INDEX
    ref = oracle_grads(d, 0, 3, h, w, allow_bad_index=True)
    assert ref["status"] == oracle.FVO_BAD_INDEX
    for key in ("dx", "dz"):
        g, r = got[key][0], ref[key][0]
        pair_g = sorted([g[k1], g[k2]], key=lambda v: float(np.abs(v).sum()))
        pair_r = sorted([r[k1], r[k2]], key=lambda v: float(np.abs(v).sum()))
        assert not pair_g[0].any() and not pair_r[0].any()
        assert_close(pair_g[1], pair_r[1], f"kept copy {key}")
        rest = [k for k in range(K) if k not in (k1, k2)]
        assert_close(g[rest], r[rest], f"other tokens {key}")
        assert_close(got[key][1], ref[key][1], f"clean sample {key}")
    for name in PARAMS:
        assert_close(got["d" + name], ref["d" + name], f"d{name}", GRAD_PARAM_ABS_RMS)


def test_empty_batch_zeroes_the_parameter_gradients():
    d = make_inputs(3, 0, 4, 4, 8, 2, 1, 2)
    got, fst, names = gpu_grads(d, 0, 3, 4, 4)
    assert names == []
    for name in PARAMS:
        assert got["d" + name].shape == d[name].shape and not got["d" + name].any()


@pytest.mark.parametrize("K,ln,R", [(0, False, 8), (48, False, 48), (0, True, 8), (100, True, 40)])
def test_gradient_is_bit_reproducible(K, ln, R):
    """Every batch sum runs over per-block partials added in a fixed order (no atomics): two calls
    give the same bits in dx, dz and every parameter gradient, dense and masked, with and without
    the LayerNorm, with the step sizes from either workspace."""
    d = make_inputs(5, 2, 16, 16, 128, 16, R, 2, K=K)
    if ln:
        rng = np.random.default_rng([5, 1])
        d["ln_gamma"] = rng.uniform(0.5, 1.5, 128).astype(np.float32)
        d["ln_beta"] = rng.uniform(-0.5, 0.5, 128).astype(np.float32)
    a, _, _ = gpu_grads(d, 0, 3, 16, 16, path="auto" if K else "staged")
    b, _, _ = gpu_grads(d, 0, 3, 16, 16, path="auto" if K else "staged")
    assert a.keys() == b.keys()
    for name in a:
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)


LN_CASES = [
    # B, h, w, E, N, R, pool_axis, K, path   (K > 0: masked, 75 % of the grid kept)
    (2, 14, 14, 384, 16, 12, 0, 0, "staged"),
    (2, 14, 14, 384, 16, 12, 1, 0, "staged"),
    (2, 64, 64, 1024, 16, 64, 0, 0, "fused"),
    (3, 13, 7, 68, 5, 3, 1, 0, "staged"),
    (2, 8, 8, 1536, 16, 48, 0, 48, "auto"),
    (1, 3, 5, 4096, 16, 8, 0, 0, "staged"),
    (2, 16, 16, 132, 16, 8, 1, 100, "auto"),
]


@pytest.mark.parametrize("case", LN_CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-a{c[6]}K{c[7]}{c[8]}")
def test_layernorm_gradient(case):
    """The gradient through the post-SSM LayerNorm (gamma, beta drawn around their init): up to
    E = 2048 the register kernel with 1 to 8 warps per token (E = 68, 132, 384 and 1024, 1536),
    above it the shared-memory-row kernel (E = 4096); dense on either forward path and masked."""
    B, h, w, E, N, R, axis, K, path = case
    d = make_inputs(17, B, h, w, E, N, R, 2, K=K)
    rng = np.random.default_rng([17, 5])
    d["ln_gamma"] = rng.uniform(0.5, 1.5, E).astype(np.float32)
    d["ln_beta"] = rng.uniform(-0.5, 0.5, E).astype(np.float32)
    got, fst, names = gpu_grads(d, axis, 3, h, w, path=path)
    assert fst == 0 and names[0] == ("bwd_ln_gate_reg_kernel" if E <= 2048 else "bwd_ln_gate_kernel")
    ref = oracle_grads(d, axis, 3, h, w)
    compare(got, ref, f"layernorm {case}")


KEEP_CASES = [
    # B, h, w, E, N, R, pool_axis, dir_flags, zoh_exact, path, K
    (2, 40, 3, 132, 16, 7, 0, 3, False, "staged", 0),    # T = 40: two whole chunks, then 8 steps
    (3, 13, 7, 68, 5, 3, 1, 2, True, "staged", 0),       # T = 7 < 8, one direction, exact ZOH, N = 5
    (2, 64, 64, 1024, 16, 64, 0, 3, False, "fused", 0),  # the fused launch keeps the states
    (2, 64, 64, 1024, 16, 64, 0, 3, False, "staged", 0),  # step sizes from the dt_proj kernel
    (2, 16, 16, 132, 16, 8, 1, 3, False, "auto", 100),   # masked
]


@pytest.mark.parametrize("case", KEEP_CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-{c[9]}K{c[10]}")
def test_gradient_from_kept_states(case):
    """FV_FLAG_KEEP_STATES: the forward stores the scan states every 8 steps and the gradient reads
    them instead of running the recurrences a first time.  y keeps its bits, the gradient matches
    the oracle, and the kept states match the oracle's states at the steps their slots stand for
    and the ones the gradient computes itself without the flag (slots of chunks of at most 8
    steps are never written)."""
    B, h, w, E, N, R, axis, dirs, zoh, path, K = case
    nd = bin(dirs).count("1")
    d = make_inputs(23, B, h, w, E, N, R, nd, K=K)
    kept, plain = {}, {}
    got, fst, names = gpu_grads(d, axis, dirs, h, w, 1.0, zoh, path, keep_states=True, out=kept)
    _, fst0, names0 = gpu_grads(d, axis, dirs, h, w, 1.0, zoh, path, out=plain)
    assert fst == 0 and fst0 == 0 and names == names0
    np.testing.assert_array_equal(kept["y"], plain["y"])
    compare(got, oracle_grads(d, axis, dirs, h, w, 1.0, zoh), f"kept states {case}")
    # the states themselves: forward's (kept) against the gradient call's own pass
    T = h if axis == 0 else w
    nck = 2 * (-(-T // 16))
    L = nat.FvWsLayout()
    a = kept["shape"].args()
    assert nat.lib().fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    Lb = nat.FvBwdWsLayout()
    a0 = plain["shape"].args()
    assert nat.lib().fastvim_ssm_backward_workspace_layout(ctypes.byref(a0), ctypes.byref(Lb)) == nat.FV_OK
    n = B * nd * nck * E * 16
    fk = kept["fws"][L.ckpt:L.ckpt + 4 * n].view(torch.float32).cpu().numpy().reshape(B, nd, nck, E, 16)
    bk = plain["bws"][Lb.ckpt:Lb.ckpt + 4 * n].view(torch.float32).cpu().numpy().reshape(B, nd, nck, E, 16)
    # the oracle's states entering every scan step, [nd][B][T][E][N]
    inter = oracle.forward_intermediates(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], axis,
                                         dirs, keep_idx=d.get("keep_idx"), h=h, w=w, zoh_exact=zoh)
    hin = oracle.scan_states(inter["xbar"], inter["delta"], inter["u"], d["A_log"], R, N, dirs, zoh)
    fwd_slot = [k == 0 if nd == 2 else bool(dirs & 1) for k in range(nd)]
    nchunks = nck // 2
    for k in range(nd):
        lens = [min(16, T - 16 * (it if fwd_slot[k] else nchunks - 1 - it)) for it in range(nchunks)]
        for c in range(nck):
            it, half = divmod(c, 2)
            if half == 1 and lens[it] <= 8:
                continue  # no second half in this chunk
            step = sum(lens[:it]) + 8 * half  # the scan step the slot's state enters
            assert not np.isnan(fk[:, k, c]).any()
            assert_close(fk[:, k, c, :, :N], hin[k, :, step], f"states dir {k} slot {c} vs oracle")
            assert_close(fk[:, k, c], bk[:, k, c], f"states dir {k} slot {c}")
            if c == 0:
                assert not fk[:, k, c].any()  # every scan starts from zero
            assert not fk[:, k, c, :, N:].any()  # states past N stay zero
