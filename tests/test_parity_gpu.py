"""Parity of the CUDA layer with the fp64 oracle on the same seeded inputs (needs a B200).

Small layers are compared element by element, intermediates included (pooled tokens, the
projections, the scan output, the masked row buckets), over shapes that span several tiles
and ragged tails: channels not a multiple of the 32-channel projection chunk or of a 4-lane
scan tile, more than 256 float4 slots per token, state counts that leave lanes half empty,
T = 1, both pool axes, each direction alone, exact ZOH, a pooling scale, masked grids with
empty rows, all-kept and permuted keep lists, and rejected indices.  Full-size workloads are
in test_parity_full_gpu.py.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close, gpu_forward  # noqa: E402
from pooled_selective_scan_b200 import inputs  # noqa: E402
from pooled_selective_scan_b200.configs import CONFIGS  # noqa: E402

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def rand_layer(seed, B, h, w, E, N, R, dir_flags, K=0, dt_hi=0.1):
    """Seeded layer with the init distributions of the workload recipe at arbitrary sizes."""
    rng = np.random.default_rng(seed)
    nd = oracle.nd_of(dir_flags)
    p = inputs.params(E, N, R, nd, seed)
    # random A_log too, so that every state has its own decay
    p["A_log"] = rng.uniform(-1.0, 2.5, size=(nd, E, N)).astype(np.float32)
    p["D"] = rng.uniform(0.5, 1.5, size=(nd, E)).astype(np.float32)
    shp = (B, K, E) if K else (B, h, w, E)
    p["x"] = rng.standard_normal(shp, dtype=np.float32)
    p["z"] = rng.standard_normal(shp, dtype=np.float32)
    if K:
        p["keep_idx"] = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
    return p


def check_layer(p, pool_axis, dir_flags, h=None, w=None, pool_scale=1.0, zoh_exact=False):
    """Every implementation of the layer against the oracle, intermediates and output: the staged
    kernels and (dense) the single persistent launch."""
    keep = p.get("keep_idx")
    ref = oracle.forward_intermediates(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"],
                                       pool_axis, dir_flags, keep_idx=keep, h=h, w=w, pool_scale=pool_scale,
                                       zoh_exact=zoh_exact)
    rep = None
    for path in (("staged",) if keep is not None else ("staged", "fused")):
        got = gpu_forward(p, pool_axis, dir_flags, h=h, w=w, pool_scale=pool_scale, zoh_exact=zoh_exact, path=path)
        assert got["status"] == 0, path
        assert (got["launches"] == ["fused_layer_kernel"]) == (path == "fused")
        if keep is not None:
            assert np.array_equal(got["row_of"], ref["row_of"])
            assert np.array_equal(got["row_off"], ref["row_off"])
            assert np.array_equal(got["row_tok"], ref["row_tok"])
        assert_close(got["xbar"], ref["xbar"], f"{path} xbar")
        assert_close(got["u"], ref["u"], f"{path} u")
        assert_close(got["ys"], ref["ys"], f"{path} ys")
        rep = assert_close(got["y"], ref["y"], f"{path} y")
    return rep


def test_config0_tiny_fastvim_t():
    cfg = CONFIGS[0]
    d = inputs.layer_inputs(cfg)
    rep = check_layer(d, cfg.pool_axes[0], cfg.dir_flags)
    assert rep["max_abs_over_rms"] < 1e-5


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
def test_ragged_dense(pool_axis, dir_flags):
    p = rand_layer(11 + 3 * pool_axis + dir_flags, B=3, h=5, w=7, E=20, N=16, R=3, dir_flags=dir_flags)
    check_layer(p, pool_axis, dir_flags)


@pytest.mark.parametrize("N", [1, 3, 4, 6, 8, 13, 16])
def test_state_counts(N):
    p = rand_layer(40 + N, B=2, h=9, w=4, E=72, N=N, R=5, dir_flags=3)
    check_layer(p, 0, 3)


@pytest.mark.parametrize("R,N", [(32, 3), (36, 6), (33, 16), (64, 16), (61, 16)])
def test_dt_proj_copy_paths(R, N):
    """The step-size GEMM (dt_rank >= 32) copies its operands 16 bytes at a time when every row of u
    (R + 2N floats) and of W_dt (R floats) starts on 16 bytes, 4 bytes at a time otherwise; R above
    32 takes two or more slices of the tensor-core K loop."""
    p = rand_layer(70 + R + N, B=3, h=11, w=5, E=136, N=N, R=R, dir_flags=3)
    check_layer(p, 0, 3)


@pytest.mark.parametrize("E,R", [(4, 1), (100, 7), (1032, 40), (1536, 48)])
def test_channel_counts(E, R):
    p = rand_layer(60 + E, B=2, h=3, w=6, E=E, N=16, R=R, dir_flags=3)
    check_layer(p, 1, 3)


@pytest.mark.parametrize("h,w,pool_axis", [(1, 9, 0), (9, 1, 1), (2, 2, 0), (1, 1, 0), (130, 3, 0), (3, 140, 1)])
def test_degenerate_and_long_grids(h, w, pool_axis):
    p = rand_layer(80 + h + w, B=2, h=h, w=w, E=36, N=16, R=4, dir_flags=3)
    check_layer(p, pool_axis, 3)


def test_exact_zoh_and_pool_scale():
    p = rand_layer(90, B=2, h=8, w=6, E=68, N=16, R=6, dir_flags=3)
    check_layer(p, 0, 3, zoh_exact=True)
    check_layer(p, 1, 3, pool_scale=0.25)


def test_large_steps():
    # step sizes up to ~3 make Abar small: the recurrence forgets quickly
    p = rand_layer(91, B=2, h=16, w=5, E=64, N=16, R=8, dir_flags=3)
    p["b_dt"] = np.full_like(p["b_dt"], 3.0)
    check_layer(p, 0, 3)


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("K", [1, 5, 20, 64])
def test_masked_small(pool_axis, K):
    p = rand_layer(100 + K + pool_axis, B=3, h=8, w=8, E=36, N=16, R=4, dir_flags=3, K=K)
    check_layer(p, pool_axis, 3, h=8, w=8)


def test_masked_nonsquare_and_wide():
    p = rand_layer(120, B=2, h=5, w=12, E=1040, N=16, R=16, dir_flags=3, K=33)
    check_layer(p, 0, 3, h=5, w=12)
    check_layer(p, 1, 3, h=5, w=12)


@pytest.mark.parametrize("lag", ["3", "4", "5", "9"])
def test_fused_pipeline_lags(lag, monkeypatch):
    monkeypatch.setenv("FASTVIM_FUSED_LAG", lag)
    p = rand_layer(125, B=7, h=24, w=20, E=136, N=16, R=6, dir_flags=3)
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3)
    got = gpu_forward(p, 0, 3, path="fused", intermediates=False)
    assert got["status"] == 0 and got["launches"] == ["fused_layer_kernel"]
    assert_close(got["y"], ref)


def test_path_auto_choice():
    from pooled_selective_scan_b200 import ssm
    big = ssm.LayerShape(B=2, h=128, w=128, E=384, N=16, R=12, pool_axis=0, dir_flags=3)
    small = ssm.LayerShape(B=2, h=14, w=14, E=384, N=16, R=12, pool_axis=0, dir_flags=3)
    masked = ssm.LayerShape(B=2, h=64, w=64, E=384, N=16, R=12, pool_axis=0, dir_flags=3, K=100)
    assert ssm.launch_names(big) == ["fused_layer_kernel"]
    assert ssm.launch_names(small) == ["pool_dense_kernel", "proj_gemm_kernel", "scan_seq_kernel", "epilogue_dense_kernel"]
    assert ssm.launch_names(masked)[0] == "mask_bucket_kernel"


def test_masked_all_kept_equals_dense():
    h, w = 6, 7
    p = rand_layer(130, B=2, h=h, w=w, E=44, N=16, R=4, dir_flags=3)
    dense = gpu_forward(p, 0, 3, intermediates=False)["y"]
    q = dict(p)
    q["x"] = p["x"].reshape(2, h * w, 44)
    q["z"] = p["z"].reshape(2, h * w, 44)
    q["keep_idx"] = np.tile(np.arange(h * w, dtype=np.int32), (2, 1))
    masked = gpu_forward(q, 0, 3, h=h, w=w, intermediates=False)["y"]
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3)
    assert_close(dense, ref)
    assert_close(masked.reshape(dense.shape), ref)


def test_masked_permutation_covariance():
    p = rand_layer(131, B=2, h=8, w=8, E=32, N=16, R=4, dir_flags=3, K=24)
    y = gpu_forward(p, 0, 3, h=8, w=8, intermediates=False)["y"]
    perm = np.random.default_rng(5).permutation(24)
    q = dict(p, x=p["x"][:, perm], z=p["z"][:, perm], keep_idx=p["keep_idx"][:, perm])
    yp = gpu_forward(q, 0, 3, h=8, w=8, intermediates=False)["y"]
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3,
                         keep_idx=p["keep_idx"], h=8, w=8)
    assert_close(y, ref)
    assert_close(yp, ref[:, perm])


@pytest.mark.parametrize("masked", [False, True])
def test_host_entry_point_pipelines_chunks(masked):
    """Over 64 MB of x, the host entry point runs the batch as chunks of images (here 3 + 2): y
    equals the device entry point's bit for bit and the oracle within tolerance, and a bad keep
    index in the first chunk is still reported after the last chunk ran clean."""
    from pooled_selective_scan_b200 import ssm
    if masked:
        h = w = 64
        p = rand_layer(181, B=5, h=h, w=w, E=1152, N=16, R=8, dir_flags=3, K=3000)
    else:
        h = w = None
        p = rand_layer(182, B=5, h=48, w=48, E=1536, N=16, R=8, dir_flags=3)
    assert p["x"].nbytes > 64 << 20
    t = {k: torch.from_numpy(v).pin_memory() for k, v in p.items()}
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 0, 3, t.get("keep_idx"), h, w)
    run = ssm.HostForward(shape)
    y_host = torch.empty(t["x"].shape, dtype=torch.float32).pin_memory()
    run(t, y_host)
    assert ssm.device_status(run.workspace) == 0
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3,
                         keep_idx=p.get("keep_idx"), h=h, w=w)
    assert_close(y_host.numpy(), ref)
    dev = gpu_forward(p, 0, 3, h=h, w=w, intermediates=False)["y"]
    assert np.array_equal(dev, y_host.numpy())
    if masked:
        t["keep_idx"][0, 7] = h * w  # out of range, in image 0 (first chunk)
        run(t, y_host)
        assert ssm.device_status(run.workspace) == 4  # FV_ERR_INDEX
        assert_close(y_host.numpy()[3:], ref[3:])  # the second chunk is untouched by it


@pytest.mark.parametrize("bad", ["dup", "neg", "big"])
def test_masked_bad_index_reported_on_device(bad):
    p = rand_layer(140, B=2, h=4, w=4, E=16, N=16, R=2, dir_flags=3, K=6)
    if bad == "dup":
        p["keep_idx"][1, 5] = p["keep_idx"][1, 0]
    elif bad == "neg":
        p["keep_idx"][0, 2] = -7
    else:
        p["keep_idx"][0, 3] = 16
    got = gpu_forward(p, 0, 3, h=4, w=4)
    assert got["status"] == 4  # FV_ERR_INDEX
    assert (got["row_of"] < 0).sum() == 1
    # the sample without a bad id is still computed exactly as the oracle does
    good = 1 if bad != "dup" else 0
    ref = oracle.forward(p["x"][good:good + 1], p["z"][good:good + 1], p["A_log"], p["D"], p["W_x"], p["W_dt"],
                         p["b_dt"], 0, 3, keep_idx=p["keep_idx"][good:good + 1], h=4, w=4)
    assert_close(got["y"][good:good + 1], ref)
    # and a following good call on the same workspace-free path reports OK
    p["keep_idx"] = np.stack([np.random.default_rng(3).permutation(16)[:6] for _ in range(2)]).astype(np.int32)
    assert gpu_forward(p, 0, 3, h=4, w=4)["status"] == 0


def test_empty_batch():
    from pooled_selective_scan_b200 import ssm
    p = rand_layer(150, B=1, h=4, w=4, E=16, N=16, R=2, dir_flags=3)
    dev = torch.device("cuda")
    x = torch.empty((0, 4, 4, 16), device=dev)
    prm = {k: torch.from_numpy(p[k]).to(dev) for k in ("A_log", "D", "W_x", "W_dt", "b_dt")}
    y = ssm.forward(x, x.clone(), prm["A_log"], prm["D"], prm["W_x"], prm["W_dt"], prm["b_dt"], 0, 3)
    torch.cuda.synchronize()
    assert y.shape == (0, 4, 4, 16)


def test_repeated_calls_are_deterministic():
    p = rand_layer(160, B=4, h=16, w=16, E=96, N=16, R=6, dir_flags=3, K=100)
    a = gpu_forward(p, 0, 3, h=16, w=16)
    b = gpu_forward(p, 0, 3, h=16, w=16)
    for k in ("y", "xbar", "u", "ys", "row_tok"):
        assert np.array_equal(a[k], b[k]), k


def test_streams_and_noncurrent_stream():
    from pooled_selective_scan_b200 import ssm
    p = rand_layer(170, B=2, h=8, w=8, E=64, N=16, R=4, dir_flags=3)
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(v).to(dev) for k, v in p.items()}
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], 0, 3)
    s.synchronize()
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3)
    assert_close(y.cpu().numpy(), ref)


def test_host_entry_point_matches_device_entry_point():
    from pooled_selective_scan_b200 import ssm
    p = rand_layer(180, B=3, h=10, w=12, E=48, N=16, R=4, dir_flags=3)
    t = {k: torch.from_numpy(v).pin_memory() for k, v in p.items()}
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 1, 3)
    run = ssm.HostForward(shape)
    y_host = torch.empty(t["x"].shape, dtype=torch.float32).pin_memory()
    run(t, y_host)
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 1, 3)
    assert_close(y_host.numpy(), ref)
    dev = gpu_forward(p, 1, 3, intermediates=False)["y"]
    assert np.array_equal(dev, y_host.numpy())


@pytest.mark.parametrize("path", ["staged", "fused"])
def test_longest_pooled_sequence(path):
    # T = 4096 pooled tokens (the largest the library takes): 256 scan chunks of 16 steps
    p = rand_layer(500, B=1, h=4096, w=3, E=8, N=16, R=2, dir_flags=3)
    got = gpu_forward(p, 0, 3, intermediates=False, path=path)
    assert got["status"] == 0
    ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3)
    assert_close(got["y"], ref)


@pytest.mark.parametrize("h,w,E,N,R,pool_axis,dir_flags", [(1, 1, 4, 1, 1, 0, 3), (1, 7, 4, 1, 1, 1, 1),
                                                          (9, 1, 8, 2, 1, 0, 2), (1, 9, 12, 3, 2, 0, 3)])
def test_smallest_layers(h, w, E, N, R, pool_axis, dir_flags):
    p = rand_layer(510 + h + w, B=3, h=h, w=w, E=E, N=N, R=R, dir_flags=dir_flags)
    for path in ("staged", "fused"):
        got = gpu_forward(p, pool_axis, dir_flags, intermediates=False, path=path)
        assert got["status"] == 0
        ref = oracle.forward(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], pool_axis, dir_flags)
        assert_close(got["y"], ref)


def test_masked_largest_grid():
    # a 1024 x 1024 grid (2^20 ids, the masked limit) with 300 kept tokens per sample
    p = rand_layer(520, B=2, h=1024, w=1024, E=16, N=16, R=2, dir_flags=3, K=300)
    got = gpu_forward(p, 1, 3, h=1024, w=1024)
    assert got["status"] == 0
    ref = oracle.forward_intermediates(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 1, 3,
                                       keep_idx=p["keep_idx"], h=1024, w=1024)
    assert np.array_equal(got["row_of"], ref["row_of"])
    assert_close(got["y"], ref["y"])


def test_events_bracket_every_staged_launch():
    """fastvim_ssm_forward_events records a start and an end event around each launch; every
    bracket has a positive duration and the result still matches the oracle."""
    from pooled_selective_scan_b200 import ssm, workload
    from pooled_selective_scan_b200.configs import by_name
    cfg = by_name("fastvim_t_224")
    dev = torch.device("cuda")
    t = workload.layer_tensors(cfg, dev)
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 0, 3, path="staged")
    y = torch.empty_like(t["x"])
    ws = ssm.alloc_workspace(shape, dev)
    fwd = ssm.BoundForward(shape, t, y, ws)
    n = fwd.n_launch
    assert n == 4
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
    fwd.run_events(evs)
    torch.cuda.synchronize()
    assert ssm.device_status(ws) == 0
    d = [evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(n)]
    assert all(v > 0 for v in d)
    ref = oracle.forward(*(t[k][:4].cpu().numpy() if k in ("x", "z") else t[k].cpu().numpy()
                           for k in ("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt")), 0, 3)
    assert_close(y[:4].cpu().numpy(), ref)
