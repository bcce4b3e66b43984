"""Parity of the layer with the block's Conv1D in front (x = the Conv1D's input) against the fp64
oracle, on the GPU.

Each direction convolves x with its own depthwise filter along the block's sequence (the pooled
lines in order, tokens along each line; the backward filter over the reversed sequence), pools,
projects and scans its own convolved tokens, and the skip adds each direction's D times its own
convolved input.  Compared element by element, intermediates included (the per-direction pooled
tokens, the projections, the scan output), over filter widths 1-4, with and without the SiLU
after the filter, each direction alone and both, both pool axes, lines shorter than the filter
(the window reaches across several lines), more than 256 float4 slots per token, the post-SSM
LayerNorm, exact ZOH and a pooling scale; an identity filter reproduces the layer without the
Conv1D; the host entry point carries the filter; the full-size 2048 px layer matches on sampled
images.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close, gpu_forward  # noqa: E402
from pooled_selective_scan_b200 import inputs  # noqa: E402

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def conv_layer(seed, B, h, w, E, N, R, dir_flags, dc, silu=False):
    rng = np.random.default_rng(seed)
    nd = oracle.nd_of(dir_flags)
    p = inputs.params(E, N, R, nd, seed)
    p["A_log"] = rng.uniform(-1.0, 1.5, size=p["A_log"].shape).astype(np.float32)
    p["D"] = rng.uniform(0.5, 1.5, size=p["D"].shape).astype(np.float32)
    p.update(inputs.conv_params(E, dc, nd, seed))
    p["x"] = rng.standard_normal((B, h, w, E), dtype=np.float32)
    p["z"] = rng.standard_normal((B, h, w, E), dtype=np.float32)
    p["conv_silu"] = silu
    return p


def ref_of(p, pool_axis, dir_flags, **kw):
    return oracle.forward_intermediates(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], pool_axis,
                                        dir_flags, conv_w=p["conv_w"], conv_b=p["conv_b"],
                                        conv_silu=p["conv_silu"], **kw)


def check(p, pool_axis, dir_flags, **kw):
    got = gpu_forward(p, pool_axis, dir_flags, **kw)
    assert got["status"] == 0
    assert got["launches"][0] == "pool_conv_kernel"
    okw = {k: v for k, v in kw.items() if k in ("pool_scale", "zoh_exact", "ln_eps")}
    if "ln_gamma" in p:
        okw.update(ln_gamma=p["ln_gamma"], ln_beta=p["ln_beta"])
    ref = ref_of(p, pool_axis, dir_flags, **okw)
    assert_close(got["xbar"], ref["xbar"], "xbar")
    for k in range(ref["u"].shape[0]):
        assert_close(got["u"][k], ref["u"][k], f"u[{k}]")
    assert_close(got["ys"], ref["ys"], "ys")
    assert_close(got["y"], ref["y"], "y")
    return got, ref


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("dir_flags", [1, 2, 3])
@pytest.mark.parametrize("dc,silu", [(1, False), (2, True), (3, False), (4, False), (4, True)])
def test_conv_small(pool_axis, dir_flags, dc, silu):
    p = conv_layer(2000 + 100 * dc + 10 * dir_flags + 2 * pool_axis + silu, B=3, h=7, w=5, E=36, N=16, R=4,
                   dir_flags=dir_flags, dc=dc, silu=silu)
    check(p, pool_axis, dir_flags)


@pytest.mark.parametrize("h,w,pool_axis", [(5, 1, 0), (1, 5, 1), (3, 2, 0), (2, 3, 1), (1, 1, 0), (6, 2, 1)])
def test_conv_lines_shorter_than_the_filter(h, w, pool_axis):
    p = conv_layer(2100 + 10 * h + w + pool_axis, B=2, h=h, w=w, E=20, N=8, R=3, dir_flags=3, dc=4, silu=True)
    check(p, pool_axis, 3)


@pytest.mark.parametrize("E,pool_axis", [(1040, 0), (1040, 1), (384, 0), (768, 1)])
def test_conv_wide_channels_and_workload_widths(E, pool_axis):
    p = conv_layer(2200 + E + pool_axis, B=2, h=12, w=10, E=E, N=16, R=12, dir_flags=3, dc=4)
    check(p, pool_axis, 3)


def test_conv_with_layernorm_exact_zoh_and_pool_scale():
    p = conv_layer(2300, B=2, h=9, w=6, E=72, N=16, R=5, dir_flags=3, dc=4, silu=True)
    rng = np.random.default_rng(2301)
    p["ln_gamma"] = rng.uniform(0.5, 1.5, 72).astype(np.float32)
    p["ln_beta"] = (0.2 * rng.standard_normal(72)).astype(np.float32)
    for pool_axis in (0, 1):
        check(p, pool_axis, 3, zoh_exact=True, pool_scale=0.25)


def test_identity_filter_is_the_layer_without_the_conv1d():
    p = conv_layer(2400, B=2, h=8, w=12, E=64, N=16, R=4, dir_flags=3, dc=4)
    p["conv_w"][:] = 0.0
    p["conv_w"][..., 3] = 1.0
    p["conv_b"][:] = 0.0
    for pool_axis in (0, 1):
        with_conv = gpu_forward(p, pool_axis, 3)
        plain = gpu_forward({k: v for k, v in p.items() if k not in ("conv_w", "conv_b", "conv_silu")}, pool_axis, 3,
                            path="staged")
        assert with_conv["status"] == 0 and plain["status"] == 0
        assert_close(with_conv["y"], plain["y"].astype(np.float64), "identity filter")


def test_conv_host_entry_point():
    """fastvim_ssm_forward_host copies the filter with the other parameters."""
    from pooled_selective_scan_b200 import ssm
    p = conv_layer(2500, B=3, h=10, w=8, E=48, N=16, R=4, dir_flags=3, dc=3, silu=True)
    host = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in p.items() if k != "conv_silu"}
    shape = ssm.infer_shape(host["x"], host["A_log"], host["W_dt"], 1, 3, d_conv=3, conv_silu=True)
    run = ssm.HostForward(shape, torch.device("cuda"))
    y = torch.empty(host["x"].shape, dtype=torch.float32).pin_memory()
    run(host, y)
    assert ssm.device_status(run.workspace) == 0
    ref = ref_of(p, 1, 3)
    assert_close(y.numpy(), ref["y"], "host entry y")


@pytest.mark.slow
def test_conv_full_size_2048px_layer():
    """The FastVim-T 2048 px layer (B = 128, 128 x 128 grid, E = 384) with a 4-tap filter per
    direction in front, in the launch configuration the benchmark times; three sampled images
    against the oracle."""
    from pooled_selective_scan_b200 import ssm, workload
    from pooled_selective_scan_b200.configs import by_name
    cfg = by_name("fastvim_t_2048")
    dev = torch.device("cuda")
    t = workload.layer_tensors(cfg, dev)
    t.update(workload.conv_tensors(cfg, dev, 4))
    y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], 0, cfg.dir_flags,
                    conv_w=t["conv_w"], conv_b=t["conv_b"], conv_silu=True)
    samples = [0, cfg.B // 2, cfg.B - 1]
    got = y[samples].cpu().numpy()
    del t, y
    torch.cuda.empty_cache()
    d = inputs.layer_inputs(cfg, which=samples)
    c = inputs.conv_params(cfg.E, 4, cfg.nd, cfg.seed)
    ref = oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], 0, cfg.dir_flags,
                         conv_w=c["conv_w"], conv_b=c["conv_b"], conv_silu=True, nthreads=3)
    assert_close(got, ref, "2048 px layer with the Conv1D")
