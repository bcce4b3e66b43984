"""Parity of the post-SSM LayerNorm variant (FV_FLAG_LAYERNORM) with the fp64 oracle: the
staged LayerNorm epilogues (a token's share per lane in registers up to 1536 channels, shared-memory
rows above; dense and masked) and the fused launch's gate tasks, over ragged channel counts
(every register-slot count: 1-4, 6, 8, 12 float4 slots per lane), both pool axes, one and two directions, a large epsilon, rejected keep ids and
the host entry point."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close, gpu_forward  # noqa: E402
from test_parity_gpu import rand_layer  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def with_ln(p, seed, E):
    rng = np.random.default_rng(seed)
    q = dict(p)
    q["ln_gamma"] = rng.uniform(0.5, 1.5, E).astype(np.float32)
    q["ln_beta"] = (0.3 * rng.standard_normal(E)).astype(np.float32)
    return q


def ref_of(q, pool_axis, dir_flags, h=None, w=None, eps=1e-5):
    return oracle.forward(q["x"], q["z"], q["A_log"], q["D"], q["W_x"], q["W_dt"], q["b_dt"], pool_axis, dir_flags,
                          keep_idx=q.get("keep_idx"), h=h, w=w, ln_gamma=q["ln_gamma"], ln_beta=q["ln_beta"],
                          ln_eps=eps)


@pytest.mark.parametrize("E,pool_axis,dir_flags", [(52, 0, 3), (52, 1, 3), (384, 0, 3), (388, 1, 1), (704, 1, 3), (772, 0, 3),
                                                   (1024, 1, 3), (1536, 0, 3), (1540, 0, 2), (4096, 1, 3)])
@pytest.mark.parametrize("path", ["staged", "fused"])
def test_layernorm_dense(E, pool_axis, dir_flags, path):
    if path == "fused" and E > 2048:
        pytest.skip("the fused launch takes E <= 2048")
    p = with_ln(rand_layer(300 + E + pool_axis, B=2, h=5, w=7, E=E, N=16, R=6, dir_flags=dir_flags), 1 + E, E)
    got = gpu_forward(p, pool_axis, dir_flags, intermediates=False, path=path)
    assert got["status"] == 0
    staged = "ln_epilogue_reg_kernel" if E <= 1536 else "ln_epilogue_kernel"  # registers / shared-memory rows
    assert got["launches"][-1] == ("fused_layer_kernel" if path == "fused" else staged)
    assert_close(got["y"], ref_of(p, pool_axis, dir_flags))


@pytest.mark.parametrize("path", ["auto", "fused"])
def test_layernorm_large_eps_at_2048px(path):
    # 2048 px FastVim-T images (the LayerNorm layer takes the staged kernels by default, and the
    # single launch when forced), eps large enough to matter
    p = with_ln(rand_layer(320, B=2, h=128, w=128, E=384, N=16, R=12, dir_flags=3), 7, 384)
    got = gpu_forward(p, 0, 3, intermediates=False, ln_eps=0.25, path=path)
    assert got["launches"][-1] == ("fused_layer_kernel" if path == "fused" else "ln_epilogue_reg_kernel")
    assert_close(got["y"], ref_of(p, 0, 3, eps=0.25))


@pytest.mark.parametrize("pool_axis", [0, 1])
def test_layernorm_masked(pool_axis):
    p = with_ln(rand_layer(330 + pool_axis, B=3, h=8, w=6, E=200, N=16, R=8, dir_flags=3, K=29), 9, 200)
    got = gpu_forward(p, pool_axis, 3, h=8, w=6, intermediates=False)
    assert got["status"] == 0
    assert_close(got["y"], ref_of(p, pool_axis, 3, h=8, w=6))


def test_layernorm_masked_rejected_id_gives_zero():
    p = with_ln(rand_layer(340, B=2, h=4, w=4, E=16, N=16, R=2, dir_flags=3, K=6), 11, 16)
    p["keep_idx"][0, 2] = 99  # out of range
    got = gpu_forward(p, 0, 3, h=4, w=4, intermediates=False)
    assert got["status"] == 4  # FV_ERR_INDEX
    assert np.all(got["y"][0, 2] == 0.0)
    ref = oracle.forward(p["x"][1:], p["z"][1:], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 0, 3,
                         keep_idx=p["keep_idx"][1:], h=4, w=4, ln_gamma=p["ln_gamma"], ln_beta=p["ln_beta"])
    assert_close(got["y"][1:], ref)


def test_layernorm_host_entry_point():
    from pooled_selective_scan_b200 import ssm
    p = with_ln(rand_layer(350, B=3, h=6, w=10, E=96, N=16, R=4, dir_flags=3), 13, 96)
    t = {k: torch.from_numpy(v).pin_memory() for k, v in p.items()}
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 1, 3, ln=True, ln_eps=1e-5)
    run = ssm.HostForward(shape)
    y_host = torch.empty(t["x"].shape, dtype=torch.float32).pin_memory()
    run(t, y_host)
    assert_close(y_host.numpy(), ref_of(p, 1, 3))
