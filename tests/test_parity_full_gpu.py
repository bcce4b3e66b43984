"""Full-size parity: every workload at its full batch, in the launch configuration the benchmark
times (one fastvim_ssm_forward call over the whole batch), compared with the fp64 oracle on
sampled images (first, middle, last), each against the tolerance element by element.  The
oracle recomputes a sampled image alone from its own seeded stream; nothing it reads comes from
the GPU."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close  # noqa: E402
from pooled_selective_scan_b200 import inputs, ssm, workload  # noqa: E402
from pooled_selective_scan_b200.configs import CONFIGS  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run_full(cfg, pool_axis, path="auto"):
    dev = torch.device("cuda")
    t = workload.layer_tensors(cfg, dev)
    keep = t.get("keep_idx")
    h, w = (cfg.h, cfg.w)
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, cfg.dir_flags, keep, h, w, path=path)
    ws = ssm.alloc_workspace(shape, dev)
    y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], pool_axis, cfg.dir_flags,
                    keep_idx=keep, h=h, w=w, workspace=ws, path=path)
    assert ssm.device_status(ws) == 0
    samples = sorted({0, cfg.B // 2, cfg.B - 1})
    got = y[samples].cpu().numpy()
    del t, y, ws
    torch.cuda.empty_cache()
    return samples, got


@pytest.mark.parametrize("ci,pool_axis,path", [(1, 0, "auto"), (1, 1, "auto"), (1, 0, "fused"), (2, 1, "auto"),
                                               (2, 1, "staged"), (3, 0, "auto"), (3, 0, "staged"), (4, 0, "auto")])
def test_full_size_config(ci, pool_axis, path):
    cfg = CONFIGS[ci]
    assert pool_axis in cfg.pool_axes
    samples, got = run_full(cfg, pool_axis, path)
    d = inputs.layer_inputs(cfg, which=samples)
    ref = oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], pool_axis,
                         cfg.dir_flags, keep_idx=d.get("keep_idx"), h=cfg.h, w=cfg.w, nthreads=len(samples))
    rep = assert_close(got, ref, f"{cfg.name} y")
    print(cfg.name, pool_axis, path, rep)
    assert np.isfinite(got).all()
