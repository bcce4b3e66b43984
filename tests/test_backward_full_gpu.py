"""Full-size parity of the gradient in the launch configuration the benchmark's gradient leg
times (one forward call over the batch, then one gradient call on its workspace): the 2048 px
FastVim-T layer (B = 128, 128 x 128 grid, E = 384) and the masked FastMaskVim-B layer (B = 64,
1,024 of 4,096 tokens kept, E = 1536).  The parameter gradients, sums over the whole batch, are
compared in full with the oracle's sum (computed image by image from each image's seeded
stream); dx and dz on sampled images (first, middle, last)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import GRAD_PARAM_ABS_RMS, assert_close  # noqa: E402
from pooled_selective_scan_b200 import inputs, ssm, workload  # noqa: E402
from pooled_selective_scan_b200.configs import CONFIGS  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PARAMS = ("A_log", "D", "W_x", "W_dt", "b_dt")


@pytest.mark.parametrize("ci", [3, 4])
def test_full_size_gradient(ci):
    """ci 3: the 2048 px FastVim-T layer (fused forward); ci 4: the 75 %-masked FastMaskVim-B layer
    (E = 1536, staged forward)."""
    cfg = CONFIGS[ci]
    axis = cfg.pool_axes[0]
    dev = torch.device("cuda")
    t = workload.layer_tensors(cfg, dev)
    dy = workload.upstream_grad(cfg, dev)
    keep = t.get("keep_idx")
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], axis, cfg.dir_flags, keep, cfg.h, cfg.w)
    fws = ssm.alloc_workspace(shape, dev)
    ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], axis, cfg.dir_flags, keep_idx=keep,
                h=cfg.h, w=cfg.w, workspace=fws)
    assert ssm.device_status(fws) == 0
    g = ssm.backward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], dy, fws, axis, cfg.dir_flags,
                     keep_idx=keep, h=cfg.h, w=cfg.w)
    torch.cuda.synchronize()
    samples = [0, cfg.B // 2, cfg.B - 1]
    got = {k: g[k][samples].cpu().numpy() for k in ("dx", "dz")}
    got.update({"d" + n: g["d" + n].cpu().numpy() for n in PARAMS})
    del t, dy, g, fws
    torch.cuda.empty_cache()

    p = inputs.params(cfg.E, cfg.N, cfg.R, cfg.nd, cfg.seed)
    shp = inputs.token_shape(cfg)
    sums = {"d" + n: np.zeros(p[n].shape) for n in PARAMS}
    ref = {"dx": [], "dz": []}
    chunk = 16
    for b0 in range(0, cfg.B, chunk):
        ids = range(b0, min(cfg.B, b0 + chunk))
        x = np.stack([inputs.image_x(cfg.seed, b, shp) for b in ids])
        z = np.stack([inputs.image_z(cfg.seed, b, shp) for b in ids])
        dyi = np.stack([inputs.image_dy(cfg.seed, b, shp) for b in ids])
        kw = {}
        if cfg.masked:
            kw = dict(keep_idx=np.stack([inputs.image_keep_idx(cfg.seed, b, cfg.h, cfg.w, cfg.K) for b in ids]),
                      h=cfg.h, w=cfg.w)
        r = oracle.backward(x, z, p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], dyi, axis, cfg.dir_flags,
                            nthreads=chunk, **kw)
        for n in PARAMS:
            sums["d" + n] += r["d" + n]
        for b in ids:
            if b in samples:
                ref["dx"].append(r["dx"][b - b0])
                ref["dz"].append(r["dz"][b - b0])
    reps = {}
    for k in ("dx", "dz"):
        reps[k] = assert_close(got[k], np.stack(ref[k]), f"{cfg.name} {k}")
    for n in PARAMS:
        reps["d" + n] = assert_close(got["d" + n], sums["d" + n], f"{cfg.name} d{n}", GRAD_PARAM_ABS_RMS)
    print(cfg.name, {k: (round(v["max_abs_over_rms"], 9), round(v["max_err_over_bound"], 4)) for k, v in reps.items()})
