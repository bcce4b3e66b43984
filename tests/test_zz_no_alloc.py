"""fastvim_ssm_forward_noalloc: the allocation-free entry point, for callers that are handed
their input and output buffers by a host framework and have no way to allocate device memory
(or must not, since cudaMalloc/cudaFree can stall the device).  It runs the same layer with its
scratch in a fixed 16 MiB static device array instead of a caller workspace.

Checked through the C ABI: three calls in a row (different layers, so each later call runs on
the scratch the one before left behind: the staged kernels on a dense layer, then on a masked
layer, then the single persistent launch, whose control block must be reset by the call itself)
each match fastvim_ssm_forward with a caller workspace and the fp64 oracle, within the layer's
tolerance; a layer whose scratch would exceed 16 MiB is refused with FV_ERR_UNSUPPORTED and
queues nothing.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close  # noqa: E402
from pooled_selective_scan_b200 import _native as nat  # noqa: E402
from pooled_selective_scan_b200 import inputs, ssm  # noqa: E402
from pooled_selective_scan_b200.configs import CONFIGS  # noqa: E402

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

STATIC_SCRATCH_BYTES = 16 << 20


def _layer(seed, B, h, w, E, R, K=0):
    d = inputs.params(E, 16, R, 2, seed)
    rng = np.random.default_rng(seed)
    shp = (B, K, E) if K else (B, h, w, E)
    d["x"] = rng.standard_normal(shp, dtype=np.float32)
    d["z"] = rng.standard_normal(shp, dtype=np.float32)
    if K:
        d["keep_idx"] = np.stack([rng.permutation(h * w)[:K] for _ in range(B)]).astype(np.int32)
    dev = torch.device("cuda")
    return {k: torch.from_numpy(v).to(dev) for k, v in d.items()}


def _both_entry_points(t, pool_axis, h, w, path="auto"):
    keep = t.get("keep_idx")
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, 3, keep, h, w, path=path)
    assert ssm.workspace_size(shape) <= STATIC_SCRATCH_BYTES
    y_ref = torch.full_like(t["x"], float("nan"))
    y_new = torch.full_like(t["x"], float("nan"))
    ws = ssm.alloc_workspace(shape)
    lib = nat.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    a_ref = shape.args(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], keep, y_ref)
    a_new = shape.args(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], keep, y_new)
    nat.check(lib.fastvim_ssm_forward(ctypes.byref(a_ref), ctypes.c_void_p(ws.data_ptr()),
                                      ctypes.c_size_t(ws.numel()), stream), "fastvim_ssm_forward")
    nat.check(lib.fastvim_ssm_forward_noalloc(ctypes.byref(a_new), stream), "fastvim_ssm_forward_noalloc")
    torch.cuda.synchronize()
    assert ssm.device_status(ws) == 0
    return y_new.cpu().numpy(), y_ref.cpu().numpy(), ssm.launch_names(shape)


def _oracle(t, pool_axis, h, w, images):
    """The fp64 oracle on the given images of the layer (inputs copied back from the device)."""
    g = {k: v.cpu().numpy() for k, v in t.items()}
    keep = g.get("keep_idx")
    return oracle.forward(g["x"][images], g["z"][images], g["A_log"], g["D"], g["W_x"], g["W_dt"], g["b_dt"],
                          pool_axis, 3, keep_idx=None if keep is None else keep[images], h=h, w=w,
                          nthreads=len(images))


def test_noalloc_matches_workspace_entry_point_and_oracle_three_times_in_a_row():
    cfg = CONFIGS[1]  # FastVim-T layer, 224 px, batch 128 (about 6 MiB of scratch)
    first = _layer(1, B=cfg.B, h=cfg.h, w=cfg.w, E=cfg.E, R=cfg.R)
    second = _layer(2, B=8, h=12, w=10, E=96, R=6, K=70)  # a masked layer of another shape
    third = _layer(5, B=3, h=40, w=36, E=136, R=6)  # dense, forced onto the single persistent launch
    y_new, y_ref, names = _both_entry_points(first, 1, cfg.h, cfg.w)
    assert names[0] == "pool_dense_kernel"
    assert np.isfinite(y_new).all()
    assert_close(y_new, y_ref, "first call")
    sample = [0, cfg.B // 2, cfg.B - 1]
    assert_close(y_new[sample], _oracle(first, 1, cfg.h, cfg.w, sample), "first call vs oracle")
    y_new, y_ref, names = _both_entry_points(second, 0, 12, 10)
    assert names[0] == "mask_bucket_kernel"
    assert np.isfinite(y_new).all()
    assert_close(y_new, y_ref, "second call")
    assert_close(y_new, _oracle(second, 0, 12, 10, list(range(8))), "second call vs oracle")
    y_new, y_ref, names = _both_entry_points(third, 0, 40, 36, path="fused")
    assert names == ["fused_layer_kernel"]
    assert np.isfinite(y_new).all()
    assert_close(y_new, y_ref, "third call")
    assert_close(y_new, _oracle(third, 0, 40, 36, [0, 1, 2]), "third call vs oracle")


def test_noalloc_refuses_layers_beyond_the_static_scratch():
    t = _layer(3, B=1, h=2, w=2, E=16, R=2)
    shape = ssm.LayerShape(B=128, h=128, w=128, E=384, N=16, R=12, pool_axis=0, dir_flags=3)
    assert ssm.workspace_size(shape) > STATIC_SCRATCH_BYTES
    # fake, never-dereferenced addresses: the size check comes before anything is queued
    a = shape.args()
    fake = 1 << 40
    for i, name in enumerate(("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt", "y")):
        setattr(a, name, fake + (i << 36))
    st = nat.lib().fastvim_ssm_forward_noalloc(ctypes.byref(a), None)
    assert st == nat.FV_ERR_UNSUPPORTED
    assert "static scratch" in nat.last_error()
    torch.cuda.synchronize()
    del t
