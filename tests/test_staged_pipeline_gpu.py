"""The staged kernels as a pipeline of image chunks over two streams (FASTVIM_STAGED_CHUNKS > 1:
projections and scans of a chunk on the library's side stream, between the chunk's pooling and
its epilogue on the caller's stream): results equal the single-chunk run bit for bit and the oracle within
tolerance, for ragged chunk sizes, dense and masked layers, with and without the LayerNorm, the
intermediates included; and timing events bracket every launch."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close, gpu_forward  # noqa: E402
from test_parity_gpu import rand_layer  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("chunks", [2, 3, 5])
@pytest.mark.parametrize("masked,ln", [(False, False), (True, False), (False, True), (True, True)])
def test_chunked_equals_single_chunk_and_oracle(monkeypatch, chunks, masked, ln):
    kw = dict(B=5, h=6, w=9, E=64, N=16, R=6, dir_flags=3)
    if masked:
        kw["K"] = 23
    p = rand_layer(400 + chunks + 10 * masked + 20 * ln, **kw)
    if ln:
        rng = np.random.default_rng(7)
        p["ln_gamma"] = rng.uniform(0.5, 1.5, 64).astype(np.float32)
        p["ln_beta"] = (0.2 * rng.standard_normal(64)).astype(np.float32)
    hw = dict(h=6, w=9) if masked else {}
    monkeypatch.setenv("FASTVIM_STAGED_CHUNKS", "1")
    one = gpu_forward(p, 1, 3, path="staged", **hw)
    monkeypatch.setenv("FASTVIM_STAGED_CHUNKS", str(chunks))
    many = gpu_forward(p, 1, 3, path="staged", **hw)
    assert one["status"] == 0 and many["status"] == 0
    assert len(many["launches"]) == chunks * len(one["launches"])
    for key in ("y", "xbar", "u", "ys"):
        assert np.array_equal(one[key], many[key]), key
    ref = oracle.forward_intermediates(p["x"], p["z"], p["A_log"], p["D"], p["W_x"], p["W_dt"], p["b_dt"], 1, 3,
                                       keep_idx=p.get("keep_idx"), ln_gamma=p.get("ln_gamma"),
                                       ln_beta=p.get("ln_beta"), **hw)
    assert_close(many["y"], ref["y"])
    assert_close(many["u"], ref["u"], "u")


def test_events_bracket_every_launch(monkeypatch):
    from pooled_selective_scan_b200 import ssm, workload
    from pooled_selective_scan_b200.configs import by_name
    monkeypatch.setenv("FASTVIM_STAGED_CHUNKS", "3")
    cfg = by_name("fastvim_t_224")
    dev = torch.device("cuda")
    t = workload.layer_tensors(cfg, dev)
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 0, 3, path="staged")
    y = torch.empty_like(t["x"])
    ws = ssm.alloc_workspace(shape, dev)
    fwd = ssm.BoundForward(shape, t, y, ws)
    n = fwd.n_launch
    assert n == 12
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
    fwd.run_events(evs)
    torch.cuda.synchronize()
    assert ssm.device_status(ws) == 0
    d = [evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(n)]
    assert all(v > 0 for v in d)
    ref = oracle.forward(*(t[k][:4].cpu().numpy() if k in ("x", "z") else t[k].cpu().numpy()
                           for k in ("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt")), 0, 3)
    assert_close(y[:4].cpu().numpy(), ref)
