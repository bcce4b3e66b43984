"""The fused single-launch path: its per-task trace and its bounded waits (needs a B200).

The trace records one entry per task of the call; the schedule must hand out every task
exactly once and start each consumer only after its producers finished.  The bounded-wait
self-test makes a wait on a counter that nothing increments run out, and checks that the kernel
reports FV_ERR_TIMEOUT and leaves the context usable (a layer call right after still matches
the oracle)."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from fv_testlib import assert_close  # noqa: E402
from pooled_selective_scan_b200 import _native as nat  # noqa: E402
from pooled_selective_scan_b200 import inputs, ssm  # noqa: E402

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _layer(seed, B, h, w, E, R):
    d = inputs.params(E, 16, R, 2, seed)
    rng = np.random.default_rng(seed)
    d["x"] = rng.standard_normal((B, h, w, E), dtype=np.float32)
    d["z"] = rng.standard_normal((B, h, w, E), dtype=np.float32)
    return d


def test_trace_covers_every_task_once_in_dependency_order():
    d = _layer(7, B=6, h=48, w=40, E=192, R=8)
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(v).to(dev) for k, v in d.items()}
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], 0, 3, path="fused")
    a = shape.args(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], None, None)
    a.flags |= nat.FV_FLAG_TRACE
    L = nat.FvWsLayout()
    nat.check(nat.lib().fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)), "layout")
    assert L.trace_records > 0
    ws = torch.zeros(L.total_bytes, dtype=torch.uint8, device=dev)
    y = torch.empty_like(t["x"])
    a.y = ctypes.c_void_p(y.data_ptr())
    nat.check(nat.lib().fastvim_ssm_forward(ctypes.byref(a), ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(L.total_bytes),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)), "forward")
    assert ssm.device_status(ws) == 0
    rec = ws[L.trace:L.trace + 32 * L.trace_records].cpu().numpy().view(np.uint64).reshape(-1, 4)
    kind = (rec[:, 0] >> np.uint64(60)).astype(int)
    img = ((rec[:, 0] >> np.uint64(32)) & np.uint64(0xFFFFFFF)).astype(int)
    idx = (rec[:, 0] & np.uint64(0xFFFFFFFF)).astype(int)
    start = rec[:, 2].astype(np.int64)
    total = (rec[:, 3] & np.uint64((1 << 40) - 1)).astype(np.int64)
    wait = (rec[:, 3] >> np.uint64(40)).astype(np.int64)
    end = start + total
    keys = set(zip(kind.tolist(), img.tolist(), idx.tolist()))
    assert len(keys) == L.trace_records  # every ticket ran a distinct task
    assert set(kind.tolist()) == {0, 1, 2, 3}
    assert (wait >= 0).all() and (wait <= total).all()
    for b in range(6):
        pool_end = end[(kind == 0) & (img == b)].max()
        proj = (kind == 3) & (img == b)
        assert (start[proj] + wait[proj] >= pool_end).all()  # projections start after the pools end
        scan = (kind == 1) & (img == b)
        assert (start[scan] + wait[scan] >= end[proj].max()).all()
        gate = (kind == 2) & (img == b)
        assert (start[gate] + wait[gate] >= end[scan].max()).all()
    ref = oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], 0, 3)
    assert_close(y.cpu().numpy(), ref)


def test_bounded_wait_times_out_and_context_stays_usable():
    dev = torch.device("cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev)
    st = nat.lib().fastvim_selftest_bounded_wait(ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(4096), 20000,
                                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nat.FV_OK
    assert ssm.device_status(ws) == nat.FV_ERR_TIMEOUT
    # the device is still healthy: a layer call right after is correct
    d = _layer(8, B=2, h=16, w=16, E=64, R=4)
    t = {k: torch.from_numpy(v).to(dev) for k, v in d.items()}
    y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], 0, 3, path="fused")
    ref = oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], 0, 3)
    assert_close(y.cpu().numpy(), ref)


def test_bounded_wait_rejects_bad_arguments():
    lib = nat.lib()
    assert lib.fastvim_selftest_bounded_wait(None, 4096, 1000, None) == nat.FV_ERR_NULL
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert lib.fastvim_selftest_bounded_wait(ctypes.c_void_p(ws.data_ptr()), 512, 1000, None) == nat.FV_ERR_WORKSPACE
    assert lib.fastvim_selftest_bounded_wait(ctypes.c_void_p(ws.data_ptr()), 4096, 0, None) == nat.FV_ERR_SHAPE
