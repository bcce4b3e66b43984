"""The fused launch's task schedule, checked on the host (no GPU).

The launch hands out tickets in rounds: round r holds the projections of image r-1, the pooling of
image r, the gates of image r-L and the scans of image r-2.  A Python restatement of that
definition checks, for forced lags, that every task is handed out exactly once and that every
consumer comes after all its producers in ticket order: the property the kernel's deadlock-freedom
rests on.  The library's task count (its trace-record count) must cover every task once."""
import ctypes

import pytest

from pooled_selective_scan_b200 import _native as nat
from pooled_selective_scan_b200 import build as fvbuild

FAKE = 1 << 40


@pytest.fixture(scope="module")
def lib():
    fvbuild.build()
    return nat.lib()


def args(B, h, w, E, R=12, N=16, pool_axis=0):
    a = nat.FvSsmArgs()
    a.B, a.h, a.w, a.E, a.N, a.R = B, h, w, E, N, R
    a.pool_axis, a.dir_flags, a.K, a.pool_scale = pool_axis, 3, 0, 1.0
    a.flags = nat.FV_FLAG_PATH_FUSED | nat.FV_FLAG_TRACE
    for i, name in enumerate(("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt", "y")):
        setattr(a, name, FAKE + i * (1 << 34))
    return a


def schedule(B, nP, nQ, nS, L):
    def e(b):
        return b + L
    last = max(B + 1, e(B - 1)) if B else 1
    tickets = []
    for r in range(last + 1):
        if 0 <= r - 1 < B:
            tickets += [("Q", r - 1, i) for i in range(nQ)]
        if r < B:
            tickets += [("P", r, i) for i in range(nP)]
        for b in range(B):
            if e(b) == r:
                tickets += [("E", b, i) for i in range(nP)]
        if 0 <= r - 2 < B:
            tickets += [("S", r - 2, i) for i in range(nS)]
    return tickets


def check_order(tickets, B, nP, nQ, nS):
    assert len(set(tickets)) == len(tickets)
    assert len(tickets) == B * (2 * nP + nQ + nS)
    pos = {t: i for i, t in enumerate(tickets)}
    for b in range(B):
        last_p = max(pos[("P", b, i)] for i in range(nP))
        first_q = min(pos[("Q", b, i)] for i in range(nQ))
        last_q = max(pos[("Q", b, i)] for i in range(nQ))
        first_s = min(pos[("S", b, i)] for i in range(nS))
        last_s = max(pos[("S", b, i)] for i in range(nS))
        first_e = min(pos[("E", b, i)] for i in range(nP))
        assert last_p < first_q and last_q < first_s and last_s < first_e


@pytest.mark.parametrize("B,h,w,E", [(128, 128, 128, 384), (4, 128, 128, 384), (1, 64, 64, 768), (33, 96, 80, 256),
                                     (128, 64, 64, 768)])
@pytest.mark.parametrize("lag", [None, 3, 7, 64])
def test_schedule_hands_out_every_task_once_in_dependency_order(lib, monkeypatch, B, h, w, E, lag):
    if lag is not None:
        monkeypatch.setenv("FASTVIM_FUSED_LAG", str(lag))
    a = args(B, h, w, E)
    L = nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    # the schedule's task counts, restated: streaming tasks of >= 384 KB of x (up to 4 lines),
    # 16-token projection tasks, 128-channel scan tasks (both directions in one task)
    T, line = h, w * E * 4
    lp = 1
    while lp < 4 and lp < T and lp * line < 384 * 1024:
        lp += 1
    nP, nQ, nS = -(-T // lp), -(-T // 16), -(-E // 128)
    assert L.trace_records == B * (2 * nP + nQ + nS)  # the library hands out each task once
    if lag is not None:
        check_order(schedule(B, nP, nQ, nS, lag), B, nP, nQ, nS)
