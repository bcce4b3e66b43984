"""Host-side fuzzing of the C ABI (no GPU; no pointer is ever dereferenced).

Arguments are drawn as a layer the ABI accepts, then, in about half the draws, one field is
broken in a way whose status the header fixes.  For accepted layers the workspace size equals the
layout's total, every region is 256-byte aligned, disjoint from the others and large enough for
what it holds, and the launch list matches the path the flags and the shape choose."""
import ctypes

import pytest

pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

from pooled_selective_scan_b200 import _native as nat  # noqa: E402
from pooled_selective_scan_b200 import build as fvbuild  # noqa: E402
from pooled_selective_scan_b200.ssm import POOL_H, POOL_W  # noqa: E402

FAKE = 1 << 40          # fake device addresses, 16-byte aligned, never dereferenced
SLOT = 1 << 50          # far apart: no two tensors alias at any drawn size
MAX_N, MAX_J, MAX_T = 16, 96, 4096
CTRL_WORDS = lambda B: 64 + 3 * B  # noqa: E731  header + 3 counters per image (fused control block)
PTRS = ("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt", "y")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fvbuild.build()


@st.composite
def valid_layer(draw):
    a = nat.FvSsmArgs()
    a.B = draw(st.integers(0, 300))
    a.h = draw(st.integers(1, 300))
    a.w = draw(st.integers(1, 300))
    a.E = draw(st.sampled_from([4, 8, 12, 64, 192, 384, 768, 1536, 4096]))
    a.N = draw(st.integers(1, MAX_N))
    a.R = draw(st.integers(1, MAX_J - 2 * a.N))
    a.pool_axis = draw(st.sampled_from([POOL_W, POOL_H]))
    a.dir_flags = draw(st.sampled_from([1, 2, 3]))
    a.K = draw(st.integers(1, a.h * a.w)) if draw(st.booleans()) else 0
    a.pool_scale = draw(st.sampled_from([0.0, 1.0, 0.25]))
    a.flags = (draw(st.sampled_from([0, nat.FV_FLAG_PATH_STAGED, nat.FV_FLAG_PATH_FUSED]))
               | draw(st.sampled_from([0, nat.FV_FLAG_ZOH_EXACT]))
               | draw(st.sampled_from([0, nat.FV_FLAG_TRACE]))
               | draw(st.sampled_from([0, nat.FV_FLAG_LAYERNORM]))
               | draw(st.sampled_from([0, nat.FV_FLAG_KEEP_STATES])))
    for i, name in enumerate(PTRS):
        setattr(a, name, FAKE + i * SLOT)
    if a.K:
        a.keep_idx = FAKE + 9 * SLOT
    if a.flags & nat.FV_FLAG_LAYERNORM:
        a.ln_gamma, a.ln_beta, a.ln_eps = FAKE + 10 * SLOT, FAKE + 11 * SLOT, 1e-5
    return a


def _set(field, value):
    return lambda a: setattr(a, field, value(a) if callable(value) else value)


# (name, applies to, change, status the header gives)
BREAKS = [
    ("E not a multiple of 4", lambda a: True, _set("E", lambda a: a.E + 2), nat.FV_ERR_SHAPE),
    ("no direction", lambda a: True, _set("dir_flags", 0), nat.FV_ERR_SHAPE),
    ("unknown direction bit", lambda a: True, _set("dir_flags", lambda a: a.dir_flags | 4), nat.FV_ERR_SHAPE),
    ("unknown pool axis", lambda a: True, _set("pool_axis", 2), nat.FV_ERR_SHAPE),
    ("both paths forced", lambda a: True,
     _set("flags", lambda a: a.flags | nat.FV_FLAG_PATH_STAGED | nat.FV_FLAG_PATH_FUSED), nat.FV_ERR_SHAPE),
    ("unknown flag", lambda a: True, _set("flags", lambda a: a.flags | 32), nat.FV_ERR_SHAPE),
    ("undefined flag bit", lambda a: True, _set("flags", lambda a: a.flags | 128), nat.FV_ERR_SHAPE),
    ("negative batch", lambda a: True, _set("B", -1), nat.FV_ERR_SHAPE),
    ("K above the grid", lambda a: True, _set("K", lambda a: a.h * a.w + 1), nat.FV_ERR_SHAPE),
    ("NaN pool scale", lambda a: True, _set("pool_scale", float("nan")), nat.FV_ERR_SHAPE),
    ("d_state above the limit", lambda a: True, _set("N", MAX_N + 1), nat.FV_ERR_UNSUPPORTED),
    ("R + 2N above the limit", lambda a: True, _set("R", lambda a: MAX_J - 2 * a.N + 1), nat.FV_ERR_UNSUPPORTED),
    ("no A_log", lambda a: True, _set("A_log", None), nat.FV_ERR_NULL),
    ("no x", lambda a: a.B > 0, _set("x", None), nat.FV_ERR_NULL),
    ("no keep list", lambda a: a.K > 0 and a.B > 0, _set("keep_idx", None), nat.FV_ERR_NULL),
    ("keep list without K", lambda a: a.K == 0, _set("keep_idx", FAKE + 9 * SLOT), nat.FV_ERR_SHAPE),
    ("LayerNorm without gamma", lambda a: a.flags & nat.FV_FLAG_LAYERNORM, _set("ln_gamma", None), nat.FV_ERR_NULL),
    ("LayerNorm eps 0", lambda a: a.flags & nat.FV_FLAG_LAYERNORM, _set("ln_eps", 0.0), nat.FV_ERR_SHAPE),
    ("gamma without the flag", lambda a: not a.flags & nat.FV_FLAG_LAYERNORM,
     _set("ln_gamma", FAKE + 10 * SLOT), nat.FV_ERR_SHAPE),
    ("misaligned z", lambda a: True, _set("z", FAKE + 1 * SLOT + 4), nat.FV_ERR_ALIGN),
    ("misaligned W_x", lambda a: True, _set("W_x", FAKE + 4 * SLOT + 8), nat.FV_ERR_ALIGN),
    ("y aliases x", lambda a: a.B > 0, _set("y", FAKE), nat.FV_ERR_ALIAS),
    ("y overlaps z", lambda a: a.B > 0, _set("y", FAKE + SLOT + 16), nat.FV_ERR_ALIAS),
]


def _check_layout(lib, a):
    size = lib.fastvim_ssm_workspace_size(ctypes.byref(a))
    L = nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    assert size == L.total_bytes
    B, E = a.B, a.E
    T = a.h if a.pool_axis == POOL_W else a.w
    assert (L.T, L.S, L.nd) == (T, a.w + a.h - T, bin(a.dir_flags).count("1"))
    ub = -(-T * (a.R + 2 * a.N) // 32) * 32
    regions = [(L.status, 8), (L.xbar, B * T * E * 4), (L.u, B * L.nd * ub * 4), (L.ys, B * T * E * 4)]
    if a.K:
        assert L.ctrl == 0 and L.trace == 0
        regions += [(L.row_of, B * a.K * 4), (L.row_off, B * (T + 1) * 4), (L.row_tok, B * a.K * 4)]
    else:
        assert L.row_of == L.row_off == L.row_tok == 0
        regions.append((L.ctrl, CTRL_WORDS(B) * 4))
        if L.trace:
            assert a.flags & nat.FV_FLAG_TRACE and L.trace_records > 0
            regions.append((L.trace, L.trace_records * 32))
    if L.delta:  # the staged path's step sizes (dt_rank >= 32)
        assert a.R >= 32
        regions.append((L.delta, L.nd * B * T * E * 4))
    # the scan states kept for the gradient: exactly with FV_FLAG_KEEP_STATES
    assert (L.ckpt != 0) == bool(a.flags & nat.FV_FLAG_KEEP_STATES)
    if L.ckpt:
        regions.append((L.ckpt, B * L.nd * 2 * -(-T // 16) * E * 16 * 4))
    regions.sort()
    end = 0
    for off, n in regions:
        assert off % 256 == 0 and off >= end, (off, end)
        end = off + n
    assert end <= L.total_bytes < end + 256 * len(regions)


def _check_launches(lib, a):
    n = lib.fastvim_ssm_launch_count(ctypes.byref(a))
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(n)]
    assert lib.fastvim_ssm_launch_name(ctypes.byref(a), n).decode() == ""
    if a.B == 0:
        assert n == 0
        return
    if n == 0:
        # only a forced fused path on a layer it cannot run (masked, or token rows wider than half
        # a 24 KB ring stage) has no launches: the forward call refuses it with FV_ERR_UNSUPPORTED
        assert a.flags & nat.FV_FLAG_PATH_FUSED
        assert a.K > 0 or a.E * 4 > 12 * 1024
        return
    if names == ["fused_layer_kernel"]:
        assert a.K == 0 and not a.flags & nat.FV_FLAG_PATH_STAGED
        return
    assert not a.flags & nat.FV_FLAG_PATH_FUSED
    assert "fused_layer_kernel" not in names
    # pooling (masked: bucketing, pooling), x_proj, (dt_proj from dt_rank 32), scans, epilogue
    full = (5 if a.K else 4) + (1 if a.R >= 32 else 0)
    if a.flags & nat.FV_FLAG_LAYERNORM:  # registers up to 1536 channels, shared-memory rows above
        assert n == full and names[-1] == ("ln_epilogue_reg_kernel" if a.E <= 1536 else "ln_epilogue_kernel")
    else:
        assert n == full and names[-1] == ("mask_epilogue_kernel" if a.K else "epilogue_dense_kernel")
    assert "proj_gemm_kernel" in names and any(k.startswith("scan") for k in names)
    assert ("dt_proj_kernel" in names) == (a.R >= 32)
    if a.K:
        assert names[0].startswith("mask_")


@settings(max_examples=600, deadline=None)
@given(valid_layer(), st.integers(-len(BREAKS), len(BREAKS) - 1))
def test_validation_layout_and_launch_list(a, pick):
    lib = nat.lib()
    base = lib.fastvim_ssm_validate(ctypes.byref(a))
    T = a.h if a.pool_axis == POOL_W else a.w
    limited = T > MAX_T or (a.K and a.h * a.w > (1 << 20))
    assert base == (nat.FV_ERR_UNSUPPORTED if limited else nat.FV_OK)
    if base != nat.FV_OK:
        assert lib.fastvim_ssm_workspace_size(ctypes.byref(a)) == 0
        return
    if pick < 0:  # keep the layer as drawn
        _check_layout(lib, a)
        _check_launches(lib, a)
        return
    name, applies, change, want = BREAKS[pick]
    if not applies(a):
        return
    change(a)
    assert lib.fastvim_ssm_validate(ctypes.byref(a)) == want, name
    if want in (nat.FV_ERR_SHAPE, nat.FV_ERR_UNSUPPORTED) and name not in (
            "keep list without K", "gamma without the flag"):
        # shape errors: no workspace, no launches
        assert lib.fastvim_ssm_workspace_size(ctypes.byref(a)) == 0
        assert lib.fastvim_ssm_launch_count(ctypes.byref(a)) == 0


GRAD_NAMES = ("dy", "dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt")


def _grads_for(a):
    g = nat.FvSsmGrads()
    for i, name in enumerate(GRAD_NAMES):
        setattr(g, name, FAKE + (12 + i) * SLOT)
    if a.flags & nat.FV_FLAG_LAYERNORM:
        g.dln_gamma, g.dln_beta = FAKE + 20 * SLOT, FAKE + 21 * SLOT
    return g


GRAD_BREAKS = [
    ("no grads block", lambda a, g: True, None, nat.FV_ERR_NULL),
    ("no dA_log", lambda a, g: True, ("dA_log", None), nat.FV_ERR_NULL),
    ("no dx", lambda a, g: a.B > 0, ("dx", None), nat.FV_ERR_NULL),
    ("no dy", lambda a, g: a.B > 0, ("dy", None), nat.FV_ERR_NULL),
    ("misaligned dW_x", lambda a, g: True, ("dW_x", FAKE + 17 * SLOT + 4), nat.FV_ERR_ALIGN),
    ("dx aliases x", lambda a, g: a.B > 0, ("dx", FAKE), nat.FV_ERR_ALIAS),
    ("dz aliases dy", lambda a, g: a.B > 0, ("dz", FAKE + 12 * SLOT), nat.FV_ERR_ALIAS),
    ("LayerNorm gradient missing", lambda a, g: a.flags & nat.FV_FLAG_LAYERNORM, ("dln_beta", None),
     nat.FV_ERR_NULL),
    ("LayerNorm gradient without the flag", lambda a, g: not a.flags & nat.FV_FLAG_LAYERNORM,
     ("dln_gamma", FAKE + 20 * SLOT), nat.FV_ERR_SHAPE),
]


@settings(max_examples=300, deadline=None)
@given(valid_layer(), st.integers(-len(GRAD_BREAKS), len(GRAD_BREAKS) - 1))
def test_gradient_validation_and_plan(a, pick):
    lib = nat.lib()
    if lib.fastvim_ssm_validate(ctypes.byref(a)) != nat.FV_OK:
        return
    L = nat.FvBwdWsLayout()
    assert lib.fastvim_ssm_backward_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    assert lib.fastvim_ssm_backward_workspace_size(ctypes.byref(a)) == L.total_bytes
    T = a.h if a.pool_axis == POOL_W else a.w
    nd = bin(a.dir_flags).count("1")
    ub = -(-T * (a.R + 2 * a.N) // 32) * 32
    bte = a.B * T * a.E * 4
    regions = [(L.status, 8), (L.dys, bte), (L.dxbar, bte), (L.du, nd * a.B * ub * 4), (L.dxs, nd * bte)]
    # the scan states live in exactly one of the workspaces: the forward's with FV_FLAG_KEEP_STATES
    assert (L.ckpt == 0) == bool(a.flags & nat.FV_FLAG_KEEP_STATES)
    if L.ckpt:
        regions.append((L.ckpt, a.B * nd * 2 * -(-T // 16) * a.E * 16 * 4))
    FL = nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(FL)) == nat.FV_OK
    assert (L.delta == 0) == (FL.delta != 0)  # the step sizes live in exactly one of the workspaces
    if L.delta:
        regions.append((L.delta, nd * bte))
    regions = sorted(regions)
    end = 0
    for off, n in regions:
        assert off % 256 == 0 and off >= end
        end = off + n
    assert end <= L.partials < L.total_bytes  # then the partial sums of the fixed-order reductions
    n = lib.fastvim_ssm_backward_launch_count(ctypes.byref(a))
    names = [lib.fastvim_ssm_backward_launch_name(ctypes.byref(a), i).decode() for i in range(n)]
    if a.B == 0:
        assert n == 0
    else:
        first = (("bwd_ln_gate_reg_kernel" if a.E <= 2048 else "bwd_ln_gate_kernel") if a.flags & nat.FV_FLAG_LAYERNORM else
                 "bwd_gate_masked_kernel" if a.K else "bwd_gate_dense_kernel")
        mid = ["bwd_scan_kernel"] if FL.delta else ["dt_proj_kernel", "bwd_scan_kernel"]
        assert names[0] == first and names[1:1 + len(mid)] == mid and len(names) == 6 + len(mid)
        assert names[-1] == "bwd_reduce_kernel:params"
    g = _grads_for(a)
    fws = lib.fastvim_ssm_workspace_size(ctypes.byref(a))

    def call(gp):
        # a NULL gradient workspace: every argument check runs, nothing is queued
        return lib.fastvim_ssm_backward(ctypes.byref(a), gp, ctypes.c_void_p(FAKE + 40 * SLOT), fws, None, 0, None)

    if pick < 0:
        assert call(ctypes.byref(g)) == nat.FV_ERR_WORKSPACE
        return
    name, applies, change, want = GRAD_BREAKS[pick]
    if not applies(a, g):
        return
    if change is None:
        assert call(None) == want, name
        return
    setattr(g, change[0], change[1])
    assert call(ctypes.byref(g)) == want, name
