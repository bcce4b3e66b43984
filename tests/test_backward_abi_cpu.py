"""The gradient's C entry points on the host, without a GPU: workspace plan, launch list, and
every argument error returned before anything is queued (fake, never dereferenced addresses)."""
import ctypes
import os
import subprocess

import pytest

from pooled_selective_scan_b200 import _native as nat
from pooled_selective_scan_b200 import build as fvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fastvim_ssm.h")
FAKE = 1 << 40
SLOT = 1 << 34


@pytest.fixture(scope="module")
def lib():
    fvbuild.build()
    return nat.lib()


def args(**kw):
    a = nat.FvSsmArgs()
    a.B, a.h, a.w, a.E, a.N, a.R = 2, 14, 14, 384, 16, 12
    a.pool_axis, a.dir_flags, a.K, a.pool_scale, a.flags = 0, 3, 0, 1.0, 0
    for i, name in enumerate(("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt", "y")):
        setattr(a, name, FAKE + i * SLOT)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def grads(ln=False, **kw):
    g = nat.FvSsmGrads()
    for i, name in enumerate(("dy", "dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt")):
        setattr(g, name, FAKE + (12 + i) * SLOT)
    if ln:
        g.dln_gamma, g.dln_beta = FAKE + 30 * SLOT, FAKE + 31 * SLOT
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def test_struct_layouts_match_header(tmp_path):
    src = tmp_path / "off.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fastvim_ssm.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu\\n", sizeof(fv_ssm_grads), offsetof(fv_ssm_grads, db_dt), '
                   'sizeof(fv_bwd_ws_layout), offsetof(fv_bwd_ws_layout, partials)); return 0;}\n')
    exe = tmp_path / "off"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got == [ctypes.sizeof(nat.FvSsmGrads), nat.FvSsmGrads.db_dt.offset, ctypes.sizeof(nat.FvBwdWsLayout),
                   nat.FvBwdWsLayout.partials.offset]


@pytest.mark.parametrize("pool_axis,K,dirs", [(0, 0, 3), (1, 0, 1), (0, 37, 3), (1, 37, 2)])
def test_workspace_plan(lib, pool_axis, K, dirs):
    kw = dict(pool_axis=pool_axis, h=6, w=9, E=68, N=5, R=3, B=3, K=K, dir_flags=dirs)
    if K:
        kw["keep_idx"] = FAKE + 9 * SLOT
    a = args(**kw)
    L = nat.FvBwdWsLayout()
    assert lib.fastvim_ssm_backward_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    assert lib.fastvim_ssm_backward_workspace_size(ctypes.byref(a)) == L.total_bytes
    T = 6 if pool_axis == 0 else 9
    nd = bin(dirs).count("1")
    J = 3 + 2 * 5
    ub = -(-T * J // 32) * 32
    # dt_rank 3: the forward's scans compute their step sizes, so the gradient keeps its own Delta
    assert L.delta > 0
    regions = sorted([(L.status, 8), (L.dys, 3 * T * 68 * 4), (L.dxbar, 3 * T * 68 * 4), (L.du, nd * 3 * ub * 4),
                      (L.dxs, nd * 3 * T * 68 * 4),
                      (L.ckpt, 3 * nd * 2 * -(-T // 16) * 68 * 16 * 4), (L.delta, nd * 3 * T * 68 * 4)])
    end = 0
    for off, n in regions:
        assert off % 256 == 0 and off >= end
        end = off + n
    assert end <= L.partials < L.total_bytes  # then the partial sums of the fixed-order reductions


def test_launch_lists(lib):
    # dt_rank 12: the forward workspace holds no step sizes, so the gradient computes them first
    dense = [lib.fastvim_ssm_backward_launch_name(ctypes.byref(args()), i).decode() for i in range(8)]
    assert lib.fastvim_ssm_backward_launch_count(ctypes.byref(args())) == 8
    assert dense == ["bwd_gate_dense_kernel", "dt_proj_kernel", "bwd_scan_kernel", "bwd_reduce_kernel:du",
                     "bwd_dwx_kernel", "bwd_dxbar_kernel", "bwd_pool_dense_kernel",
                     "bwd_reduce_kernel:params"]
    m = args(K=49, keep_idx=FAKE + 9 * SLOT)
    masked = [lib.fastvim_ssm_backward_launch_name(ctypes.byref(m), i).decode() for i in range(8)]
    assert masked[0] == "bwd_gate_masked_kernel" and masked[-2] == "bwd_pool_masked_kernel"
    assert lib.fastvim_ssm_backward_launch_name(ctypes.byref(args()), 8) == b""
    assert lib.fastvim_ssm_backward_launch_count(ctypes.byref(args(B=0, x=None, z=None, y=None))) == 0
    ln = args(flags=nat.FV_FLAG_LAYERNORM, ln_gamma=FAKE + 10 * SLOT, ln_beta=FAKE + 11 * SLOT, ln_eps=1e-5)
    names = [lib.fastvim_ssm_backward_launch_name(ctypes.byref(ln), i).decode() for i in range(8)]
    assert lib.fastvim_ssm_backward_launch_count(ctypes.byref(ln)) == 8
    assert names[0] == "bwd_ln_gate_reg_kernel" and names[1:] == dense[1:]  # E = 384: tokens in registers
    wide = args(E=2560, flags=nat.FV_FLAG_LAYERNORM, ln_gamma=FAKE + 10 * SLOT, ln_beta=FAKE + 11 * SLOT, ln_eps=1e-5)
    assert lib.fastvim_ssm_backward_launch_name(ctypes.byref(wide), 0) == b"bwd_ln_gate_kernel"
    # dt_rank 48 on the staged path: the forward's step sizes are read, no dt_proj launch
    big = args(h=64, w=64, E=1536, R=48, K=1024, keep_idx=FAKE + 9 * SLOT)
    n = lib.fastvim_ssm_backward_launch_count(ctypes.byref(big))
    assert n == 7 and "dt_proj_kernel" not in [lib.fastvim_ssm_backward_launch_name(ctypes.byref(big), i).decode()
                                               for i in range(n)]
    L = nat.FvBwdWsLayout()
    assert lib.fastvim_ssm_backward_workspace_layout(ctypes.byref(big), ctypes.byref(L)) == nat.FV_OK
    assert L.delta == 0 and L.status == 0


def _bwd(lib, a, g, fwd=FAKE + 20 * SLOT, fwd_n=None, ws=FAKE + 22 * SLOT, ws_n=None):
    if fwd_n is None:
        fwd_n = lib.fastvim_ssm_workspace_size(ctypes.byref(a))
    if ws_n is None:
        ws_n = lib.fastvim_ssm_backward_workspace_size(ctypes.byref(a))
    return lib.fastvim_ssm_backward(ctypes.byref(a), g if g is None else ctypes.byref(g), ctypes.c_void_p(fwd), fwd_n,
                                    ctypes.c_void_p(ws), ws_n, None)


def test_rejections_before_any_launch(lib):
    a = args()
    # argument errors of the layer itself
    assert _bwd(lib, args(E=382), grads()) == nat.FV_ERR_SHAPE
    assert _bwd(lib, args(W_x=None), grads()) == nat.FV_ERR_NULL
    ln = args(flags=nat.FV_FLAG_LAYERNORM, ln_gamma=FAKE + 10 * SLOT, ln_beta=FAKE + 11 * SLOT, ln_eps=1e-5)
    assert _bwd(lib, ln, grads()) == nat.FV_ERR_NULL  # the LayerNorm's gradients are required
    assert _bwd(lib, ln, grads(ln=True, dln_beta=FAKE + 31 * SLOT + 4)) == nat.FV_ERR_ALIGN
    assert _bwd(lib, ln, grads(ln=True), ws=0) == nat.FV_ERR_WORKSPACE  # accepted up to the workspace check
    assert _bwd(lib, a, grads(ln=True)) == nat.FV_ERR_SHAPE  # LayerNorm gradients without the flag
    # gradient arrays
    assert _bwd(lib, a, None) == nat.FV_ERR_NULL
    for name in ("dy", "dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt"):
        assert _bwd(lib, a, grads(**{name: None})) == nat.FV_ERR_NULL, name
        assert _bwd(lib, a, grads(**{name: FAKE + 14 * SLOT + 4 if name == "dz" else getattr(grads(), name) + 8})) \
            == nat.FV_ERR_ALIGN, name
    assert _bwd(lib, a, grads(dx=a.x)) == nat.FV_ERR_ALIAS
    assert _bwd(lib, a, grads(dz=a.z + 4096)) == nat.FV_ERR_ALIAS
    assert _bwd(lib, a, grads(dx=grads().dy + 16)) == nat.FV_ERR_ALIAS
    assert _bwd(lib, a, grads(dz=grads().dx)) == nat.FV_ERR_ALIAS
    # workspaces
    assert _bwd(lib, a, grads(), fwd=0) == nat.FV_ERR_WORKSPACE
    assert _bwd(lib, a, grads(), fwd_n=lib.fastvim_ssm_workspace_size(ctypes.byref(a)) - 1) == nat.FV_ERR_WORKSPACE
    assert _bwd(lib, a, grads(), fwd=FAKE + 20 * SLOT + 16) == nat.FV_ERR_WORKSPACE
    assert _bwd(lib, a, grads(), ws=0) == nat.FV_ERR_WORKSPACE
    assert _bwd(lib, a, grads(), ws_n=lib.fastvim_ssm_backward_workspace_size(ctypes.byref(a)) - 1) \
        == nat.FV_ERR_WORKSPACE
    assert _bwd(lib, a, grads(), ws=FAKE + 20 * SLOT + 256) == nat.FV_ERR_WORKSPACE  # overlaps fwd_ws
    # y is not read: NULL is accepted up to the first check it does not take part in
    assert _bwd(lib, args(y=None), grads(), ws=0) == nat.FV_ERR_WORKSPACE
    # too few events
    ev = (ctypes.c_void_p * 4)()  # 5 launches need 10
    need_f = lib.fastvim_ssm_workspace_size(ctypes.byref(a))
    need_b = lib.fastvim_ssm_backward_workspace_size(ctypes.byref(a))
    assert lib.fastvim_ssm_backward_events(ctypes.byref(a), ctypes.byref(grads()), ctypes.c_void_p(FAKE + 20 * SLOT),
                                           need_f, ctypes.c_void_p(FAKE + 22 * SLOT), need_b, None, ev, 4) \
        == nat.FV_ERR_SHAPE
    assert lib.fastvim_ssm_backward_events(ctypes.byref(a), ctypes.byref(grads()), ctypes.c_void_p(FAKE + 20 * SLOT),
                                           need_f, ctypes.c_void_p(FAKE + 22 * SLOT), need_b, None, None, 14) \
        == nat.FV_ERR_NULL
