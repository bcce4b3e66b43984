"""The C ABI on the host, without a GPU: the library loads, exports exactly what the header
declares, and the host-side checks reject bad arguments before anything would be queued."""
import ctypes
import os
import re
import subprocess

import pytest

from pooled_selective_scan_b200 import _native as nat
from pooled_selective_scan_b200 import build as fvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fastvim_ssm.h")


@pytest.fixture(scope="module")
def lib():
    fvbuild.build()
    return nat.lib()


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FV_API\s+[\w\s\*]+?\b(fastvim_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for must in ("fastvim_ssm_forward", "fastvim_ssm_workspace_size", "fastvim_get_device_status",
                 "fastvim_status_string"):
        assert must in fns
    assert sorted(nat.EXPORTS) == fns


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", nat.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = sorted(set(re.findall(r"\sT\s(fastvim_\w+)$", out, re.M)))
    assert exported == header_functions()
    for name in header_functions():
        assert getattr(lib, name) is not None


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "fastvim_ssm.h"\nint main(void){fv_ssm_args a={0}; (void)a; '
                   'return (int)fastvim_ssm_workspace_size(&a);}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.dirname(HEADER), str(src),
                    "-o", str(tmp_path / "use.o")], check=True)


def test_struct_layout_matches_header(tmp_path):
    src = tmp_path / "off.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fastvim_ssm.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(fv_ssm_args), '
                   'offsetof(fv_ssm_args, pool_scale), offsetof(fv_ssm_args, x), offsetof(fv_ssm_args, y), '
                   'sizeof(fv_ws_layout), offsetof(fv_ssm_args, d_conv), offsetof(fv_ssm_args, conv_w), '
                   'offsetof(fv_ssm_args, conv_b)); return 0;}\n')
    exe = tmp_path / "off"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [ctypes.sizeof(nat.FvSsmArgs), nat.FvSsmArgs.pool_scale.offset, nat.FvSsmArgs.x.offset,
            nat.FvSsmArgs.y.offset, ctypes.sizeof(nat.FvWsLayout), nat.FvSsmArgs.d_conv.offset,
            nat.FvSsmArgs.conv_w.offset, nat.FvSsmArgs.conv_b.offset]
    assert got == want


def test_status_strings(lib):
    assert nat.status_string(0) == "FV_OK"
    for s in range(1, 10):
        assert nat.status_string(s).startswith("FV_ERR_")
    assert lib.fastvim_abi_version() == 6


# ---------------------------------------------------------------------------------------------
# Host validation with fake (never dereferenced) aligned addresses.
# ---------------------------------------------------------------------------------------------
FAKE = 1 << 40


def good_args(**kw):
    a = nat.FvSsmArgs()
    a.B, a.h, a.w, a.E, a.N, a.R = 2, 14, 14, 384, 16, 12
    a.pool_axis, a.dir_flags, a.K, a.pool_scale, a.flags = 0, 3, 0, 1.0, 0
    base = FAKE
    for i, name in enumerate(("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt", "y")):
        setattr(a, name, base + i * (1 << 32))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def validate(a):
    return nat.lib().fastvim_ssm_validate(ctypes.byref(a))


def test_valid_dense_and_masked(lib):
    assert validate(good_args()) == nat.FV_OK
    assert validate(good_args(K=49, keep_idx=FAKE + (9 << 32))) == nat.FV_OK
    assert validate(good_args(B=0, x=None, z=None, y=None)) == nat.FV_OK


@pytest.mark.parametrize("field,value,status", [
    ("E", 382, nat.FV_ERR_SHAPE), ("E", 0, nat.FV_ERR_SHAPE), ("B", -1, nat.FV_ERR_SHAPE),
    ("h", 0, nat.FV_ERR_SHAPE), ("N", 0, nat.FV_ERR_SHAPE), ("R", 0, nat.FV_ERR_SHAPE),
    ("N", 17, nat.FV_ERR_UNSUPPORTED), ("R", 70, nat.FV_ERR_UNSUPPORTED),
    ("pool_axis", 2, nat.FV_ERR_SHAPE), ("dir_flags", 0, nat.FV_ERR_SHAPE), ("dir_flags", 4, nat.FV_ERR_SHAPE),
    ("flags", 16, nat.FV_ERR_SHAPE), ("flags", 6, nat.FV_ERR_SHAPE), ("K", 14 * 14 + 1, nat.FV_ERR_SHAPE), ("K", -3, nat.FV_ERR_SHAPE),
    ("pool_scale", float("nan"), nat.FV_ERR_SHAPE),
    ("x", None, nat.FV_ERR_NULL), ("y", None, nat.FV_ERR_NULL), ("W_x", None, nat.FV_ERR_NULL),
    ("b_dt", None, nat.FV_ERR_NULL), ("x", FAKE + 4, nat.FV_ERR_ALIGN), ("D", FAKE + 8, nat.FV_ERR_ALIGN),
    ("keep_idx", FAKE + (9 << 32), nat.FV_ERR_SHAPE),  # a keep list without K
])
def test_bad_arguments_rejected(lib, field, value, status):
    assert validate(good_args(**{field: value})) == status


def test_masked_without_indices_rejected(lib):
    assert validate(good_args(K=10)) == nat.FV_ERR_NULL


def test_alias_rejected(lib):
    a = good_args()
    a.y = a.x + 1024 * 16
    assert validate(a) == nat.FV_ERR_ALIAS
    a = good_args()
    a.y = a.z
    assert validate(a) == nat.FV_ERR_ALIAS


def test_null_args_and_outputs(lib):
    assert lib.fastvim_ssm_validate(None) == nat.FV_ERR_NULL
    assert lib.fastvim_ssm_workspace_size(None) == 0
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(good_args()), None) == nat.FV_ERR_NULL
    assert lib.fastvim_get_device_status(None, None) == nat.FV_ERR_NULL


def test_forward_rejects_before_touching_the_gpu(lib):
    a = good_args(E=382)
    assert lib.fastvim_ssm_forward(ctypes.byref(a), None, 0, None) == nat.FV_ERR_SHAPE
    a = good_args()
    assert lib.fastvim_ssm_forward(ctypes.byref(a), None, 0, None) == nat.FV_ERR_WORKSPACE
    assert lib.fastvim_ssm_forward(ctypes.byref(a), ctypes.c_void_p(FAKE + 16), 1 << 30, None) == nat.FV_ERR_WORKSPACE
    need = lib.fastvim_ssm_workspace_size(ctypes.byref(a))
    assert lib.fastvim_ssm_forward(ctypes.byref(a), ctypes.c_void_p(FAKE), need - 1, None) == nat.FV_ERR_WORKSPACE


@pytest.mark.parametrize("pool_axis", [0, 1])
@pytest.mark.parametrize("K", [0, 37])
def test_workspace_layout(lib, pool_axis, K):
    kw = dict(pool_axis=pool_axis, h=6, w=9, E=64, N=16, R=4, B=3)
    if K:
        kw.update(K=K, keep_idx=FAKE + (9 << 32))
    a = good_args(**kw)
    L = nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    T = 6 if pool_axis == 0 else 9
    assert (L.T, L.S, L.nd) == (T, 15 - T, 2)
    ub = -(-T * 36 // 32) * 32
    regions = [(L.status, 4), (L.xbar, 3 * T * 64 * 4), (L.u, 2 * 3 * ub * 4), (L.ys, 3 * T * 64 * 4)]
    assert L.delta == 0  # dt_rank 4: the scans compute their step sizes themselves
    if K:
        regions += [(L.row_of, 3 * K * 4), (L.row_off, 3 * (T + 1) * 4), (L.row_tok, 3 * K * 4)]
    else:
        regions += [(L.ctrl, (64 + 3 * 3) * 4)]
    end = 0
    for off, size in regions:
        assert off % 256 == 0 and off >= end
        end = off + size
    assert L.total_bytes >= end
    assert lib.fastvim_ssm_workspace_size(ctypes.byref(a)) == L.total_bytes
    assert lib.fastvim_ssm_launch_count(ctypes.byref(a)) == (5 if K else 4)


@pytest.mark.parametrize("flags,want", [(0, ["fused_layer_kernel"]), (4, ["fused_layer_kernel"]),
                                        (2, ["pool_dense_kernel", "proj_gemm_kernel", "scan_seq_kernel",
                                             "epilogue_dense_kernel"])])
def test_path_selection_is_host_side(lib, flags, want):
    a = good_args(h=128, w=128, B=4, flags=flags)  # 2048 px FastVim-T images: fused by default
    n = lib.fastvim_ssm_launch_count(ctypes.byref(a))
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(n)]
    assert names == want
    small = good_args(flags=flags)  # 224 px: staged unless forced
    n = lib.fastvim_ssm_launch_count(ctypes.byref(small))
    assert n == (1 if flags == 4 else 4)


def test_forced_fused_path_refuses_masked_layers(lib):
    a = good_args(K=49, keep_idx=FAKE + (9 << 32), flags=4)
    assert lib.fastvim_ssm_launch_count(ctypes.byref(a)) == 0


def test_math_selftest_rejects_bad_arguments(lib):
    f = lib.fastvim_selftest_math
    assert f(3, ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + (1 << 32)), 8, None) == nat.FV_ERR_SHAPE
    assert f(0, ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + (1 << 32)), -1, None) == nat.FV_ERR_SHAPE
    assert f(0, None, ctypes.c_void_p(FAKE), 8, None) == nat.FV_ERR_NULL
    assert f(0, ctypes.c_void_p(FAKE + 4), ctypes.c_void_p(FAKE + (1 << 32)), 8, None) == nat.FV_ERR_ALIGN
    assert f(0, ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 16), 8, None) == nat.FV_ERR_ALIAS
    assert f(1, None, None, 0, None) == nat.FV_OK  # nothing to do


def test_layernorm_arguments(lib):
    LN = nat.FV_FLAG_LAYERNORM
    g, b = FAKE + (10 << 32), FAKE + (11 << 32)
    assert validate(good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5)) == nat.FV_OK
    assert validate(good_args(flags=LN, ln_gamma=g, ln_beta=None, ln_eps=1e-5)) == nat.FV_ERR_NULL
    assert validate(good_args(flags=LN, ln_gamma=None, ln_beta=None, ln_eps=1e-5)) == nat.FV_ERR_NULL
    assert validate(good_args(ln_gamma=g, ln_beta=b)) == nat.FV_ERR_SHAPE  # weights without the flag
    for eps in (0.0, -1e-5, float("nan"), float("inf")):
        assert validate(good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=eps)) == nat.FV_ERR_SHAPE
    assert validate(good_args(flags=LN, ln_gamma=g + 4, ln_beta=b, ln_eps=1e-5)) == nat.FV_ERR_ALIGN
    assert validate(good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5, E=4100)) == nat.FV_ERR_UNSUPPORTED
    assert lib.fastvim_abi_version() == 6


def test_layernorm_launches(lib):
    LN = nat.FV_FLAG_LAYERNORM
    g, b = FAKE + (10 << 32), FAKE + (11 << 32)
    small = good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5)
    n = lib.fastvim_ssm_launch_count(ctypes.byref(small))
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(small), i).decode() for i in range(n)]
    # rows of up to 1536 channels keep each lane's share of a token in registers, wider ones in shared memory
    assert names == ["pool_dense_kernel", "proj_gemm_kernel", "scan_seq_kernel", "ln_epilogue_reg_kernel"]
    masked = good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5, K=49, keep_idx=FAKE + (9 << 32))
    n = lib.fastvim_ssm_launch_count(ctypes.byref(masked))
    assert lib.fastvim_ssm_launch_name(ctypes.byref(masked), n - 1).decode() == "ln_epilogue_reg_kernel"
    wide = good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5, E=2048, R=12)
    n = lib.fastvim_ssm_launch_count(ctypes.byref(wide))
    assert lib.fastvim_ssm_launch_name(ctypes.byref(wide), n - 1).decode() == "ln_epilogue_kernel"
    conv = good_args(flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5, d_conv=4, conv_w=FAKE + (12 << 32),
                     conv_b=FAKE + (13 << 32))
    n = lib.fastvim_ssm_launch_count(ctypes.byref(conv))
    assert lib.fastvim_ssm_launch_name(ctypes.byref(conv), n - 1).decode() == "ln_epilogue_kernel"
    # large images: the staged kernels by default (their register epilogue is the faster one); the
    # forced single launch does the LayerNorm in its gate tasks
    big = good_args(h=128, w=128, B=4, flags=LN, ln_gamma=g, ln_beta=b, ln_eps=1e-5)
    assert lib.fastvim_ssm_launch_count(ctypes.byref(big)) == 4
    big.flags = LN | nat.FV_FLAG_PATH_FUSED
    assert lib.fastvim_ssm_launch_count(ctypes.byref(big)) == 1


@pytest.mark.parametrize("masked,ln", [(False, False), (False, True), (True, False), (True, True)])
def test_staged_launch_order(lib, masked, ln):
    kw = dict(B=5, flags=2)
    if masked:
        kw.update(K=49, keep_idx=FAKE + (9 << 32))
    if ln:
        kw.update(flags=2 | nat.FV_FLAG_LAYERNORM, ln_gamma=FAKE + (10 << 32), ln_beta=FAKE + (11 << 32), ln_eps=1e-5)
    a = good_args(**kw)
    front = ["mask_bucket_kernel", "mask_pool_kernel"] if masked else ["pool_dense_kernel"]
    middle = ["proj_gemm_kernel", "scan_seq_kernel"]
    back = ["ln_epilogue_reg_kernel" if ln else ("mask_epilogue_kernel" if masked else "epilogue_dense_kernel")]
    want = front + middle + back
    n = lib.fastvim_ssm_launch_count(ctypes.byref(a))
    assert [lib.fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(n)] == want


@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("R", [31, 32, 48])
def test_delta_kernel_from_dt_rank_32(lib, masked, R):
    """With dt_rank >= 32 the staged path computes the step sizes in their own (tensor-core) GEMM
    launch between x_proj and the scans and keeps them in the workspace; below, the scans compute
    them."""
    kw = dict(B=3, h=6, w=9, E=64, R=R, flags=2)
    if masked:
        kw.update(K=37, keep_idx=FAKE + (9 << 32))
    a = good_args(**kw)
    n = lib.fastvim_ssm_launch_count(ctypes.byref(a))
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(n)]
    front = ["mask_bucket_kernel", "mask_pool_kernel"] if masked else ["pool_dense_kernel"]
    mid = ["proj_gemm_kernel"] + (["dt_proj_kernel"] if R >= 32 else []) + ["scan_seq_kernel"]
    assert names == front + mid + ["mask_epilogue_kernel" if masked else "epilogue_dense_kernel"]
    L = nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    if R >= 32:  # [nd][B][T][E] fp32 after ys, inside the workspace
        assert L.delta % 256 == 0 and L.delta >= L.ys + 3 * 6 * 64 * 4
        assert L.total_bytes >= L.delta + 2 * 3 * 6 * 64 * 4
    else:
        assert L.delta == 0


@pytest.mark.parametrize("K", [0, 37])
@pytest.mark.parametrize("flags", [2, 4])
def test_kept_scan_states_layout(lib, K, flags):
    """FV_FLAG_KEEP_STATES adds the scan states every 8 steps to the forward workspace
    ([B][nd][2 ceil(T/16)][E][16] fp32, on either path) and drops the gradient's own copy; the
    launches stay the same."""
    if K and flags == 4:
        flags = 0  # masked layers run staged
    kw = dict(B=3, h=20, w=9, E=64, R=4, flags=flags)
    if K:
        kw.update(K=K, keep_idx=FAKE + (9 << 32))
    a, ak = good_args(**kw), good_args(**dict(kw, flags=flags | nat.FV_FLAG_KEEP_STATES))
    L, Lk = nat.FvWsLayout(), nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)) == nat.FV_OK
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(ak), ctypes.byref(Lk)) == nat.FV_OK
    T = 20
    size = 3 * 2 * (2 * 2) * 64 * 16 * 4
    assert L.ckpt == 0 and Lk.ckpt % 256 == 0 and Lk.ckpt >= Lk.ys + 3 * T * 64 * 4
    assert Lk.total_bytes >= Lk.ckpt + size and Lk.total_bytes - L.total_bytes >= size
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(a), i) for i in range(lib.fastvim_ssm_launch_count(ctypes.byref(a)))]
    assert names == [lib.fastvim_ssm_launch_name(ctypes.byref(ak), i)
                     for i in range(lib.fastvim_ssm_launch_count(ctypes.byref(ak)))]
    B, Bk = nat.FvBwdWsLayout(), nat.FvBwdWsLayout()
    assert lib.fastvim_ssm_backward_workspace_layout(ctypes.byref(a), ctypes.byref(B)) == nat.FV_OK
    assert lib.fastvim_ssm_backward_workspace_layout(ctypes.byref(ak), ctypes.byref(Bk)) == nat.FV_OK
    assert B.ckpt > 0 and Bk.ckpt == 0 and B.total_bytes - Bk.total_bytes >= size
    assert lib.fastvim_ssm_validate(ctypes.byref(good_args(**dict(kw, flags=flags | 128)))) == nat.FV_ERR_SHAPE


# ---------------------------------------------------------------------------------------------
# The block's Conv1D in front of the layer (d_conv, conv_w, conv_b, FV_FLAG_CONV_SILU).
# ---------------------------------------------------------------------------------------------
CW, CB = FAKE + (12 << 32), FAKE + (13 << 32)


def test_conv_arguments(lib):
    assert validate(good_args(d_conv=4, conv_w=CW, conv_b=CB)) == nat.FV_OK
    assert validate(good_args(d_conv=1, conv_w=CW, conv_b=CB, flags=nat.FV_FLAG_CONV_SILU)) == nat.FV_OK
    assert validate(good_args(d_conv=4, conv_w=None, conv_b=CB)) == nat.FV_ERR_NULL
    assert validate(good_args(d_conv=4, conv_w=CW, conv_b=None)) == nat.FV_ERR_NULL
    assert validate(good_args(conv_w=CW, conv_b=CB)) == nat.FV_ERR_SHAPE          # weights without taps
    assert validate(good_args(flags=nat.FV_FLAG_CONV_SILU)) == nat.FV_ERR_SHAPE   # SiLU of no Conv1D
    assert validate(good_args(d_conv=-1)) == nat.FV_ERR_SHAPE
    assert validate(good_args(d_conv=5, conv_w=CW, conv_b=CB)) == nat.FV_ERR_UNSUPPORTED
    assert validate(good_args(d_conv=4, conv_w=CW + 4, conv_b=CB)) == nat.FV_ERR_ALIGN
    masked = good_args(d_conv=4, conv_w=CW, conv_b=CB, K=49, keep_idx=FAKE + (9 << 32))
    assert validate(masked) == nat.FV_ERR_UNSUPPORTED


def test_conv_launches_and_workspace(lib):
    a = good_args(d_conv=4, conv_w=CW, conv_b=CB)
    n = lib.fastvim_ssm_launch_count(ctypes.byref(a))
    names = [lib.fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(n)]
    assert names == ["pool_conv_kernel", "proj_gemm_kernel", "scan_seq_kernel", "epilogue_conv_kernel"]
    ln = good_args(d_conv=4, conv_w=CW, conv_b=CB, flags=nat.FV_FLAG_LAYERNORM, ln_gamma=FAKE + (10 << 32),
                   ln_beta=FAKE + (11 << 32), ln_eps=1e-5)
    assert lib.fastvim_ssm_launch_name(ctypes.byref(ln), 3).decode() == "ln_epilogue_kernel"  # neighbours: rows
    # large images take the staged kernels with the Conv1D; forcing the single launch is refused
    big = good_args(h=128, w=128, d_conv=4, conv_w=CW, conv_b=CB)
    assert lib.fastvim_ssm_launch_name(ctypes.byref(big), 0).decode() == "pool_conv_kernel"
    assert lib.fastvim_ssm_launch_count(ctypes.byref(good_args(h=128, w=128, d_conv=4, conv_w=CW, conv_b=CB,
                                                                flags=nat.FV_FLAG_PATH_FUSED))) == 0
    # each direction pools its own convolved tokens: two sets of pooled tokens
    L0, L1 = nat.FvWsLayout(), nat.FvWsLayout()
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(good_args()), ctypes.byref(L0)) == nat.FV_OK
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L1)) == nat.FV_OK
    assert L1.u - L1.xbar == 2 * (L0.u - L0.xbar)
    one = good_args(dir_flags=2, d_conv=2, conv_w=CW, conv_b=CB)
    assert lib.fastvim_ssm_workspace_layout(ctypes.byref(one), ctypes.byref(L1)) == nat.FV_OK
    assert L1.u - L1.xbar == L0.u - L0.xbar


def test_conv_gradient_not_built(lib):
    a = good_args(d_conv=4, conv_w=CW, conv_b=CB)
    g = nat.FvSsmGrads()
    for i, name in enumerate(("dy", "dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt")):
        setattr(g, name, FAKE + ((20 + i) << 32))
    st = lib.fastvim_ssm_backward(ctypes.byref(a), ctypes.byref(g), ctypes.c_void_p(FAKE + (40 << 32)),
                                  ctypes.c_size_t(1 << 30), ctypes.c_void_p(FAKE + (41 << 32)), ctypes.c_size_t(1 << 30),
                                  None)
    assert st == nat.FV_ERR_UNSUPPORTED


def test_binding_constants_and_every_struct_field_match_the_header(tmp_path):
    """Every status, flag and struct field offset of the ctypes binding equals what a C compiler
    makes of include/fastvim_ssm.h (the binding only marshals; a drifted offset would pass
    arguments to the wrong fields)."""
    consts = [n for n in dir(nat) if n.startswith(("FV_OK", "FV_ERR_", "FV_FLAG_"))]
    structs = {"fv_ssm_args": nat.FvSsmArgs, "fv_ws_layout": nat.FvWsLayout, "fv_ssm_grads": nat.FvSsmGrads,
               "fv_bwd_ws_layout": nat.FvBwdWsLayout}
    lines = [f'printf("%lld\\n", (long long){n});' for n in consts]
    for cname, cls in structs.items():
        lines.append(f'printf("%zu\\n", sizeof({cname}));')
        lines += [f'printf("%zu\\n", offsetof({cname}, {f[0]}));' for f in cls._fields_]
    src = tmp_path / "abi.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fastvim_ssm.h"\nint main(void){\n'
                   + "\n".join(lines) + "\nreturn 0;}\n")
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)],
                   check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [getattr(nat, n) for n in consts]
    for cls in structs.values():
        want.append(ctypes.sizeof(cls))
        want += [getattr(cls, f[0]).offset for f in cls._fields_]
    assert got == want
