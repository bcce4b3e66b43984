"""fp64 CPU oracle of the FastVim SSM layer (pooled selective scan).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline / reference leg may import this module.  It wraps the plain C library
built from ``fastvim_oracle.c`` (fp64, nested loops, no GPU code, no code shared with the CUDA
library); see that file for the method passages each step follows and the readings taken where
the method description is silent.

Every function takes numpy arrays in the layouts of ``fastvim_oracle.h`` and returns fp64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fastvim_oracle.c")
_GRAD_SRC = os.path.join(_HERE, "fastvim_oracle_grad.c")
_HDR = os.path.join(_HERE, "fastvim_oracle.h")
_LIB_PATH = os.path.join(_HERE, "libfastvim_oracle.so")

FVO_OK, FVO_BAD_SHAPE, FVO_BAD_INDEX, FVO_NO_MEMORY = 0, 2, 4, 8
POOL_W, POOL_H = 0, 1
FWD, BWD = 1, 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``libfastvim_oracle.so`` (gcc, -O2, OpenMP over images)."""
    srcs = [_SRC, _GRAD_SRC]
    newest_src = max(os.path.getmtime(p) for p in srcs + [_HDR])
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest_src:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, *srcs, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            U = ctypes.c_uint
            Dbl = ctypes.c_double
            sigs = {
                "fvo_pool": [P, I, I, I, I, I, Dbl, P],
                "fvo_mask_rows": [P, I, I, I, I, I, P, P, P],
                "fvo_pool_masked": [P, P, P, I, I, I, I, I, Dbl, P],
                "fvo_proj": [P, I, I, I, I, I, I, P, P, P, P, P],
                "fvo_scan": [P, P, P, P, I, I, I, I, I, I, U, I, P],
                "fvo_scan_states": [P, P, P, P, I, I, I, I, I, I, U, I, P],
                "fvo_gate_dense": [P, P, P, P, I, I, I, I, I, I, P, P, Dbl, P],
                "fvo_gate_masked": [P, P, P, P, P, I, I, I, I, I, P, P, Dbl, P],
                "fvo_forward": [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, U, Dbl, I, P, P, Dbl, I, P],
                "fvo_backward": [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, U, Dbl, I, P, P, Dbl, P, I,
                                 P, P, P, P, P, P, P, P, P],
                "fvo_conv": [P, I, I, I, I, I, U, I, P, P, I, P],
                "fvo_pool_d": [P, I, I, I, I, I, Dbl, P],
                "fvo_gate_dense_conv": [P, P, P, P, I, I, I, I, I, I, P, P, Dbl, P],
                "fvo_forward_conv": [P, P, P, P, P, P, P, I, I, I, I, I, I, I, U, Dbl, I, I, P, P, I, P, P, Dbl, I,
                                     P],
            }
            for name, argtypes in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = argtypes
                fn.restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"oracle {where} returned status {status}")
        self.status = status


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(st, where, allow=()):
    if st != FVO_OK and st not in allow:
        raise OracleError(st, where)
    return st


def nd_of(dir_flags: int) -> int:
    return int(bool(dir_flags & FWD)) + int(bool(dir_flags & BWD))


def pooled_len(h: int, w: int, pool_axis: int) -> int:
    return h if pool_axis == POOL_W else w


def pooled_over(h: int, w: int, pool_axis: int) -> int:
    return w if pool_axis == POOL_W else h


def pool(x, pool_axis, pool_scale=1.0):
    """Dense mean pooling: x [B,h,w,E] -> xbar [B,T,E]."""
    x = _f32(x)
    B, h, w, E = x.shape
    out = np.empty((B, pooled_len(h, w, pool_axis), E), np.float64)
    _check(_load().fvo_pool(_p(x), B, h, w, E, pool_axis, float(pool_scale), _p(out)), "pool")
    return out


def mask_rows(keep_idx, h, w, pool_axis):
    """Row bucketing of kept-token ids -> (status, row_of [B,K], row_off [B,T+1], row_tok [B,K])."""
    idx = _i32(keep_idx)
    B, K = idx.shape
    T = pooled_len(h, w, pool_axis)
    row_of = np.empty((B, K), np.int32)
    row_off = np.empty((B, T + 1), np.int32)
    row_tok = np.empty((B, K), np.int32)
    st = _load().fvo_mask_rows(_p(idx), B, K, h, w, pool_axis, _p(row_of), _p(row_off), _p(row_tok))
    _check(st, "mask_rows", allow=(FVO_BAD_INDEX,))
    return st, row_of, row_off, row_tok


def pool_masked(x, row_off, row_tok, S, pool_scale=1.0):
    """Masked mean pooling: x [B,K,E] + row CSR -> xbar [B,T,E] (divisor S, fixed)."""
    x = _f32(x)
    B, K, E = x.shape
    row_off = _i32(row_off)
    row_tok = _i32(row_tok)
    T = row_off.shape[1] - 1
    out = np.empty((B, T, E), np.float64)
    st = _load().fvo_pool_masked(_p(x), _p(row_off), _p(row_tok), B, K, T, S, E, float(pool_scale), _p(out))
    _check(st, "pool_masked")
    return out


def proj(xbar, W_x, W_dt, b_dt, R, N):
    """x_proj + dt_proj + softplus: xbar [B,T,E] -> u [nd,B,T,R+2N], delta [nd,B,T,E]."""
    xbar = _f64(xbar)
    W_x, W_dt, b_dt = _f32(W_x), _f32(W_dt), _f32(b_dt)
    B, T, E = xbar.shape
    nd = W_x.shape[0]
    u = np.empty((nd, B, T, R + 2 * N), np.float64)
    delta = np.empty((nd, B, T, E), np.float64)
    st = _load().fvo_proj(_p(xbar), B, T, E, nd, R, N, _p(W_x), _p(W_dt), _p(b_dt), _p(u), _p(delta))
    _check(st, "proj")
    return u, delta


def scan(xbar, delta, u, A_log, R, N, dir_flags, zoh_exact=False):
    """ZOH + forward/backward selective scans, directions summed -> ys [B,T,E]."""
    xbar, delta, u = _f64(xbar), _f64(delta), _f64(u)
    A_log = _f32(A_log)
    B, T, E = xbar.shape
    nd = nd_of(dir_flags)
    ys = np.empty((B, T, E), np.float64)
    st = _load().fvo_scan(_p(xbar), _p(delta), _p(u), _p(A_log), B, T, E, nd, R, N,
                          int(dir_flags), int(bool(zoh_exact)), _p(ys))
    _check(st, "scan")
    return ys


def scan_states(xbar, delta, u, A_log, R, N, dir_flags, zoh_exact=False):
    """The scans' states [nd,B,T,E,N]: [k,b,s] = the state of direction slot k entering its s-th
    step in scan order (zero at s = 0)."""
    xbar, delta, u = _f64(xbar), _f64(delta), _f64(u)
    A_log = _f32(A_log)
    B, T, E = xbar.shape
    nd = nd_of(dir_flags)
    hin = np.empty((nd, B, T, E, N), np.float64)
    st = _load().fvo_scan_states(_p(xbar), _p(delta), _p(u), _p(A_log), B, T, E, nd, R, N,
                                 int(dir_flags), int(bool(zoh_exact)), _p(hin))
    _check(st, "scan_states")
    return hin


def _ln(ln_gamma, ln_beta, E):
    """LayerNorm gamma and beta as fp32 [E] arrays (None stays None: the C side checks that both
    or neither are given)."""
    out = []
    for v in (ln_gamma, ln_beta):
        a = None if v is None else _f32(v)
        assert a is None or a.shape == (E,)
        out.append(a)
    return out


def gate_dense(x, z, ys, D, pool_axis, ln_gamma=None, ln_beta=None, ln_eps=1e-5):
    """Repeat + D x skip (+ post-SSM LayerNorm) + SiLU(z) gate on the dense grid -> y [B,h,w,E]."""
    x, z, D = _f32(x), _f32(z), _f32(D)
    ys = _f64(ys)
    B, h, w, E = x.shape
    g, b = _ln(ln_gamma, ln_beta, E)
    y = np.empty(x.shape, np.float64)
    st = _load().fvo_gate_dense(_p(x), _p(z), _p(ys), _p(D), B, h, w, E, D.shape[0], pool_axis, _p(g), _p(b),
                                float(ln_eps), _p(y))
    _check(st, "gate_dense")
    return y


def gate_masked(x, z, ys, D, row_of, ln_gamma=None, ln_beta=None, ln_eps=1e-5):
    """Repeat to kept tokens + skip (+ post-SSM LayerNorm) + gate -> y [B,K,E]."""
    x, z, D = _f32(x), _f32(z), _f32(D)
    ys = _f64(ys)
    row_of = _i32(row_of)
    B, K, E = x.shape
    T = ys.shape[1]
    g, b = _ln(ln_gamma, ln_beta, E)
    y = np.empty(x.shape, np.float64)
    st = _load().fvo_gate_masked(_p(x), _p(z), _p(ys), _p(D), _p(row_of), B, K, T, E, D.shape[0], _p(g), _p(b),
                                 float(ln_eps), _p(y))
    _check(st, "gate_masked")
    return y


def conv(x, conv_w, conv_b, pool_axis, dir_flags, conv_silu=False):
    """The block's Conv1D, one filter per direction slot: x [B,h,w,E], conv_w [nd,E,dc],
    conv_b [nd,E] -> xc [nd,B,h,w,E] (fp64)."""
    x, conv_w, conv_b = _f32(x), _f32(conv_w), _f32(conv_b)
    B, h, w, E = x.shape
    nd, E2, dc = conv_w.shape
    assert E2 == E and conv_b.shape == (nd, E) and nd == nd_of(dir_flags)
    xc = np.empty((nd, B, h, w, E), np.float64)
    st = _load().fvo_conv(_p(x), B, h, w, E, pool_axis, int(dir_flags), dc, _p(conv_w), _p(conv_b),
                          int(bool(conv_silu)), _p(xc))
    _check(st, "conv")
    return xc


def pool_d(x, pool_axis, pool_scale=1.0):
    """Mean pooling of an fp64 grid x [B,h,w,E] -> xbar [B,T,E]."""
    x = _f64(x)
    B, h, w, E = x.shape
    out = np.empty((B, pooled_len(h, w, pool_axis), E), np.float64)
    _check(_load().fvo_pool_d(_p(x), B, h, w, E, pool_axis, float(pool_scale), _p(out)), "pool_d")
    return out


def gate_dense_conv(xc, z, ys, D, pool_axis, ln_gamma=None, ln_beta=None, ln_eps=1e-5):
    """Repeat + skip with each direction's convolved input (+ LayerNorm) + gate -> y [B,h,w,E]."""
    xc, ys = _f64(xc), _f64(ys)
    z, D = _f32(z), _f32(D)
    nd, B, h, w, E = xc.shape
    g, b = _ln(ln_gamma, ln_beta, E)
    y = np.empty(z.shape, np.float64)
    st = _load().fvo_gate_dense_conv(_p(xc), _p(z), _p(ys), _p(D), B, h, w, E, nd, pool_axis, _p(g), _p(b),
                                     float(ln_eps), _p(y))
    _check(st, "gate_dense_conv")
    return y


def forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, dir_flags, keep_idx=None, h=None,
            w=None, pool_scale=1.0, zoh_exact=False, nthreads=1, allow_bad_index=False, ln_gamma=None,
            ln_beta=None, ln_eps=1e-5, conv_w=None, conv_b=None, conv_silu=False):
    """The whole layer, image by image.

    Dense: x, z [B,h,w,E] -> y [B,h,w,E].  Masked: x, z [B,K,E], keep_idx [B,K] with the grid
    given by h, w -> y [B,K,E].  Returns fp64 y (and the status when allow_bad_index is set).
    With conv_w [nd,E,dc] and conv_b [nd,E] (dense only) x is the input of the block's Conv1D.
    """
    x, z = _f32(x), _f32(z)
    A_log, D, W_x, W_dt, b_dt = map(_f32, (A_log, D, W_x, W_dt, b_dt))
    N = A_log.shape[2]
    E = A_log.shape[1]
    R = W_dt.shape[2]
    if conv_w is not None or conv_b is not None:
        assert keep_idx is None and conv_w is not None and conv_b is not None
        cw, cb = _f32(conv_w), _f32(conv_b)
        B, h, w, E2 = x.shape
        assert E2 == E and z.shape == x.shape and cw.shape[:2] == (nd_of(dir_flags), E)
        g, b = _ln(ln_gamma, ln_beta, E)
        y = np.empty(x.shape, np.float64)
        st = _load().fvo_forward_conv(_p(x), _p(z), _p(A_log), _p(D), _p(W_x), _p(W_dt), _p(b_dt), B, h, w, E, N, R,
                                      pool_axis, int(dir_flags), float(pool_scale), int(bool(zoh_exact)),
                                      cw.shape[2], _p(cw), _p(cb), int(bool(conv_silu)), _p(g), _p(b), float(ln_eps),
                                      int(nthreads), _p(y))
        _check(st, "forward_conv")
        return (y, st) if allow_bad_index else y
    if keep_idx is None:
        B, h, w, E2 = x.shape
        K = 0
        idx = None
    else:
        B, K, E2 = x.shape
        idx = _i32(keep_idx)
        assert h is not None and w is not None and idx.shape == (B, K)
    assert E2 == E and z.shape == x.shape
    g, b = _ln(ln_gamma, ln_beta, E)
    y = np.empty(x.shape, np.float64)
    st = _load().fvo_forward(_p(x), _p(z), _p(A_log), _p(D), _p(W_x), _p(W_dt), _p(b_dt), _p(idx),
                             B, h, w, E, N, R, K, pool_axis, int(dir_flags), float(pool_scale),
                             int(bool(zoh_exact)), _p(g), _p(b), float(ln_eps), int(nthreads), _p(y))
    _check(st, "forward", allow=(FVO_BAD_INDEX,) if allow_bad_index else ())
    return (y, st) if allow_bad_index else y


def forward_intermediates(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis, dir_flags, keep_idx=None,
                          h=None, w=None, pool_scale=1.0, zoh_exact=False, ln_gamma=None, ln_beta=None,
                          ln_eps=1e-5, conv_w=None, conv_b=None, conv_silu=False):
    """The same chain step by step, returning every intermediate as a dict (small sizes only).
    With the Conv1D (conv_w, conv_b) the per-direction intermediates are stacked: xc [nd,B,h,w,E],
    xbar [B,nd,T,E] (each direction pools its own convolved tokens), u [nd,B,T,J], delta
    [nd,B,T,E]."""
    A_log, W_dt = _f32(A_log), _f32(W_dt)
    N = A_log.shape[2]
    R = W_dt.shape[2]
    out = {}
    if conv_w is not None:
        assert keep_idx is None
        W_x, b_dt = _f32(W_x), _f32(b_dt)
        xc = conv(x, conv_w, conv_b, pool_axis, dir_flags, conv_silu)
        dirs = [d for d in (FWD, BWD) if dir_flags & d]
        xbars, us, deltas = [], [], []
        ys = 0.0
        for k, d in enumerate(dirs):
            xb = pool_d(xc[k], pool_axis, pool_scale)
            u, delta = proj(xb, W_x[k:k + 1], W_dt[k:k + 1], b_dt[k:k + 1], R, N)
            ys = ys + scan(xb, delta, u, A_log[k:k + 1], R, N, d, zoh_exact)
            xbars.append(xb)
            us.append(u[0])
            deltas.append(delta[0])
        y = gate_dense_conv(xc, z, ys, D, pool_axis, ln_gamma, ln_beta, ln_eps)
        out.update(xc=xc, xbar=np.stack(xbars, axis=1), u=np.stack(us), delta=np.stack(deltas), ys=ys, y=y)
        return out
    if keep_idx is None:
        xbar = pool(x, pool_axis, pool_scale)
    else:
        st, row_of, row_off, row_tok = mask_rows(keep_idx, h, w, pool_axis)
        if st != FVO_OK:
            raise OracleError(st, "mask_rows")
        out.update(row_of=row_of, row_off=row_off, row_tok=row_tok)
        xbar = pool_masked(x, row_off, row_tok, pooled_over(h, w, pool_axis), pool_scale)
    u, delta = proj(xbar, W_x, W_dt, b_dt, R, N)
    ys = scan(xbar, delta, u, A_log, R, N, dir_flags, zoh_exact)
    if keep_idx is None:
        y = gate_dense(x, z, ys, D, pool_axis, ln_gamma, ln_beta, ln_eps)
    else:
        y = gate_masked(x, z, ys, D, out["row_of"], ln_gamma, ln_beta, ln_eps)
    out.update(xbar=xbar, u=u, delta=delta, ys=ys, y=y)
    return out


def backward(x, z, A_log, D, W_x, W_dt, b_dt, dy, pool_axis, dir_flags, keep_idx=None, h=None, w=None,
             pool_scale=1.0, zoh_exact=False, nthreads=1, allow_bad_index=False, ln_gamma=None, ln_beta=None,
             ln_eps=1e-5):
    """The gradient of the layer for the upstream gradient dy (layout of y), image by image.

    Returns a dict of fp64 arrays: dx, dz (layouts of x, z) and the parameter gradients summed
    over the batch, dA_log, dD, dW_x, dW_dt, db_dt (layouts of the parameters), plus dln_gamma,
    dln_beta when the post-SSM LayerNorm is given; with allow_bad_index, also the status under
    "status".
    """
    x, z, dy = _f32(x), _f32(z), _f32(dy)
    A_log, D, W_x, W_dt, b_dt = map(_f32, (A_log, D, W_x, W_dt, b_dt))
    nd, E, N = A_log.shape
    R = W_dt.shape[2]
    if keep_idx is None:
        B, h, w, E2 = x.shape
        K = 0
        idx = None
    else:
        B, K, E2 = x.shape
        idx = _i32(keep_idx)
        assert h is not None and w is not None and idx.shape == (B, K)
    assert E2 == E and z.shape == x.shape and dy.shape == x.shape and nd == nd_of(dir_flags)
    g, b = _ln(ln_gamma, ln_beta, E)
    out = {"dx": np.empty(x.shape), "dz": np.empty(x.shape), "dA_log": np.empty(A_log.shape),
           "dD": np.empty(D.shape), "dW_x": np.empty(W_x.shape), "dW_dt": np.empty(W_dt.shape),
           "db_dt": np.empty(b_dt.shape)}
    if g is not None:
        out["dln_gamma"], out["dln_beta"] = np.empty(E), np.empty(E)
    st = _load().fvo_backward(_p(x), _p(z), _p(A_log), _p(D), _p(W_x), _p(W_dt), _p(b_dt), _p(idx), B, h, w, E,
                              N, R, K, pool_axis, int(dir_flags), float(pool_scale), int(bool(zoh_exact)), _p(g),
                              _p(b), float(ln_eps), _p(dy), int(nthreads),
                              *(_p(out[k]) for k in ("dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt")),
                              _p(out.get("dln_gamma")), _p(out.get("dln_beta")))
    _check(st, "backward", allow=(FVO_BAD_INDEX,) if allow_bad_index else ())
    if allow_bad_index:
        out["status"] = st
    return out
