"""Seeded synthetic inputs for the FastVim SSM layer (numpy only; none of the layer's arithmetic).

The oracle and the CUDA library are both fed from here; neither imports the other.  The draws
follow the usual Mamba/Vim initialisation that the layer is specified with:

  x, z   ~ N(0, 1) fp32, one independent stream per image:  default_rng([seed, 1, b]) for x,
           default_rng([seed, 2, b]) for z, so that any single image can be regenerated alone;
  per direction slot k (stream default_rng([seed, 0]), drawn in the order W_x, W_dt, Delta0):
           A_log = log([1 .. N]) for every channel (A = -[1 .. N]);  D = 1;
           W_x  ~ U(-1/sqrt(E), 1/sqrt(E))   [R+2N, E]
           W_dt ~ U(-1/sqrt(R), 1/sqrt(R))   [E, R]
           Delta0 ~ exp(U(ln 1e-3, ln 0.1))  [E],  b_dt = Delta0 + log(-expm1(-Delta0)),
           i.e. the value whose softplus is Delta0 (the initial step sizes are log-uniform);
  keep_idx[b] = default_rng([seed, 3, b]).permutation(h*w)[:K] (int32, unsorted) for a masked
           layer at keep ratio K / (h*w);
  dy     ~ N(0, 1) fp32, the upstream gradient of a training step, default_rng([seed, 4, b]);
  the block's Conv1D (per direction slot, stream default_rng([seed, 5])): taps and bias
           ~ U(-1/sqrt(d_conv), 1/sqrt(d_conv)), the default initialisation of a depthwise
           torch Conv1d (fan-in d_conv).
"""
from __future__ import annotations

import numpy as np

from .configs import LayerConfig


def params(E: int, N: int, R: int, nd: int, seed: int) -> dict:
    rng = np.random.default_rng([seed, 0])
    A_log = np.empty((nd, E, N), np.float32)
    D = np.ones((nd, E), np.float32)
    W_x = np.empty((nd, R + 2 * N, E), np.float32)
    W_dt = np.empty((nd, E, R), np.float32)
    b_dt = np.empty((nd, E), np.float32)
    for k in range(nd):
        A_log[k] = np.log(np.arange(1, N + 1, dtype=np.float64))[None, :].astype(np.float32)
        bx = 1.0 / np.sqrt(E)
        W_x[k] = rng.uniform(-bx, bx, size=(R + 2 * N, E)).astype(np.float32)
        bd = 1.0 / np.sqrt(R)
        W_dt[k] = rng.uniform(-bd, bd, size=(E, R)).astype(np.float32)
        delta0 = np.exp(rng.uniform(np.log(1e-3), np.log(0.1), size=E))
        b_dt[k] = (delta0 + np.log(-np.expm1(-delta0))).astype(np.float32)
    return dict(A_log=A_log, D=D, W_x=W_x, W_dt=W_dt, b_dt=b_dt)


def image_x(seed: int, b: int, shape) -> np.ndarray:
    return np.random.default_rng([seed, 1, b]).standard_normal(shape, dtype=np.float32)


def image_z(seed: int, b: int, shape) -> np.ndarray:
    return np.random.default_rng([seed, 2, b]).standard_normal(shape, dtype=np.float32)


def image_dy(seed: int, b: int, shape) -> np.ndarray:
    return np.random.default_rng([seed, 4, b]).standard_normal(shape, dtype=np.float32)


def image_keep_idx(seed: int, b: int, h: int, w: int, K: int) -> np.ndarray:
    return np.random.default_rng([seed, 3, b]).permutation(h * w)[:K].astype(np.int32)


def token_shape(cfg: LayerConfig) -> tuple:
    """Per-image shape of x, z and y."""
    return (cfg.K, cfg.E) if cfg.masked else (cfg.h, cfg.w, cfg.E)


def images(cfg: LayerConfig, which=None) -> dict:
    """x, z (and keep_idx) for the images listed in ``which`` (all images by default)."""
    which = range(cfg.B) if which is None else list(which)
    shp = token_shape(cfg)
    out = dict(
        x=np.stack([image_x(cfg.seed, b, shp) for b in which]) if len(which) else np.empty((0,) + shp, np.float32),
        z=np.stack([image_z(cfg.seed, b, shp) for b in which]) if len(which) else np.empty((0,) + shp, np.float32),
    )
    if cfg.masked:
        out["keep_idx"] = (np.stack([image_keep_idx(cfg.seed, b, cfg.h, cfg.w, cfg.K) for b in which])
                           if len(which) else np.empty((0, cfg.K), np.int32))
    return out


def layer_inputs(cfg: LayerConfig, which=None) -> dict:
    """Parameters plus the images in ``which``."""
    d = params(cfg.E, cfg.N, cfg.R, cfg.nd, cfg.seed)
    d.update(images(cfg, which))
    return d


def conv_params(E: int, d_conv: int, nd: int, seed: int) -> dict:
    """Weights of the block's Conv1D: conv_w [nd, E, d_conv], conv_b [nd, E]."""
    rng = np.random.default_rng([seed, 5])
    bound = 1.0 / np.sqrt(d_conv)
    w = rng.uniform(-bound, bound, size=(nd, E, d_conv)).astype(np.float32)
    b = rng.uniform(-bound, bound, size=(nd, E)).astype(np.float32)
    return dict(conv_w=w, conv_b=b)
