"""Device-resident synthetic workloads (seeded, image by image from ``inputs``).

Builds the full-batch tensors of a ``LayerConfig`` on a CUDA device without ever holding more
than one image of x or z on the host, so the 3.2 GB-per-tensor 2048 px layer can be set up on
any host.  Pinned host copies (for end-to-end runs) are built the same way on request.
"""
from __future__ import annotations

import numpy as np
import torch

from . import inputs
from .configs import LayerConfig


def params_tensors(cfg: LayerConfig, device) -> dict:
    p = inputs.params(cfg.E, cfg.N, cfg.R, cfg.nd, cfg.seed)
    return {k: torch.from_numpy(v).to(device) for k, v in p.items()}


def shard_images(cfg: LayerConfig, rank: int, world: int) -> range:
    """Global image ids that rank ``rank`` of ``world`` processes: every rank holds its own batch of
    ``cfg.B`` distinct images (the global batch is world * B; images are independent, so ranks
    exchange nothing)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    return range(rank * cfg.B, (rank + 1) * cfg.B)


def activations(cfg: LayerConfig, device, pinned_host: bool = False, first_image: int = 0) -> dict:
    """x, z (and keep_idx) for images first_image .. first_image + B - 1 of ``cfg``'s seeded
    stream on ``device`` (or in pinned host memory)."""
    shp = inputs.token_shape(cfg)
    kw = dict(dtype=torch.float32)
    if pinned_host:
        x = torch.empty((cfg.B,) + shp, pin_memory=True, **kw)
        z = torch.empty((cfg.B,) + shp, pin_memory=True, **kw)
    else:
        x = torch.empty((cfg.B,) + shp, device=device, **kw)
        z = torch.empty((cfg.B,) + shp, device=device, **kw)
    for i in range(cfg.B):
        b = first_image + i
        x[i].copy_(torch.from_numpy(inputs.image_x(cfg.seed, b, shp)), non_blocking=False)
        z[i].copy_(torch.from_numpy(inputs.image_z(cfg.seed, b, shp)), non_blocking=False)
    out = dict(x=x, z=z)
    if cfg.masked:
        idx = np.stack([inputs.image_keep_idx(cfg.seed, first_image + i, cfg.h, cfg.w, cfg.K) for i in range(cfg.B)])
        t = torch.from_numpy(idx)
        out["keep_idx"] = t.pin_memory() if pinned_host else t.to(device)
    return out


def upstream_grad(cfg: LayerConfig, device, pinned_host: bool = False, first_image: int = 0) -> torch.Tensor:
    """dy (the gradient arriving at the layer's output in a training step) for the same images."""
    shp = inputs.token_shape(cfg)
    if pinned_host:
        dy = torch.empty((cfg.B,) + shp, dtype=torch.float32, pin_memory=True)
    else:
        dy = torch.empty((cfg.B,) + shp, dtype=torch.float32, device=device)
    for i in range(cfg.B):
        dy[i].copy_(torch.from_numpy(inputs.image_dy(cfg.seed, first_image + i, shp)))
    return dy


def ln_tensors(cfg: LayerConfig, device) -> dict:
    """Post-SSM LayerNorm weights at their usual initialisation: gamma = 1, beta = 0."""
    return dict(ln_gamma=torch.ones(cfg.E, dtype=torch.float32, device=device),
                ln_beta=torch.zeros(cfg.E, dtype=torch.float32, device=device))


def conv_tensors(cfg: LayerConfig, device, d_conv: int = 4) -> dict:
    """The block's Conv1D weights (seeded, default depthwise Conv1d initialisation)."""
    c = inputs.conv_params(cfg.E, d_conv, cfg.nd, cfg.seed)
    return {k: torch.from_numpy(v).to(device) for k, v in c.items()}


def layer_tensors(cfg: LayerConfig, device, pinned_host: bool = False, first_image: int = 0) -> dict:
    d = params_tensors(cfg, "cpu" if pinned_host else device)
    if pinned_host:
        d = {k: v.pin_memory() for k, v in d.items()}
    d.update(activations(cfg, device, pinned_host, first_image))
    return d
