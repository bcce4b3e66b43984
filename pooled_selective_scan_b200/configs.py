"""Workload shapes of the FastVim SSM layer used by the tests and the benchmark.

Each entry is one SSM layer of a FastVim model on a square token grid (patch 16), fp32:
FastVim-T (d_model 192, E = 384, dt_rank 12), FastVim-S (d_model 384, E = 768, dt_rank 24) and
a FastMaskVim-B layer (d_model 768, E = 1536, dt_rank 48) under a 75 % random keep-mask.  The
method's efficiency study measures batch 128, fp32, at 224 to 2048 px (gptget.net summary of
FastVim 2502.00594, section "关键结果"; pith.science verdict, Table 23 as quoted there).
"""
from __future__ import annotations

from dataclasses import dataclass, field

POOL_W = 0  # mean over the w index, T = h tokens
POOL_H = 1  # mean over the h index, T = w tokens
DIR_FWD = 1
DIR_BWD = 2


@dataclass(frozen=True)
class LayerConfig:
    name: str
    B: int
    h: int
    w: int
    E: int
    R: int
    pool_axes: tuple = (POOL_W,)
    N: int = 16
    dir_flags: int = DIR_FWD | DIR_BWD
    K: int = 0  # kept tokens per sample (masked layer); 0 = dense grid
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def nd(self) -> int:
        return int(bool(self.dir_flags & DIR_FWD)) + int(bool(self.dir_flags & DIR_BWD))

    @property
    def masked(self) -> bool:
        return self.K > 0

    def tokens_per_call(self) -> int:
        """Grid tokens one call processes (kept tokens for the masked layer)."""
        return self.B * (self.K if self.masked else self.h * self.w)

    def algorithmic_bytes_per_call(self) -> int:
        """x and z read once, y written once: 12 E bytes per processed token."""
        return 12 * self.E * self.tokens_per_call()


CONFIGS = [
    LayerConfig("fastvim_t_224_tiny", B=2, h=14, w=14, E=384, R=12, pool_axes=(POOL_W,), seed=0,
                note="FastVim-T layer, 224 px, batch 2, column pooling"),
    LayerConfig("fastvim_t_224", B=128, h=14, w=14, E=384, R=12, pool_axes=(POOL_W, POOL_H), seed=1,
                note="FastVim-T layer, 224 px, batch 128, both pool axes (alternating blocks)"),
    LayerConfig("fastvim_s_1024", B=128, h=64, w=64, E=768, R=24, pool_axes=(POOL_H,), seed=2,
                note="FastVim-S layer, 1024 px, batch 128, row pooling"),
    LayerConfig("fastvim_t_2048", B=128, h=128, w=128, E=384, R=12, pool_axes=(POOL_W,), seed=3,
                note="FastVim-T layer, 2048 px, batch 128, column pooling"),
    LayerConfig("fastmaskvim_b_1024_mask75", B=64, h=64, w=64, E=1536, R=48, pool_axes=(POOL_W,),
                K=1024, seed=4,
                note="FastMaskVim-B layer, 64x64 grid, 75 % of tokens masked"),
]

HEADLINE = CONFIGS[3]


def by_name(name: str) -> LayerConfig:
    for c in CONFIGS:
        if c.name == name:
            return c
    raise KeyError(name)
