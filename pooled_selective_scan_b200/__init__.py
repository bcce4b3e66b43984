"""B200-native FastVim SSM layer (pooled selective scan) behind a C-ABI CUDA library.

The compute lives in ``libfastvim_ssm.so`` (hand-written sm_100a kernels, built from ``csrc/``);
this package only marshals arguments to it (``ssm``), holds the workload shapes (``configs``)
and the seeded synthetic inputs (``inputs``).  The native library is loaded on first use and a
missing or unloadable library raises instead of falling back to anything else.
"""
from .configs import CONFIGS, DIR_BWD, DIR_FWD, HEADLINE, POOL_H, POOL_W, LayerConfig  # noqa: F401

__all__ = ["CONFIGS", "HEADLINE", "LayerConfig", "POOL_W", "POOL_H", "DIR_FWD", "DIR_BWD"]
