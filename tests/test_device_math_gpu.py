"""The SFU-based device math of the layer (softplus, SiLU, 2^x) against fp64 numpy over their
whole input range, through fastvim_selftest_math.  Error bounds: the SFU exp2/log2/rcp are
accurate to about 2^-22 relative; rounding the exponent argument to fp32 adds |arg| * 2^-24 * ln2
relative; results below 2^-126 flush to zero."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from pooled_selective_scan_b200 import _native as nat  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run(fn, v):
    dev = torch.device("cuda")
    x = torch.from_numpy(v.astype(np.float32)).to(dev)
    y = torch.empty_like(x)
    st = nat.lib().fastvim_selftest_math(fn, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                         x.numel(), None)
    assert st == nat.FV_OK
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), x.cpu().numpy().astype(np.float64)


def grid(lo, hi, n=400_001):
    v = np.linspace(lo, hi, n)
    return np.concatenate([v, [0.0, -0.0, 1e-30, -1e-30, 20.0, -20.0]])


def test_softplus():
    g, v = run(0, grid(-87.0, 60.0))
    r = np.logaddexp(0.0, v)
    bound = (1e-6 + 2 ** -24 * np.log(2) * np.abs(v) * np.log2(np.e) * 2) * r + 1e-37
    assert np.all(np.abs(g - r) <= bound), float(np.max(np.abs(g - r) / bound))


def test_silu():
    g, v = run(1, grid(-87.0, 87.0))
    r = v / (1.0 + np.exp(-v))
    bound = (1e-6 + 2 ** -24 * np.abs(v) * 2) * np.abs(r) + 1e-35
    assert np.all(np.abs(g - r) <= bound), float(np.max(np.abs(g - r) / bound))


def test_exp2():
    g, v = run(2, grid(-126.0, 127.0))
    r = np.exp2(v)
    assert np.all(np.abs(g - r) <= 1e-6 * r), float(np.max(np.abs(g - r) / r))
    g2, _ = run(2, np.array([-127.5, -150.0, -1e4]))
    assert np.all(g2 == 0.0)  # below 2^-126: flushed to zero
