"""The gradient pins catch plausible mistakes in the gradient oracle.

Each mutant below is a slip one could make deriving or writing the backward rule (a derivative
of SiLU taken as the sigmoid, the adjoint carried with the wrong step's decay, a dropped chain
factor, a missed 1/S, a transposed weight).  It is compiled from a patched copy of
``oracle/fastvim_oracle_grad.c`` and run through the pins of ``test_oracle_grad_pins.py``; the
test passes when at least one pin fails.
"""
import importlib.util
import inspect
import os
import shutil

import pytest

import test_oracle_grad_pins as pins

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

MUTATIONS = {
    "SiLU derivative taken as the sigmoid": ("s * sg * (1.0 + zz * (1.0 - sg))", "s * sg"),
    "skip gradient from one direction": ("        dysr[e] += ds;\n        dx[e] = ds * Dsum;\n        for (int k = 0; k < g->nd; ++k) dD[",
                                         "        dysr[e] += ds;\n        dx[e] = ds * (double)D[e];\n        for (int k = 0; k < g->nd; ++k) dD["),
    "LayerNorm adjoint without the mean term": ("(gs[e] - mean_gs - sh[e] * mean_gs_sh) * inv", "(gs[e] - sh[e] * mean_gs_sh) * inv"),
    "LayerNorm adjoint without the projection term": ("(gs[e] - mean_gs - sh[e] * mean_gs_sh) * inv", "(gs[e] - mean_gs) * inv"),
    "LayerNorm dgamma without the normalised value": ("gp->dln_gamma[e] += dn * sh[e];", "gp->dln_gamma[e] += dn;"),
    "LayerNorm dz from the pre-norm value": ("dz[e] = (double)dy[e] * n * sg", "dz[e] = (double)dy[e] * s[e] * sg"),
    "adjoint decays with the current step": ("lam = Cn * dyt + Abar_next * lam;", "lam = Cn * dyt + Abar * lam;"),
    "dC from the previous state": ("+= dyt * hist[t];", "+= dyt * hprev;"),
    "Abar term of dDelta dropped": ("double d_dt = lam * hprev * Abar * A;", "double d_dt = 0.0;"),
    "dA_log without the chain factor": ("+= dA * A;", "+= dA;"),
    "Euler dB without Delta": ("+= lam * dt * xb;", "+= lam * xb;"),
    "softplus derivative dropped": ("ddelta[((size_t)k * T + t) * E + e] * sigmoid(v)", "ddelta[((size_t)k * T + t) * E + e]"),
    "dW_dt transposed": ("gp->dW_dt[((size_t)k * E + e) * R + r]", "gp->dW_dt[((size_t)k * R + r) * E + e]"),
    "pooling gradient without 1/S": ("g->pool_scale / (double)g->S *", "g->pool_scale *"),
    "exact ZOH dA term dropped": ("dA += lam * Bn * xb * (dt * Abar * A - (Abar - 1.0)) / (A * A);", ""),
    "backward scan adjoint runs forward": ("const int tp = (dir == FVO_FWD) ? t - 1 : t + 1;",
                                          "const int tp = (dir == FVO_FWD) ? t + 1 : t - 1;"),
}


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argname, values = mark.args[0], mark.args[1]
            params = [dict(p, **{argname: v}) for p in params for v in values]
        calls += [(name, fn, p) for p in params]
    return calls


def _mutant(tmp_path, old, new):
    src = open(os.path.join(ORACLE_DIR, "fastvim_oracle_grad.c")).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    d = tmp_path / "mutant"
    d.mkdir()
    for f in ("fastvim_oracle.h", "fastvim_oracle.c"):
        shutil.copy(os.path.join(ORACLE_DIR, f), d / f)
    (d / "fastvim_oracle_grad.c").write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("oracle_grad_mutant", os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(d / "fastvim_oracle.c")
    mod._GRAD_SRC = str(d / "fastvim_oracle_grad.c")
    mod._HDR = str(d / "fastvim_oracle.h")
    mod._LIB_PATH = str(d / "libfastvim_oracle.so")
    mod._lib = None
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_every_gradient_mutant_fails_a_pin(tmp_path, mutation):
    old, new = MUTATIONS[mutation]
    mod = _mutant(tmp_path, old, new)
    for name, fn, kw in _pin_calls():
        try:
            fn(oracle_mod=mod, **kw)
        except (AssertionError, mod.OracleError):
            return
    pytest.fail(f"no pin caught the mutant '{mutation}'")
