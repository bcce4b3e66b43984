"""The pins catch plausible mistakes: each mutant of the oracle's C source must fail a pin.

Every mutation below is a slip one could make writing the layer (a wrong divisor, a swapped
operand, a transposed weight, a scan emitting before it updates, ...).  Each mutant is compiled
from a patched copy of ``oracle/fastvim_oracle.c`` into a temporary directory and run through
the pins of ``test_oracle_pins.py``; the test passes when at least one pin fails.  Mutations
are chosen so that the mutant never indexes out of bounds on the pins' shapes.
"""
import importlib.util
import inspect
import os
import shutil

import pytest

import test_oracle_pins as pins

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

MUTATIONS = {
    "pool divides by T": ("acc / (double)S;\n            }\n    return FVO_OK;\n}\n\n/* Row of",
                          "acc / (double)T;\n            }\n    return FVO_OK;\n}\n\n/* Row of"),
    "scan emits before update": ("hs = Abar * hs + Bbar * xbar[m * E + e];\n                        ys[m * E + e] += Cn * hs;",
                                 "ys[m * E + e] += Cn * hs;\n                        hs = Abar * hs + Bbar * xbar[m * E + e];"),
    "directions swapped": ("(dir == FVO_FWD) ? step : T - 1 - step", "(dir == FVO_BWD) ? step : T - 1 - step"),
    "A sign dropped": ("const double A = -exp(", "const double A = exp("),
    "B and C swapped": ("Bn = um[R + n], Cn = um[R + N + n]", "Bn = um[R + N + n], Cn = um[R + n]"),
    "W_dt transposed": ("W_dt[((size_t)k * E + e) * R + r]", "W_dt[((size_t)k * R + r) * E + e]"),
    "softplus without log": ("log1p(exp(-fabs(v)))", "exp(-fabs(v))"),
    "sigmoid instead of SiLU": ("return v / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(-v));"),
    "skip from one direction only": ("for (int k = 0; k < nd; ++k) Dsum +=", "for (int k = 0; k < 1; ++k) Dsum +="),
    "Abar uses Delta of previous step": ("const double Abar = exp(dt * A);",
                                         "const double Abar = exp((step ? delta[((size_t)k * M + (size_t)b * T + ((dir == FVO_FWD) ? t - 1 : t + 1)) * E + e] : dt) * A);"),
    "exact and Euler input terms swapped": ("zoh_exact ? (Abar - 1.0) / A * Bn : dt * Bn", "zoh_exact ? dt * Bn : (Abar - 1.0) / A * Bn"),
    "masked pool divides by T": ("pool_scale * acc / (double)S;\n            }\n    return FVO_OK;\n}\n\n/* Input-dependent",
                                 "pool_scale * acc / (double)T;\n            }\n    return FVO_OK;\n}\n\n/* Input-dependent"),
    "duplicate ids accepted": ("if (g < 0 || g >= G || seen[g])", "if (g < 0 || g >= G)"),
    "LayerNorm with the unbiased variance": ("var /= (double)E;", "var /= (double)(E - 1);"),
    "LayerNorm eps outside the root": ("1.0 / sqrt(var + eps)", "1.0 / (sqrt(var) + eps)"),
    "LayerNorm gamma and beta swapped": ("(double)gamma[e] * ((s[e] - mu) * inv) + (double)beta[e]",
                                         "(double)beta[e] * ((s[e] - mu) * inv) + (double)gamma[e]"),
    "LayerNorm before the skip": ("tmp[e] = ysr[e] + Dsum * (double)x[e];\n    }\n    if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);",
                                  "tmp[e] = ysr[e];\n    }\n    if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);\n"
                                  "    for (int e = 0; e < E; ++e) for (int k = 0; k < nd; ++k) tmp[e] += (double)D[(size_t)k * E + e] * (double)x[e];"),
    "LayerNorm after the gate": ("    if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);\n    for (int e = 0; e < E; ++e) y[e] = silu((double)z[e]) * tmp[e];",
                                 "    for (int e = 0; e < E; ++e) tmp[e] *= silu((double)z[e]);\n"
                                 "    if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);\n    for (int e = 0; e < E; ++e) y[e] = tmp[e];"),
    "conv taps reversed": ("(double)conv_w[((size_t)k * E + e) * dc + q]", "(double)conv_w[((size_t)k * E + e) * dc + (dc - 1 - q)]"),
    "conv filter of slot 0 for both directions": ("(double)conv_w[((size_t)k * E + e) * dc + q]",
                                                  "(double)conv_w[((size_t)0 * E + e) * dc + q]"),
    "backward conv causal too": ("(dir == FVO_FWD) ? p - (dc - 1) + q : p + (dc - 1) - q", "p - (dc - 1) + q"),
    "conv sequence row-major on both axes": ("const int t = p / S, s = p % S;\n    *i = (pool_axis == FVO_POOL_W) ? t : s;\n    *j = (pool_axis == FVO_POOL_W) ? s : t;",
                                             "(void)S;\n    *i = p / w;\n    *j = p % w;"),
    "conv bias dropped": ("double acc = (double)conv_b[(size_t)k * E + e];", "double acc = 0.0;"),
    "conv padding wraps around": ("const int pp = (dir == FVO_FWD) ? p - (dc - 1) + q : p + (dc - 1) - q;",
                                  "const int pp = (((dir == FVO_FWD) ? p - (dc - 1) + q : p + (dc - 1) - q) + L) % L;"),
    "conv skip from the forward slot only": ("v += (double)D[(size_t)k * E + e] * xc[(size_t)k * all + g + e];",
                                             "v += (double)D[(size_t)k * E + e] * xc[g + e];"),
    "both directions pool the forward convolved tokens": ("fvo_pool_d(xc + (size_t)k * img, 1,", "fvo_pool_d(xc, 1,"),
    "states stored after the update": ('                        hin[((((size_t)slot * B + b) * T + s) * E + e) * N + n] = h;\n                        const int t = d == FVO_FWD ? s : T - 1 - s;\n                        const size_t row = (size_t)b * T + t;\n                        const double dlt = delta[((size_t)slot * rows + row) * E + e];\n                        const double bn = u[((size_t)slot * rows + row) * J + R + n];\n                        const double ab = exp(dlt * a_n);\n                        const double q = zoh_exact ? (ab - 1.0) / a_n * bn : dlt * bn;\n                        h = ab * h + q * xbar[row * E + e];\n',
                                       '                        const int t = d == FVO_FWD ? s : T - 1 - s;\n                        const size_t row = (size_t)b * T + t;\n                        const double dlt = delta[((size_t)slot * rows + row) * E + e];\n                        const double bn = u[((size_t)slot * rows + row) * J + R + n];\n                        const double ab = exp(dlt * a_n);\n                        const double q = zoh_exact ? (ab - 1.0) / a_n * bn : dlt * bn;\n                        h = ab * h + q * xbar[row * E + e];\n                        hin[((((size_t)slot * B + b) * T + s) * E + e) * N + n] = h;\n'),
    "backward states in time order": ("const int t = d == FVO_FWD ? s : T - 1 - s;", "const int t = s;"),
    "state input term from C": ("const double bn = u[((size_t)slot * rows + row) * J + R + n];",
                                "const double bn = u[((size_t)slot * rows + row) * J + R + N + n];"),
    "pool scale ignored": ("pool_scale * acc / (double)S;\n            }\n    return FVO_OK;\n}\n\n/* Row of",
                           "acc / (double)S;\n            }\n    return FVO_OK;\n}\n\n/* Row of"),
}


def _pin_calls():
    """(name, fn, kwargs) for every pin, parametrisations expanded."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames, values = mark.args[0], mark.args[1]
            argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            new = []
            for p in params:
                for v in values:
                    vv = v if len(argnames) > 1 else (v,)
                    q = dict(p)
                    q.update(zip(argnames, vv))
                    new.append(q)
            params = new
        for p in params:
            calls.append((name, fn, p))
    return calls


def _mutant(tmp_path, old, new):
    src = open(os.path.join(ORACLE_DIR, "fastvim_oracle.c")).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    d = tmp_path / "mutant"
    d.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "fastvim_oracle.h"), d / "fastvim_oracle.h")
    (d / "fastvim_oracle.c").write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("oracle_mutant", os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(d / "fastvim_oracle.c")
    mod._HDR = str(d / "fastvim_oracle.h")
    mod._LIB_PATH = str(d / "libfastvim_oracle.so")
    mod._lib = None
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_every_mutant_fails_a_pin(tmp_path, mutation):
    old, new = MUTATIONS[mutation]
    mod = _mutant(tmp_path, old, new)
    for name, fn, kw in _pin_calls():
        try:
            fn(oracle_mod=mod, **kw)
        except (AssertionError, mod.OracleError):
            return  # caught
    pytest.fail(f"no pin caught the mutant '{mutation}'")


def test_unmutated_oracle_passes_every_pin(oracle_mod):
    for name, fn, kw in _pin_calls():
        fn(oracle_mod=oracle_mod, **kw)
