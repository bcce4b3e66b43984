"""Shared helpers of the test suite: the layer's tolerance and a GPU runner that also returns
the intermediates the library leaves in its workspace."""
from __future__ import annotations

import numpy as np

# The layer's fp32 tolerance, stated as "max relative error <= 1e-4 and max absolute error
# <= 1e-5 after normalising by the output RMS": an element g of the GPU result passes against
# the fp64 oracle value r when |g - r| <= 1e-5 * rms(r) + 1e-4 * |r|.
ABS_RMS = 1e-5
REL = 1e-4


# The gradient's tolerance.  dx and dz are per-token results of the same kind as y and take the
# layer's tolerance.  The parameter gradients are sums over the whole batch (dD over B h w tokens,
# the others over B T pooled tokens) accumulated in fp32 (per-thread runs of up to ~10^4 terms,
# then atomic additions in arbitrary order): rounding grows like u sqrt(n) ~ 6e-8 * 100, and each
# summand carries the few-1e-6 relative error of the fp32 chain before it, so they are held to
# |g - r| <= 1e-4 * rms(r) + 1e-4 * |r|.
GRAD_PARAM_ABS_RMS = 1e-4


def rms(a) -> float:
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def tol_report(got, ref, abs_rms=ABS_RMS) -> dict:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    r = rms(ref)
    err = np.abs(got - ref)
    bound = abs_rms * r + REL * np.abs(ref)
    bad = ~(err <= bound)  # NaN fails too
    return dict(
        rms=r,
        max_abs_over_rms=float(err.max() / r) if err.size and r > 0 else float(err.max(initial=0.0)),
        max_err_over_bound=float((err / np.maximum(bound, 1e-300)).max(initial=0.0)),
        n_bad=int(bad.sum()),
        n=int(err.size),
    )


def assert_close(got, ref, what="y", abs_rms=ABS_RMS):
    rep = tol_report(got, ref, abs_rms)
    assert rep["n_bad"] == 0, f"{what}: {rep['n_bad']}/{rep['n']} elements outside tolerance; {rep}"
    return rep


def gpu_forward(inp: dict, pool_axis: int, dir_flags: int, h=None, w=None, pool_scale=1.0, zoh_exact=False,
                intermediates=True, path="auto", ln_eps=1e-5):
    """Run the CUDA layer on numpy inputs; return y (and workspace intermediates) as numpy.  The
    post-SSM LayerNorm runs when inp holds ln_gamma and ln_beta, the block's Conv1D when it holds
    conv_w and conv_b (conv_silu: a bool entry)."""
    import torch

    from pooled_selective_scan_b200 import ssm

    dev = torch.device("cuda")
    conv_silu = bool(inp.get("conv_silu", False))
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in inp.items()
         if v is not None and k != "conv_silu"}
    keep = t.get("keep_idx")
    ln = "ln_gamma" in t
    d_conv = t["conv_w"].shape[-1] if "conv_w" in t else 0
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, dir_flags, keep, h, w, pool_scale, zoh_exact,
                            path, ln, ln_eps, d_conv, conv_silu)
    ws = ssm.alloc_workspace(shape, dev)
    ws.fill_(0xFF)  # poison: every intermediate must be written before it is read
    y = ssm.forward(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], pool_axis, dir_flags,
                    keep_idx=keep, h=h, w=w, pool_scale=pool_scale, zoh_exact=zoh_exact, workspace=ws, path=path,
                    ln_gamma=t.get("ln_gamma"), ln_beta=t.get("ln_beta"), ln_eps=ln_eps, conv_w=t.get("conv_w"),
                    conv_b=t.get("conv_b"), conv_silu=conv_silu)
    status = ssm.device_status(ws)
    out = dict(y=y.cpu().numpy(), status=status, launches=ssm.launch_names(shape))
    if intermediates:
        L = ssm.workspace_layout(shape)
        B, T, E, nd, J = shape.B, L["T"], shape.E, L["nd"], shape.R + 2 * shape.N

        def view(off, count, dtype):
            nbytes = count * np.dtype(dtype).itemsize
            return ws[off:off + nbytes].cpu().numpy().view(dtype).copy()

        nx = nd if d_conv else 1
        xb = view(L["xbar"], B * nx * T * E, np.float32).reshape(B, nx, T, E)
        out["xbar"] = xb if d_conv else xb[:, 0]
        ub = -(-T * J // 32) * 32  # per (direction, image) block stride, floats
        out["u"] = (view(L["u"], nd * B * ub, np.float32).reshape(B, nd, ub)[:, :, :T * J].reshape(B, nd, T, J)
                    .transpose(1, 0, 2, 3))
        out["ys"] = view(L["ys"], B * T * E, np.float32).reshape(B, T, E)
        if shape.K:
            out["row_of"] = view(L["row_of"], B * shape.K, np.int32).reshape(B, shape.K)
            out["row_off"] = view(L["row_off"], B * (T + 1), np.int32).reshape(B, T + 1)
            out["row_tok"] = view(L["row_tok"], B * shape.K, np.int32).reshape(B, shape.K)
    return out
