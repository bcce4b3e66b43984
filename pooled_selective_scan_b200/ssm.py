"""PyTorch-facing binding of the FastVim SSM layer (argument marshalling only).

Every step of the layer runs in the CUDA library (``libfastvim_ssm.so``); PyTorch only provides
device memory and the stream.  Tensors must be contiguous fp32 (keep_idx int32) on the current
CUDA device; parameters are stacked per enabled direction (slot 0 = forward when enabled):

    A_log [nd,E,N]   D [nd,E]   W_x [nd,R+2N,E]   W_dt [nd,E,R]   b_dt [nd,E]

Dense layer:  x, z [B,h,w,E] -> y [B,h,w,E].
Masked layer: x, z [B,K,E] with keep_idx [B,K] (grid ids r*w + c of an h x w grid) -> y [B,K,E].
With the block's Conv1D (dense layers): conv_w [nd,E,d_conv], conv_b [nd,E]; x is then the Conv1D's
input.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _native as nat
from .configs import DIR_BWD, DIR_FWD, POOL_H, POOL_W  # noqa: F401


_PATH_FLAGS = {"auto": 0, "staged": 2, "fused": 4}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(name, t, dtype, device=None, host=False):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if host:
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    else:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if device is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")


@dataclass
class LayerShape:
    B: int
    h: int
    w: int
    E: int
    N: int
    R: int
    pool_axis: int
    dir_flags: int
    K: int = 0
    pool_scale: float = 1.0
    zoh_exact: bool = False
    path: str = "auto"  # "auto", "staged" or "fused" (FV_FLAG_PATH_*)
    ln: bool = False    # post-SSM LayerNorm before the gate (FV_FLAG_LAYERNORM)
    ln_eps: float = 1e-5
    d_conv: int = 0     # taps of the block's Conv1D in front of the layer (0: none)
    conv_silu: bool = False  # SiLU after the Conv1D (FV_FLAG_CONV_SILU)
    keep_states: bool = False  # the forward keeps the scan states for the gradient (FV_FLAG_KEEP_STATES)

    @property
    def nd(self) -> int:
        return int(bool(self.dir_flags & DIR_FWD)) + int(bool(self.dir_flags & DIR_BWD))

    @property
    def T(self) -> int:
        return self.h if self.pool_axis == POOL_W else self.w

    def token_shape(self):
        return (self.B, self.K, self.E) if self.K else (self.B, self.h, self.w, self.E)

    def args(self, x=None, z=None, A_log=None, D=None, W_x=None, W_dt=None, b_dt=None, keep_idx=None,
             y=None, ln_gamma=None, ln_beta=None, conv_w=None, conv_b=None) -> nat.FvSsmArgs:
        a = nat.FvSsmArgs()
        a.B, a.h, a.w, a.E, a.N, a.R = self.B, self.h, self.w, self.E, self.N, self.R
        a.pool_axis = self.pool_axis
        a.dir_flags = self.dir_flags
        a.K = self.K
        a.pool_scale = float(self.pool_scale)
        a.flags = ((nat.FV_FLAG_ZOH_EXACT if self.zoh_exact else 0) | _PATH_FLAGS[self.path] |
                   (nat.FV_FLAG_LAYERNORM if self.ln else 0) | (nat.FV_FLAG_CONV_SILU if self.conv_silu else 0) |
                   (nat.FV_FLAG_KEEP_STATES if self.keep_states else 0))
        a.x, a.z, a.A_log, a.D, a.W_x, a.W_dt, a.b_dt, a.keep_idx, a.y = (
            _ptr(x), _ptr(z), _ptr(A_log), _ptr(D), _ptr(W_x), _ptr(W_dt), _ptr(b_dt), _ptr(keep_idx), _ptr(y))
        a.ln_gamma, a.ln_beta = _ptr(ln_gamma), _ptr(ln_beta)
        a.ln_eps = float(self.ln_eps)
        a.d_conv = int(self.d_conv)
        a.conv_w, a.conv_b = _ptr(conv_w), _ptr(conv_b)
        return a


def infer_shape(x, A_log, W_dt, pool_axis, dir_flags, keep_idx=None, h=None, w=None, pool_scale=1.0,
                zoh_exact=False, path="auto", ln=False, ln_eps=1e-5, d_conv=0, conv_silu=False,
                keep_states=False) -> LayerShape:
    nd, E, N = A_log.shape
    R = W_dt.shape[2]
    if keep_idx is None:
        if x.dim() != 4:
            raise ValueError("dense x must be [B,h,w,E]")
        B, h, w, E2 = x.shape
        K = 0
    else:
        if x.dim() != 3 or h is None or w is None:
            raise ValueError("masked x must be [B,K,E] and the grid h, w must be given")
        B, K, E2 = x.shape
        if K == 0:
            raise ValueError("a masked layer needs K >= 1 kept tokens")
    if E2 != E:
        raise ValueError(f"x has E={E2}, parameters have E={E}")
    if path not in _PATH_FLAGS:
        raise ValueError(f"path must be one of {sorted(_PATH_FLAGS)}")
    s = LayerShape(B, h, w, E, N, R, pool_axis, dir_flags, K, pool_scale, zoh_exact, path, bool(ln), float(ln_eps),
                   int(d_conv), bool(conv_silu), bool(keep_states))
    if s.nd != nd:
        raise ValueError(f"dir_flags={dir_flags} enables {s.nd} directions, parameters stack {nd}")
    return s


def workspace_size(shape: LayerShape) -> int:
    a = shape.args()
    n = nat.lib().fastvim_ssm_workspace_size(ctypes.byref(a))
    if n == 0:
        nat.check(nat.lib().fastvim_ssm_validate(ctypes.byref(a)), "fastvim_ssm_workspace_size")
    return int(n)


def workspace_layout(shape: LayerShape) -> dict:
    a = shape.args()
    L = nat.FvWsLayout()
    nat.check(nat.lib().fastvim_ssm_workspace_layout(ctypes.byref(a), ctypes.byref(L)), "fastvim_ssm_workspace_layout")
    return {name: getattr(L, name) for name, _ in L._fields_}


def launch_count(shape: LayerShape) -> int:
    a = shape.args()
    return int(nat.lib().fastvim_ssm_launch_count(ctypes.byref(a)))


def launch_names(shape: LayerShape) -> list:
    a = shape.args()
    return [nat.lib().fastvim_ssm_launch_name(ctypes.byref(a), i).decode() for i in range(launch_count(shape))]


def alloc_workspace(shape: LayerShape, device=None) -> torch.Tensor:
    return torch.empty(max(workspace_size(shape), 256), dtype=torch.uint8, device=device or "cuda")


def forward(x, z, A_log, D, W_x, W_dt, b_dt, pool_axis=POOL_W, dir_flags=DIR_FWD | DIR_BWD, keep_idx=None,
            h=None, w=None, pool_scale=1.0, zoh_exact=False, y=None, workspace=None, stream=None, path="auto",
            ln_gamma=None, ln_beta=None, ln_eps=1e-5, conv_w=None, conv_b=None, conv_silu=False,
            keep_states=False):
    """Queue the layer on ``stream`` (default: the current stream) and return y.  Passing
    ln_gamma and ln_beta ([E]) adds the post-SSM LayerNorm before the gate; conv_w [nd,E,d_conv]
    and conv_b [nd,E] put the block's Conv1D in front (x is then the Conv1D's input).
    keep_states=True also stores the scan states in the workspace for a later ``backward``
    with keep_states=True (training)."""
    dev = x.device
    for name, t in (("x", x), ("z", z), ("A_log", A_log), ("D", D), ("W_x", W_x), ("W_dt", W_dt), ("b_dt", b_dt)):
        _check_tensor(name, t, torch.float32, dev)
    if keep_idx is not None:
        _check_tensor("keep_idx", keep_idx, torch.int32, dev)
    ln = ln_gamma is not None or ln_beta is not None
    if ln:
        if ln_gamma is None or ln_beta is None:
            raise ValueError("the LayerNorm needs both ln_gamma and ln_beta")
        _check_tensor("ln_gamma", ln_gamma, torch.float32, dev)
        _check_tensor("ln_beta", ln_beta, torch.float32, dev)
    d_conv = 0
    if conv_w is not None or conv_b is not None:
        if conv_w is None or conv_b is None:
            raise ValueError("the Conv1D needs both conv_w and conv_b")
        _check_tensor("conv_w", conv_w, torch.float32, dev)
        _check_tensor("conv_b", conv_b, torch.float32, dev)
        d_conv = conv_w.shape[-1]
    shape = infer_shape(x, A_log, W_dt, pool_axis, dir_flags, keep_idx, h, w, pool_scale, zoh_exact, path, ln, ln_eps,
                        d_conv, conv_silu, keep_states)
    if z.shape != x.shape:
        raise ValueError("z must have the shape of x")
    if y is None:
        y = torch.empty_like(x)
    else:
        _check_tensor("y", y, torch.float32, dev)
        if y.shape != x.shape:
            raise ValueError("y must have the shape of x")
    if workspace is None:
        workspace = alloc_workspace(shape, dev)
    a = shape.args(x, z, A_log, D, W_x, W_dt, b_dt, keep_idx, y, ln_gamma, ln_beta, conv_w, conv_b)
    st = nat.lib().fastvim_ssm_forward(ctypes.byref(a), ctypes.c_void_p(workspace.data_ptr()),
                                       ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    nat.check(st, "fastvim_ssm_forward")
    return y


class BoundForward:
    """A forward call with its tensors, workspace and argument block bound once, for repeated
    launches (benchmark loops): ``run()`` queues the layer, ``run_events(evs)`` also records
    ``evs[2i]`` and ``evs[2i+1]`` just before and after the i-th kernel launch."""

    def __init__(self, shape: LayerShape, t: dict, y, workspace, stream=None):
        self.shape = shape
        self.workspace = workspace
        self._keep = (t, y, workspace)
        self._args = shape.args(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], t.get("keep_idx"), y,
                                t.get("ln_gamma"), t.get("ln_beta"), t.get("conv_w"), t.get("conv_b"))
        self._stream = _stream_handle(stream)
        self._ws = ctypes.c_void_p(workspace.data_ptr())
        self._wsn = ctypes.c_size_t(workspace.numel())
        self.n_launch = launch_count(shape)
        self._evbuf = (ctypes.c_void_p * (2 * self.n_launch))()
        L = nat.lib()
        nat.check(L.fastvim_ssm_validate(ctypes.byref(self._args)), "fastvim_ssm_validate")

    def run(self):
        nat.check(nat.lib().fastvim_ssm_forward(ctypes.byref(self._args), self._ws, self._wsn, self._stream),
                  "fastvim_ssm_forward")

    def run_events(self, events):
        """events: 2 * n_launch CUDA events; events[2i], events[2i+1] bracket launch i."""
        for e in events:
            if not e.cuda_event:  # torch creates the CUDA event on its first record
                e.record()
        for i, e in enumerate(events):
            self._evbuf[i] = e.cuda_event
        nat.check(nat.lib().fastvim_ssm_forward_events(ctypes.byref(self._args), self._ws, self._wsn, self._stream,
                                                       self._evbuf, len(events)), "fastvim_ssm_forward_events")


def backward_workspace_size(shape: LayerShape) -> int:
    a = shape.args()
    n = nat.lib().fastvim_ssm_backward_workspace_size(ctypes.byref(a))
    if n == 0:  # an empty batch needs none; otherwise the shape is invalid
        L = nat.FvBwdWsLayout()
        nat.check(nat.lib().fastvim_ssm_backward_workspace_layout(ctypes.byref(a), ctypes.byref(L)),
                  "fastvim_ssm_backward_workspace_size")
    return int(n)


def backward_launch_names(shape: LayerShape) -> list:
    a = shape.args()
    n = nat.lib().fastvim_ssm_backward_launch_count(ctypes.byref(a))
    return [nat.lib().fastvim_ssm_backward_launch_name(ctypes.byref(a), i).decode() for i in range(n)]


def _grads(dy, grads: dict) -> nat.FvSsmGrads:
    g = nat.FvSsmGrads()
    g.dy = _ptr(dy)
    for name in ("dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt"):
        setattr(g, name, _ptr(grads[name]))
    g.dln_gamma, g.dln_beta = _ptr(grads.get("dln_gamma")), _ptr(grads.get("dln_beta"))
    return g


def backward(x, z, A_log, D, W_x, W_dt, b_dt, dy, fwd_workspace, pool_axis=POOL_W, dir_flags=DIR_FWD | DIR_BWD,
             keep_idx=None, h=None, w=None, pool_scale=1.0, zoh_exact=False, path="auto", grads=None,
             workspace=None, stream=None, ln_gamma=None, ln_beta=None, ln_eps=1e-5, keep_states=False) -> dict:
    """Queue the gradient of the layer for the upstream gradient dy on ``stream`` and return the
    dict {dx, dz, dA_log, dD, dW_x, dW_dt, db_dt} (+ dln_gamma, dln_beta with the post-SSM
    LayerNorm).  fwd_workspace is the workspace of a forward call with the same tensors and
    options (keep_states included), queued earlier on the same stream."""
    dev = x.device
    for name, t in (("x", x), ("z", z), ("A_log", A_log), ("D", D), ("W_x", W_x), ("W_dt", W_dt), ("b_dt", b_dt),
                    ("dy", dy)):
        _check_tensor(name, t, torch.float32, dev)
    if keep_idx is not None:
        _check_tensor("keep_idx", keep_idx, torch.int32, dev)
    ln = ln_gamma is not None or ln_beta is not None
    if ln:
        if ln_gamma is None or ln_beta is None:
            raise ValueError("the LayerNorm needs both ln_gamma and ln_beta")
        _check_tensor("ln_gamma", ln_gamma, torch.float32, dev)
        _check_tensor("ln_beta", ln_beta, torch.float32, dev)
    shape = infer_shape(x, A_log, W_dt, pool_axis, dir_flags, keep_idx, h, w, pool_scale, zoh_exact, path, ln, ln_eps,
                        keep_states=keep_states)
    if z.shape != x.shape or dy.shape != x.shape:
        raise ValueError("z and dy must have the shape of x")
    if grads is None:
        grads = {"dx": torch.empty_like(x), "dz": torch.empty_like(z)}
        for name, p in (("dA_log", A_log), ("dD", D), ("dW_x", W_x), ("dW_dt", W_dt), ("db_dt", b_dt)):
            grads[name] = torch.empty_like(p)
        if ln:
            grads["dln_gamma"], grads["dln_beta"] = torch.empty_like(ln_gamma), torch.empty_like(ln_beta)
    if workspace is None:
        workspace = torch.empty(max(backward_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
    # y is not read by the gradient
    a = shape.args(x, z, A_log, D, W_x, W_dt, b_dt, keep_idx, None, ln_gamma, ln_beta)
    g = _grads(dy, grads)
    st = nat.lib().fastvim_ssm_backward(ctypes.byref(a), ctypes.byref(g), ctypes.c_void_p(fwd_workspace.data_ptr()),
                                        ctypes.c_size_t(fwd_workspace.numel()), ctypes.c_void_p(workspace.data_ptr()),
                                        ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    nat.check(st, "fastvim_ssm_backward")
    return grads


class BoundBackward:
    """A gradient call with its tensors and workspaces bound once, for repeated launches:
    ``run()`` queues it, ``run_events(evs)`` also brackets each of its kernel launches."""

    def __init__(self, shape: LayerShape, t: dict, dy, grads: dict, fwd_workspace, workspace, stream=None):
        self.shape = shape
        self._keep = (t, dy, grads, fwd_workspace, workspace)
        self._args = shape.args(t["x"], t["z"], t["A_log"], t["D"], t["W_x"], t["W_dt"], t["b_dt"], t.get("keep_idx"),
                                None, t.get("ln_gamma"), t.get("ln_beta"))
        self._g = _grads(dy, grads)
        self._fw = (ctypes.c_void_p(fwd_workspace.data_ptr()), ctypes.c_size_t(fwd_workspace.numel()))
        self._ws = (ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()))
        self._stream = _stream_handle(stream)
        self.names = backward_launch_names(shape)
        self.n_launch = len(self.names)
        self._evbuf = (ctypes.c_void_p * (2 * self.n_launch))()

    def run(self):
        nat.check(nat.lib().fastvim_ssm_backward(ctypes.byref(self._args), ctypes.byref(self._g), *self._fw, *self._ws,
                                                 self._stream), "fastvim_ssm_backward")

    def run_events(self, events):
        for e in events:
            if not e.cuda_event:
                e.record()
        for i, e in enumerate(events):
            self._evbuf[i] = e.cuda_event
        nat.check(nat.lib().fastvim_ssm_backward_events(ctypes.byref(self._args), ctypes.byref(self._g), *self._fw,
                                                        *self._ws, self._stream, self._evbuf, len(events)),
                  "fastvim_ssm_backward_events")


def device_status(workspace, stream=None) -> int:
    """Wait for the stream and return the device status word of the last call (0 = FV_OK)."""
    return int(nat.lib().fastvim_get_device_status(ctypes.c_void_p(workspace.data_ptr()), _stream_handle(stream)))


class HostForward:
    """End-to-end calls on pinned host buffers through ``fastvim_ssm_forward_host``: each call
    copies the inputs host -> device, runs the layer and copies y back, returning when y is in
    host memory.  Device buffers and the workspace are allocated once here."""

    def __init__(self, shape: LayerShape, device=None):
        self.shape = shape
        dev = torch.device(device or "cuda")
        nd, E, N, R = shape.nd, shape.E, shape.N, shape.R
        mk = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)  # noqa: E731
        self.dev = dict(x=mk(*shape.token_shape()), z=mk(*shape.token_shape()), y=mk(*shape.token_shape()),
                        A_log=mk(nd, E, N), D=mk(nd, E), W_x=mk(nd, R + 2 * N, E), W_dt=mk(nd, E, R), b_dt=mk(nd, E))
        self.dev["keep_idx"] = (torch.empty((shape.B, shape.K), dtype=torch.int32, device=dev) if shape.K else None)
        self.dev["ln_gamma"] = mk(E) if shape.ln else None
        self.dev["ln_beta"] = mk(E) if shape.ln else None
        self.dev["conv_w"] = mk(nd, E, shape.d_conv) if shape.d_conv else None
        self.dev["conv_b"] = mk(nd, E) if shape.d_conv else None
        self.workspace = alloc_workspace(shape, dev)

    def h2d_bytes(self) -> int:
        s = self.shape
        act = 2 * s.B * (s.K if s.K else s.h * s.w) * s.E * 4
        par = s.nd * (s.E * s.N + 2 * s.E + (s.R + 2 * s.N) * s.E + s.E * s.R) * 4
        conv = s.nd * s.E * (s.d_conv + 1) * 4 if s.d_conv else 0
        return act + par + (s.B * s.K * 4 if s.K else 0) + (2 * s.E * 4 if s.ln else 0) + conv

    def d2h_bytes(self) -> int:
        s = self.shape
        return s.B * (s.K if s.K else s.h * s.w) * s.E * 4

    def __call__(self, host: dict, y_host, stream=None):
        for name in ("x", "z", "A_log", "D", "W_x", "W_dt", "b_dt"):
            _check_tensor(name, host[name], torch.float32, host=True)
        _check_tensor("y", y_host, torch.float32, host=True)
        d = self.dev
        ha = self.shape.args(host["x"], host["z"], host["A_log"], host["D"], host["W_x"], host["W_dt"], host["b_dt"],
                             host.get("keep_idx"), y_host, host.get("ln_gamma"), host.get("ln_beta"),
                             host.get("conv_w"), host.get("conv_b"))
        da = self.shape.args(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], d["keep_idx"], d["y"],
                             d["ln_gamma"], d["ln_beta"], d["conv_w"], d["conv_b"])
        st = nat.lib().fastvim_ssm_forward_host(ctypes.byref(ha), ctypes.byref(da),
                                                ctypes.c_void_p(self.workspace.data_ptr()),
                                                ctypes.c_size_t(self.workspace.numel()), _stream_handle(stream))
        nat.check(st, "fastvim_ssm_forward_host")
        return y_host
