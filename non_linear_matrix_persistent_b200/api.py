"""Python binding of libm2rnn.so over torch tensors (argument marshalling only).

Every step of the recurrence runs in the CUDA library; torch only provides
device memory and the current stream.  Names follow include/m2rnn.h.

  y, HT, ckpt = forward(k, v, q, f, W, H0=None, ckpt_stride=8, want_ckpt=False)
  grads       = backward(k, v, q, f, W, ckpt, dy, dHT=None, ckpt_stride=8)
  y_t         = step(k_t, v_t, q_t, f_t, W, H)        # one decode step, H updated in place
  b           = decay_logit_bias(H)                   # per-head gate-logit bias at initialisation

k and q may carry fewer heads than v (G dividing H: grouped k / q, head h
uses group h // (H // G)); dk and dq then have G heads too.  With
f_is_logit=True, f holds gate logits a_t (f_t = sigmoid(a_t), evaluated in
the kernels) and backward returns dL/da_t as df.

bf16 k/v/q/W select the tensor-core mode (M2RNN_MODE_BF16_TC); fp32 select
the fp32 debug mode; forward(..., fast_tanh=True) and forward(...,
mma_sync=True) select the forward-only alternatives.  Tensors must be
contiguous CUDA tensors with the head-first layouts of the header.

The default checkpoint stride, 8, is the longest chunk that the V = 64
tensor-core backward keeps in tensor memory for K = 64 and 128 (16 for
K = 32); longer strides (up to 16) run the general-shape backward.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

from . import _lib
from ._lib import Dims, M2RNNError

_workspaces: Dict[Tuple[int, int], torch.Tensor] = {}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _mode(k: torch.Tensor) -> int:
    if k.dtype == torch.bfloat16:
        return _lib.MODE_BF16_TC
    if k.dtype == torch.float32:
        return _lib.MODE_FP32_DEBUG
    raise TypeError("k/v/q/W must be bfloat16 (tensor-core mode) or float32 (debug mode), got %s" % k.dtype)


def _check(name, t, shape, dtype, device):
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError("%s must be a CUDA tensor on %s" % (name, device))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype:
        raise TypeError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def dims_of(k: torch.Tensor, v: torch.Tensor, ckpt_stride: int = 8, f_is_logit: bool = False) -> Dims:
    """Dims of a call: H from v, the k / q head groups G from k."""
    B, G, T, K = k.shape
    H = v.shape[1]
    if G < 1 or H % G != 0:
        if H > 0 or G > 0:
            raise ValueError("k has %d heads: it must have H = %d heads or a divisor of H" % (G, H))
    return Dims(B, H, T, K, v.shape[-1], _mode(k), ckpt_stride, G if G != H else 0, int(bool(f_is_logit)))


def _ws_key(device) -> Tuple[int, int]:
    """Workspaces are cached per (device, stream): calls that the library
    orders on one stream may share one, calls on different streams may
    overlap on the GPU and must not."""
    index = device.index if device.index is not None else torch.cuda.current_device()
    return index, _stream(torch.device("cuda", index))


def workspace(d: Dims, backward: bool, device) -> torch.Tensor:
    """Zero-initialised device workspace (cached per device and current
    stream, grown on demand)."""
    need = _lib.lib().m2rnn_workspace_size(d, 1 if backward else 0)
    if need == 0:
        raise M2RNNError(_lib.ERR_INVALID_ARG, "m2rnn_workspace_size")
    key = _ws_key(device)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def num_checkpoints(T: int, ckpt_stride: int) -> int:
    return (T + ckpt_stride - 1) // ckpt_stride


def forward(k, v, q, f, W, H0=None, *, ckpt_stride: int = 8, want_ckpt: bool = False,
            want_HT: bool = True, out: Optional[dict] = None, fast_tanh: bool = False,
            mma_sync: bool = False, f_is_logit: bool = False):
    """Runs the forward scan.  Returns (y, HT or None, ckpt or None).

    Two bf16-only alternatives to the default tensor-core forward:
    fast_tanh selects M2RNN_MODE_BF16_TC_FAST_TANH (the single-SFU
    tanh.approx.f32, for inference; its checkpoints are not meant for the
    backward); mma_sync selects M2RNN_MODE_BF16_MMA_SYNC (the register-resident
    forward for V = 64, K <= 64; its checkpoints feed the backward as usual)."""
    dev = k.device
    d = dims_of(k, v, ckpt_stride, f_is_logit)
    if fast_tanh or mma_sync:
        if d.mode != _lib.MODE_BF16_TC:
            raise TypeError("fast_tanh / mma_sync need bf16 inputs (the tensor-core mode)")
        if fast_tanh and mma_sync:
            raise ValueError("choose one of fast_tanh and mma_sync")
        d.mode = _lib.MODE_BF16_TC_FAST_TANH if fast_tanh else _lib.MODE_BF16_MMA_SYNC
    B, H, T, K, V = d.B, d.H, d.T, d.K, d.V
    lp = k.dtype
    G = d.qk_heads or H
    _check("k", k, (B, G, T, K), lp, dev)
    _check("v", v, (B, H, T, V), lp, dev)
    _check("q", q, (B, G, T, K), lp, dev)
    _check("f", f, (B, H, T), torch.float32, dev)
    _check("W", W, (H, V, V), lp, dev)
    _check("H0", H0, (B, H, K, V), torch.float32, dev)
    out = out or {}
    y = out.get("y")
    if y is None:
        y = torch.empty(B, H, T, V, dtype=torch.float32, device=dev)
    HT = out.get("HT") if want_HT else None
    if want_HT and HT is None:
        HT = torch.empty(B, H, K, V, dtype=torch.float32, device=dev)
    ckpt = out.get("ckpt") if want_ckpt else None
    if want_ckpt and ckpt is None:
        ckpt = torch.empty(B, H, num_checkpoints(T, ckpt_stride), K, V, dtype=torch.float32, device=dev)
    ws = workspace(d, False, dev)
    st = _lib.lib().m2rnn_forward(d, _ptr(k), _ptr(v), _ptr(q), _ptr(f), _ptr(W), _ptr(H0), _ptr(y), _ptr(HT),
                                  _ptr(ckpt), _ptr(ws), ws.numel(), _stream(dev))
    if st != _lib.OK:
        raise M2RNNError(st, "m2rnn_forward")
    return y, HT, ckpt


def step(k, v, q, f, W, H, *, y: Optional[torch.Tensor] = None, f_is_logit: bool = False):
    """One decode step, in place: advances the fp32 state H [B, H, K, V] by one
    step of the recurrence with k, q [B, H, K] (or [B, G, K], grouped), v
    [B, H, V] and f [B, H], and returns y [B, H, V].  It is the forward with
    T = 1 and the state buffer passed as both H0 and H_T (the ABI allows that
    alias), so T calls give the scan's outputs bit for bit."""
    B, _, K = k.shape
    Hh, V = v.shape[1], v.shape[-1]
    if H is None:
        raise ValueError("step needs the state buffer H (it is updated in place)")
    _check("H", H, (B, Hh, K, V), torch.float32, k.device)
    if y is None:
        y = torch.empty(B, Hh, V, dtype=torch.float32, device=k.device)
    forward(k.unsqueeze(2), v.unsqueeze(2), q.unsqueeze(2), f.unsqueeze(2), W, H, ckpt_stride=1,
            out={"y": y.view(B, Hh, 1, V), "HT": H}, f_is_logit=f_is_logit)
    return y


def backward(k, v, q, f, W, ckpt, dy, dHT=None, *, ckpt_stride: int = 8, out: Optional[dict] = None,
             f_is_logit: bool = False):
    """BPTT from the forward's checkpoints.  Returns dict dk, dv, dq, df, dW, dH0 (fp32)."""
    dev = k.device
    d = dims_of(k, v, ckpt_stride, f_is_logit)
    B, H, T, K, V = d.B, d.H, d.T, d.K, d.V
    lp = k.dtype
    G = d.qk_heads or H
    _check("k", k, (B, G, T, K), lp, dev)
    _check("v", v, (B, H, T, V), lp, dev)
    _check("q", q, (B, G, T, K), lp, dev)
    _check("f", f, (B, H, T), torch.float32, dev)
    _check("W", W, (H, V, V), lp, dev)
    _check("ckpt", ckpt, (B, H, num_checkpoints(T, ckpt_stride), K, V), torch.float32, dev)
    _check("dy", dy, (B, H, T, V), lp, dev)
    _check("dHT", dHT, (B, H, K, V), torch.float32, dev)
    out = dict(out or {})
    shapes = {"dk": (B, G, T, K), "dv": (B, H, T, V), "dq": (B, G, T, K), "df": (B, H, T),
              "dW": (H, V, V), "dH0": (B, H, K, V)}
    for n, s in shapes.items():
        if out.get(n) is None:
            out[n] = torch.empty(*s, dtype=torch.float32, device=dev)
    ws = workspace(d, True, dev)
    st = _lib.lib().m2rnn_backward(d, _ptr(k), _ptr(v), _ptr(q), _ptr(f), _ptr(W), _ptr(ckpt), _ptr(dy),
                                   _ptr(dHT), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dq"]), _ptr(out["df"]),
                                   _ptr(out["dW"]), _ptr(out["dH0"]), _ptr(ws), ws.numel(), _stream(dev))
    if st != _lib.OK:
        raise M2RNNError(st, "m2rnn_backward")
    return out


def device_status(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device
    status of the workspace cached for that stream."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    key = _ws_key(dev)
    ws = _workspaces.get(key)
    if ws is None:
        return _lib.OK
    return _lib.lib().m2rnn_get_device_status(_ptr(ws), _stream(dev))


def set_wait_limit_ns(ns: int) -> None:
    _lib.lib().m2rnn_set_wait_limit_ns(int(ns))


def decay_logit_bias(H: int, tau_min: float = 2.0, tau_max: float = 256.0) -> torch.Tensor:
    """Per-head bias of the gate logit at initialisation, shape [H] (fp32, CPU).

    The pages parameterise the forget gate as f_t = ψ(x_t) in [0, 1] and start
    the heads with different decay rates (gist.science technical summary of
    "M²RNN", §2.1, forget gate), without giving the form.  This library's
    reading: ψ ends in the logistic function of a logit a_t = (projection of
    x_t) + b_h, and at initialisation, where the projection contributes about
    nothing, head h retains f_h = 1 / (1 + exp(-b_h)) of its state per step.
    The heads' retention times tau_h = 1 / (1 - f_h) are spaced geometrically
    from tau_min to tau_max steps, so b_h = log(tau_h - 1).  Pass logits built
    on it with f_is_logit=True."""
    if H < 1 or not (1.0 < tau_min <= tau_max):
        raise ValueError("need H >= 1 and 1 < tau_min <= tau_max")
    h = torch.arange(H, dtype=torch.float64)
    frac = h / (H - 1) if H > 1 else torch.zeros(1, dtype=torch.float64)
    tau = tau_min * (tau_max / tau_min) ** frac
    return torch.log(tau - 1.0).float()
