"""Seeded synthetic inputs for the M²RNN recurrence.

This module only draws random numbers and casts them; it contains none of the
recurrence's arithmetic, so both the CPU oracle (through the tests) and the
CUDA path can take their inputs from here without sharing any computation.

Draw recipe (one torch CPU ``Generator`` seeded once, draws in this order):
  k, v, q, f-logits, W, H0, dY.
* ``N(0, s2)`` means variance ``s2``: k, q ~ N(0, 1/K), v ~ N(0, 1/V),
  W ~ N(0, 1/V) per head, dY ~ N(0, 1).
* The gate value is ``f = sigmoid(z + shift)`` with ``z ~ N(0, gate_var)``; it is
  an input here (the gate parameterisation psi(x_t) is outside the recurrence).
  With ``gate_logits`` the workload passes the logit ``z + shift`` instead (the
  kernels then apply the logistic function).
* H0 is zero, or U(-h0_range, h0_range) when ``h0_range > 0``.
* All draws are fp32; in bf16 mode k, v, q, W and dY are then rounded to bf16
  (round-to-nearest-even, torch's cast).  f, H0 stay fp32.

Tensors are head-first and contiguous:
  k, q [B, G, T, K]; v [B, H, T, V]; f [B, H, T]; W [H, V, V];
  H0 [B, H, K, V]; dY [B, H, T, V].
G = H unless ``qk_heads`` is set (k and q shared by groups of H / G heads).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shape, arithmetic mode and input distribution."""

    name: str
    B: int
    H: int
    T: int
    K: int
    V: int
    mode: str = "bf16"          # "bf16" (tensor-core path) or "fp32" (debug path)
    gate_var: float = 1.0       # variance of the gate logit z
    gate_shift: float = 2.0     # f = sigmoid(z + gate_shift)
    h0_range: float = 0.0       # 0 -> H0 = 0, else U(-h0_range, h0_range)
    backward: bool = False      # whether the workload includes BPTT
    seed: int = 0
    qk_heads: int = 0           # k / q head groups G (0: one per head)
    gate_logits: bool = False   # f holds the gate logit z + gate_shift instead of its sigmoid
    ckpt_stride: int = 8        # checkpoint stride C of a training workload's forward and backward

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the M²RNN hot path (shapes follow the 410M dense and 7B
# MoE models of the M²RNN paper summaries; draw recipe in the module docstring).
WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", B=1, H=1, T=64, K=16, V=16, mode="fp32"),
    "layer410m_fwd": Workload("layer410m_fwd", B=8, H=16, T=2048, K=64, V=64),
    "long_b1_fwd": Workload("long_b1_fwd", B=1, H=16, T=16384, K=64, V=64, h0_range=0.5),
    "layer7b_moe_fwd": Workload("layer7b_moe_fwd", B=4, H=32, T=4096, K=128, V=128,
                                gate_var=1.5, gate_shift=1.5),
    "layer410m_train": Workload("layer410m_train", B=8, H=16, T=2048, K=64, V=64,
                                backward=True),
    # the 7B-MoE layer shape trained: its inputs plus dY ~ N(0, 1)
    "layer7b_moe_train": Workload("layer7b_moe_train", B=4, H=32, T=4096, K=128, V=128,
                                  gate_var=1.5, gate_shift=1.5, backward=True),
}


def make_inputs(w: Workload, device: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Draw the inputs of workload ``w`` on the CPU and optionally move them.

    Returns a dict with k, v, q, f, W, H0 (None when zero) and, for backward
    workloads, dY.  bf16 mode returns bf16 k/v/q/W/dY; fp32 mode returns fp32.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    B, H, T, K, V = w.B, w.H, w.T, w.K, w.V
    G = w.qk_heads or H
    k = torch.randn(B, G, T, K, generator=g) * (1.0 / math.sqrt(K))
    v = torch.randn(B, H, T, V, generator=g) * (1.0 / math.sqrt(V))
    q = torch.randn(B, G, T, K, generator=g) * (1.0 / math.sqrt(K))
    z = torch.randn(B, H, T, generator=g) * math.sqrt(w.gate_var)
    f = (z + w.gate_shift) if w.gate_logits else torch.sigmoid(z + w.gate_shift)
    W = torch.randn(H, V, V, generator=g) * (1.0 / math.sqrt(V))
    H0 = None
    if w.h0_range > 0:
        H0 = (torch.rand(B, H, K, V, generator=g) * 2.0 - 1.0) * w.h0_range
    dY = torch.randn(B, H, T, V, generator=g) if w.backward else None

    lp = torch.bfloat16 if w.mode == "bf16" else torch.float32
    out = {
        "k": k.to(lp), "v": v.to(lp), "q": q.to(lp), "f": f.float(),
        "W": W.to(lp), "H0": None if H0 is None else H0.float(),
    }
    if dY is not None:
        out["dY"] = dY.to(lp)
    if device is not None:
        out = {n: (None if t is None else t.to(device)) for n, t in out.items()}
    return out


def make_shard_inputs(w: Workload, rank: int, device: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Inputs of data-parallel shard `rank` of a global batch of world·B rows.

    The data (k, v, q, f, H0, dY) of shard r are drawn with seed w.seed + r; the
    per-head parameter W is the same on every shard (drawn with w.seed), as a
    shared layer parameter must be.
    """
    x = make_inputs(dataclasses.replace(w, seed=w.seed + rank))
    if rank != 0:
        x["W"] = make_inputs(w)["W"]
    if device is not None:
        x = {n: (None if t is None else t.to(device)) for n, t in x.items()}
    return x
