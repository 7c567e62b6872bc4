"""fp64 CPU oracle for the M²RNN recurrence (ctypes wrapper over m2rnn_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it and shares no code
with it.

The recurrence it evaluates is the one of "M²RNN: Non-Linear RNNs with
Matrix-Valued States for Scalable Language Modeling" (gist.science technical
summary §2.1: Z_t = tanh(H_{t-1}W + k_t v_tᵀ), H_t = f_t H_{t-1} + (1-f_t) Z_t),
plus the readout y_t = H_tᵀ q_t, the library's reading because the pages
define no readout.  The backward is the exact chain rule of the same three
equations.  Every function here is pinned by tests/test_oracle_pins.py
against closed forms, invariants, torch.nn.RNN (f = 0) and finite
differences.

All arithmetic is fp64; inputs are the exact values the GPU receives (bf16 or
fp32), widened to fp64 without rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m2rnn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libm2rnn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/libm2rnn_oracle.so (gcc, -O2, IEEE math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lpthread", "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.m2rnn_oracle_forward.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P, P, i]
        lib.m2rnn_oracle_forward.restype = i
        lib.m2rnn_oracle_backward.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P, P,
                                              P, P, P, P, P, P, i]
        lib.m2rnn_oracle_backward.restype = i
        _lib = lib
    return _lib


def _f64(x) -> Optional[np.ndarray]:
    """Exact widening of a torch tensor / array to a contiguous float64 array."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _heads_of_groups(a: np.ndarray, H: int) -> np.ndarray:
    """Grouped-value form (gist.science technical summary §2.2, tensor
    parallelism: the topology-aware strategy keeps a group's heads together;
    the other strategy all-reduces the gradients of the query and key that
    heads share).  Reading: k and q carry G head groups, G dividing H, and
    head h uses the k and q of group h // (H / G); v, f, W and the state stay
    per head.  Returns the per-head [B, H, T, K] view of a [B, G, T, K] array."""
    G = a.shape[1]
    assert G >= 1 and H % G == 0, (G, H)
    return a if G == H else np.repeat(a, H // G, axis=1)


def gate_from_logit(a: np.ndarray) -> np.ndarray:
    """Forget gate from a gate logit (gist.science technical summary §2.1: a
    parameterised ψ(x_t) keeps f_t in [0, 1], with per-head decay rates at
    initialisation).  Reading: ψ ends in the logistic function,
    f_t = 1 / (1 + exp(-a_t)); how a_t is computed from x_t (a projection and
    a per-head bias that sets each head's initial decay) lies outside the
    recurrence, so a_t is an input."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-a))


def forward(k, v, q, f, W, H0=None, nthreads: Optional[int] = None,
            f_is_logit: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """Returns (y [B,H,T,V], H_T [B,H,K,V]) in fp64.  k and q may be
    [B,G,T,K] with G dividing H (grouped-value form, _heads_of_groups).  With
    f_is_logit, f holds gate logits a_t and f_t = gate_from_logit(a_t)."""
    k, v, q, f, W, H0 = (_f64(a) for a in (k, v, q, f, W, H0))
    if f_is_logit:
        f = gate_from_logit(f)
    H = v.shape[1]
    k, q = _heads_of_groups(k, H), _heads_of_groups(q, H)
    B, H, T, K = k.shape
    V = v.shape[-1]
    assert v.shape == (B, H, T, V) and q.shape == (B, H, T, K) and f.shape == (B, H, T)
    assert W.shape == (H, V, V) and (H0 is None or H0.shape == (B, H, K, V))
    y = np.zeros((B, H, T, V))
    HT = np.zeros((B, H, K, V))
    rc = _load().m2rnn_oracle_forward(B, H, T, K, V, _ptr(k), _ptr(v), _ptr(q), _ptr(f), _ptr(W),
                                      _ptr(H0), _ptr(y), _ptr(HT), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle forward failed (%d)" % rc)
    return y, HT


def backward(k, v, q, f, W, H0, dy, dHT=None, nthreads: Optional[int] = None, f_is_logit: bool = False):
    """Returns dict of fp64 gradients dk, dv, dq, df, dW, dH0 for loss with dL/dy = dy, dL/dH_T = dHT.

    With grouped k and q ([B,G,T,K], _heads_of_groups) dk and dq are [B,G,T,K]:
    the gradient of a shared input is the sum of its uses' gradients, here
    over the H / G heads of the group.  With f_is_logit, f holds gate logits
    a_t (see forward) and df is dL/da_t = dL/df_t · f_t (1 - f_t), the chain
    rule through the logistic function."""
    k, v, q, f, W, H0, dy, dHT = (_f64(a) for a in (k, v, q, f, W, H0, dy, dHT))
    if f_is_logit:
        f = gate_from_logit(f)
    G, H = k.shape[1], v.shape[1]
    k, q = _heads_of_groups(k, H), _heads_of_groups(q, H)
    B, H, T, K = k.shape
    V = v.shape[-1]
    assert dy.shape == (B, H, T, V) and (dHT is None or dHT.shape == (B, H, K, V))
    out = {"dk": np.zeros((B, H, T, K)), "dv": np.zeros((B, H, T, V)), "dq": np.zeros((B, H, T, K)),
           "df": np.zeros((B, H, T)), "dW": np.zeros((H, V, V)), "dH0": np.zeros((B, H, K, V))}
    rc = _load().m2rnn_oracle_backward(
        B, H, T, K, V, _ptr(k), _ptr(v), _ptr(q), _ptr(f), _ptr(W), _ptr(H0), _ptr(dy), _ptr(dHT),
        _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dq"]), _ptr(out["df"]), _ptr(out["dW"]),
        _ptr(out["dH0"]), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle backward failed (%d)" % rc)
    if G != H:
        for n in ("dk", "dq"):
            out[n] = out[n].reshape(B, G, H // G, T, K).sum(axis=2)
    if f_is_logit:
        out["df"] = out["df"] * f * (1.0 - f)
    return out
