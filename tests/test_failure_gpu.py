"""Bounded device-side waits: an injected stall ends in a status, not a hang.

The fault is injected on the host (m2rnn_debug_set_fault(1) makes the input
producer of the forward, or of the backward, stop after its first chunk, so
the consumers wait on an mbarrier that nothing completes).  With a 2 ms wait limit the kernel gives
up, drains what it has in flight, frees its tensor memory and exits; the
status word reports the timeout and the same context then runs correctly.
No GPU fault, trap or hang is involved.
"""
import numpy as np
import pytest

from non_linear_matrix_persistent_b200 import Workload, make_inputs
from oracle import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("V", [64, 32])
def test_injected_stall_reports_timeout_and_context_stays_usable(V):
    """V = 64 with 4 pairs runs the row kernel, V = 32 the tensor-core kernel."""
    from non_linear_matrix_persistent_b200 import _lib, api
    L = _lib.lib()
    w = Workload("stall", B=2, H=2, T=40, K=64, V=V, h0_range=0.5, seed=4)
    x = make_inputs(w)
    xc = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    api.forward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], xc["H0"])   # creates the workspace
    assert api.device_status() == _lib.OK
    try:
        api.set_wait_limit_ns(2_000_000)
        assert L.m2rnn_debug_set_fault(1) == _lib.OK
        api.forward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], xc["H0"])
        assert api.device_status() == _lib.ERR_DEVICE_TIMEOUT
    finally:
        L.m2rnn_debug_set_fault(0)
        api.set_wait_limit_ns(2_000_000_000)
    assert L.m2rnn_debug_set_fault(5) == _lib.ERR_INVALID_ARG
    y, HT, _ = api.forward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], xc["H0"])
    assert api.device_status() == _lib.OK
    yr, HTr = oracle.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"])
    assert np.abs(y.double().cpu().numpy() - yr).max() <= 3e-2
    assert np.abs(HT.double().cpu().numpy() - HTr).max() <= 3e-2


@pytest.mark.parametrize("K,V", [(64, 64), (128, 128), (64, 32)])
def test_injected_stall_in_backward_reports_timeout(K, V):
    """The backward's producer stops after the first checkpoint chunk: K = V = 64
    runs the extended-operand kernel (chunk in tensor memory), K = V = 128 the
    general-shape kernel with the chunk on chip, V = 32 the general-shape
    kernel with the global scratch.  Each ends with the timeout status, and a
    second backward on the same context matches the oracle."""
    from non_linear_matrix_persistent_b200 import _lib, api
    L = _lib.lib()
    C = 8
    w = Workload("stall_bwd", B=1, H=2, T=40, K=K, V=V, h0_range=0.5, backward=True, seed=5)
    x = make_inputs(w)
    xc = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    _, _, ck = api.forward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], xc["H0"], ckpt_stride=C, want_ckpt=True)
    api.backward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], ck, xc["dY"], ckpt_stride=C)
    assert api.device_status() == _lib.OK
    try:
        api.set_wait_limit_ns(2_000_000)
        assert L.m2rnn_debug_set_fault(1) == _lib.OK
        api.backward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], ck, xc["dY"], ckpt_stride=C)
        assert api.device_status() == _lib.ERR_DEVICE_TIMEOUT
    finally:
        L.m2rnn_debug_set_fault(0)
        api.set_wait_limit_ns(2_000_000_000)
    g = api.backward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], ck, xc["dY"], ckpt_stride=C)
    assert api.device_status() == _lib.OK
    gr = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dY"])
    for n in ("dk", "dv", "dq", "df", "dW", "dH0"):
        got = g[n].double().cpu().numpy()
        assert np.linalg.norm(got - gr[n]) <= 1e-2 * np.linalg.norm(gr[n]), n
