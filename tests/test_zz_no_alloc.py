"""m2rnn_backward_noalloc: the allocation-free backward entry point.

For callers that cannot allocate device memory when they need gradients
(services that forbid allocator calls after start-up, because an allocation
can synchronise the device or fail under memory pressure, and hosts that hand
the library only the tensors they already own).  The entry point takes its
scratch from an array compiled into the library instead of a caller
workspace.  It runs the same deterministic kernels as m2rnn_backward (every
reduction in a fixed order), so its gradients must equal m2rnn_backward's bit
for bit on the same inputs, call after call (the array keeps the previous
call's contents).  This file is collected last so that a failure here leaves
every other test already run.
"""
import pytest
import torch

from non_linear_matrix_persistent_b200 import Workload, make_inputs

pytestmark = pytest.mark.gpu

NAMES = ("dk", "dv", "dq", "df", "dW", "dH0")


def _noalloc(d, xc, ck, dHT, out):
    from non_linear_matrix_persistent_b200 import _lib
    P = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return _lib.lib().m2rnn_backward_noalloc(
        d, P(xc["k"]), P(xc["v"]), P(xc["q"]), P(xc["f"]), P(xc["W"]), P(ck), P(xc["dY"]), P(dHT),
        P(out["dk"]), P(out["dv"]), P(out["dq"]), P(out["df"]), P(out["dW"]), P(out["dH0"]),
        torch.cuda.current_stream().cuda_stream)


def _empty_grads(w, dev):
    B, H, T, K, V = w.B, w.H, w.T, w.K, w.V
    shapes = {"dk": (B, H, T, K), "dv": (B, H, T, V), "dq": (B, H, T, K), "df": (B, H, T),
              "dW": (H, V, V), "dH0": (B, H, K, V)}
    # filled with NaN so that anything the call fails to write shows up
    return {n: torch.full(s, float("nan"), dtype=torch.float32, device=dev) for n, s in shapes.items()}


@pytest.mark.parametrize("mode,K,V", [("bf16", 64, 64), ("fp32", 64, 64), ("bf16", 128, 128)])
def test_noalloc_backward_matches_workspace_backward(mode, K, V):
    """K = V = 128 runs the general-shape tensor-core backward, whose scratch in
    the array also holds the four row slices' dv and df partials."""
    from non_linear_matrix_persistent_b200 import _lib, api
    C = 8
    w = Workload("na", B=2, H=3, T=37, K=K, V=V, mode=mode, h0_range=0.5, backward=True, seed=11)
    x = make_inputs(w)
    xc = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    dHT = torch.randn(w.B, w.H, w.K, w.V, generator=torch.Generator().manual_seed(2)).cuda()
    assert _lib.lib().m2rnn_workspace_size(api.dims_of(xc["k"], xc["v"], C), 1) <= (32 << 20)
    _, _, ck = api.forward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], xc["H0"], ckpt_stride=C, want_ckpt=True)
    ref = api.backward(xc["k"], xc["v"], xc["q"], xc["f"], xc["W"], ck, xc["dY"], dHT, ckpt_stride=C)
    torch.cuda.synchronize()
    d = api.dims_of(xc["k"], xc["v"], C)
    for call in range(2):   # two calls in a row: the shared array keeps the previous call's contents
        out = _empty_grads(w, xc["k"].device)
        st = _noalloc(d, xc, ck, dHT, out)
        assert st == _lib.OK, _lib.status_string(st)
        torch.cuda.synchronize()
        for n in NAMES:
            assert torch.isfinite(out[n]).all(), (call, n)
            # same kernels, same order of every sum: identical bits
            assert torch.equal(out[n], ref[n]), (call, n, float((out[n] - ref[n]).abs().max()))


def test_noalloc_rejects_problems_larger_than_its_array():
    from non_linear_matrix_persistent_b200 import _lib
    # 128 (b, h) pairs x 33 states x 64 x 64 fp32 of recompute scratch is far above 32 MiB
    d = _lib.Dims(8, 16, 2048, 64, 64, _lib.MODE_BF16_TC, 16)
    assert _lib.lib().m2rnn_workspace_size(d, 1) > (32 << 20)
    st = _lib.lib().m2rnn_backward_noalloc(d, *([4096] * 14), None)
    assert st == _lib.ERR_WORKSPACE
