"""The seeded input recipe (non_linear_matrix_persistent_b200/inputs.py) on
the CPU: draws are reproducible, have the stated variances, and the grouped
and gate-logit variants describe the same draws in another form."""
import math

import torch

from non_linear_matrix_persistent_b200 import WORKLOADS, Workload, make_inputs


def test_draws_are_reproducible_and_seeded():
    w = Workload("r", B=2, H=3, T=50, K=16, V=32, h0_range=0.5, backward=True, seed=4)
    a, b = make_inputs(w), make_inputs(w)
    for n in a:
        assert torch.equal(a[n], b[n]), n
    c = make_inputs(w.with_(seed=5))
    assert not torch.equal(a["k"], c["k"])


def test_variances_and_ranges_follow_the_recipe():
    w = Workload("v", B=4, H=8, T=512, K=64, V=32, h0_range=0.5, backward=True, seed=0)
    x = make_inputs(w)
    for n, var in (("k", 1 / 64), ("q", 1 / 64), ("v", 1 / 32), ("W", 1 / 32), ("dY", 1.0)):
        got = x[n].float().var().item()
        assert abs(got / var - 1) < 0.03, (n, got, var)
    assert x["k"].dtype == torch.bfloat16 and x["f"].dtype == torch.float32
    assert 0 < x["f"].min() and x["f"].max() < 1
    # f = sigmoid(z + 2), z ~ N(0, 1): mean of the logit is 2
    logit = torch.log(x["f"] / (1 - x["f"]))
    assert abs(logit.mean().item() - 2.0) < 0.02 and abs(logit.var().item() - 1.0) < 0.03
    assert x["H0"].abs().max() <= 0.5


def test_gate_logit_variant_is_the_same_draw():
    w = WORKLOADS["layer410m_train"].with_(T=64)
    f = make_inputs(w)["f"]
    a = make_inputs(w.with_(gate_logits=True))["f"]
    assert torch.allclose(torch.sigmoid(a), f, rtol=0, atol=1e-6)


def test_grouped_variant_draws_group_shaped_k_and_q():
    w = Workload("g", B=2, H=8, T=10, K=16, V=16, qk_heads=2, seed=1)
    x = make_inputs(w)
    assert x["k"].shape == (2, 2, 10, 16) and x["q"].shape == (2, 2, 10, 16)
    assert x["v"].shape == (2, 8, 10, 16) and x["W"].shape == (8, 16, 16)
    assert math.isclose(x["k"].float().std().item(), 0.25, rel_tol=0.15)
