"""The per-head gate-logit bias at initialisation (the library's reading of
the pages' per-head decay rates, gist.science technical summary of "M²RNN",
§2.1 forget gate): retention times tau_h = 1 / (1 - f_h) spaced geometrically
between tau_min and tau_max, with f_h the logistic function of the bias."""
import math

import numpy as np
import pytest
import torch

from oracle import oracle


def _bias(*a, **k):
    from non_linear_matrix_persistent_b200 import api
    return api.decay_logit_bias(*a, **k)


@pytest.mark.parametrize("H", [1, 2, 16, 32])
def test_retention_times_are_geometric_between_the_bounds(H):
    b = _bias(H, tau_min=2.0, tau_max=256.0).double().numpy()
    f = oracle.gate_from_logit(b)          # the oracle's logistic function, fp64
    tau = 1.0 / (1.0 - f)
    assert b.shape == (H,) and np.all(np.isfinite(b))
    assert abs(tau[0] - 2.0) < 1e-5 * 2.0
    if H > 1:
        assert abs(tau[-1] - 256.0) < 1e-5 * 256.0
        ratios = tau[1:] / tau[:-1]
        assert np.allclose(ratios, (256.0 / 2.0) ** (1.0 / (H - 1)), rtol=1e-5)
        assert np.all(np.diff(b) > 0)      # slower decay for later heads


def test_known_values():
    # tau = 2 -> f = 1/2 -> logit 0; tau = 256 -> logit log(255)
    b = _bias(2, tau_min=2.0, tau_max=256.0)
    assert abs(float(b[0])) < 1e-7 and abs(float(b[1]) - math.log(255.0)) < 1e-5
    assert torch.equal(_bias(4, 8.0, 8.0), torch.full((4,), math.log(7.0), dtype=torch.float32))


def test_bad_arguments():
    for a in ((0,), (4, 1.0, 8.0), (4, 8.0, 4.0)):
        with pytest.raises(ValueError):
            _bias(*a)
