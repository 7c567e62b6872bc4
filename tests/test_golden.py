"""The oracle against the stored fixtures of tests/golden/oracle_small.json
(written by tests/golden/make_golden.py from the oracle): a change in what the
oracle computes shows up here and must be justified by the passage, or the
reading of it, that it follows."""
import json
import os

import numpy as np
import pytest

from oracle import oracle

with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")) as fh:
    CASES = json.load(fh)["cases"]


@pytest.mark.parametrize("c", CASES, ids=[c["name"] for c in CASES])
def test_oracle_reproduces_stored_values(c):
    x = {n: np.array(a, dtype=np.float64) for n, a in c["inputs"].items()}
    logit = c["f_is_logit"]
    y, HT = oracle.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], nthreads=2, f_is_logit=logit)
    g = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dy"], x["dHT"], nthreads=2,
                        f_is_logit=logit)
    got = {"y": y, "HT": HT, **g}
    for n, want in c["outputs"].items():
        np.testing.assert_allclose(got[n], np.array(want), rtol=1e-12, atol=1e-14, err_msg=n)
