"""Writes tests/golden/oracle_small.json: small seeded problems and the fp64
oracle's results for them (forward y, H_T and every gradient).

The pages ("M²RNN: Non-Linear RNNs with Matrix-Valued States for Scalable
Language Modeling": the gist.science technical summary §2.1, the wispaper.ai
post §1) print no worked example, so these values are not the pages'; they
come from the oracle alone (this script imports nothing else of the
repository) and let tests/test_golden.py detect any later change in what the
oracle computes.  Cases: per-head k / q, grouped k / q (2 groups of 2 heads,
the grouped-value reading of §2.2) and gate logits (f_t = logistic(a_t), the
reading of the forget gate's ψ in §2.1).

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from oracle import oracle  # noqa: E402


def case(name, B, H, G, T, K, V, logit, seed):
    r = np.random.default_rng(seed)
    x = {
        "k": r.standard_normal((B, G, T, K)) * 0.6,
        "v": r.standard_normal((B, H, T, V)) * 0.6,
        "q": r.standard_normal((B, G, T, K)) * 0.6,
        "f": (r.standard_normal((B, H, T)) * 1.5 + 1.0) if logit
             else 1.0 / (1.0 + np.exp(-r.standard_normal((B, H, T)) - 1.0)),
        "W": r.standard_normal((H, V, V)) * (1.2 / np.sqrt(V)),
        "H0": r.uniform(-0.8, 0.8, (B, H, K, V)),
        "dy": r.standard_normal((B, H, T, V)),
        "dHT": r.standard_normal((B, H, K, V)),
    }
    y, HT = oracle.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], nthreads=1, f_is_logit=logit)
    g = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dy"], x["dHT"], nthreads=1,
                        f_is_logit=logit)
    out = {"y": y, "HT": HT, **g}
    return {"name": name, "f_is_logit": logit,
            "inputs": {n: a.tolist() for n, a in x.items()},
            "outputs": {n: np.asarray(a).tolist() for n, a in out.items()}}


def main():
    cases = [
        case("per_head", B=2, H=2, G=2, T=4, K=3, V=2, logit=False, seed=101),
        case("grouped_qk", B=1, H=4, G=2, T=3, K=2, V=3, logit=False, seed=102),
        case("gate_logits", B=1, H=2, G=2, T=5, K=2, V=2, logit=True, seed=103),
    ]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as fh:
        json.dump({"generator": "tests/golden/make_golden.py", "cases": cases}, fh, indent=None)
        fh.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
