"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake into a copy of oracle/m2rnn_oracle.c,
builds it into a temporary library, points the oracle at it and runs the pins
of tests/test_oracle_pins.py: at least one pin must fail.  The real oracle is
restored afterwards.  The mistakes are slips that the chain rule of the
recurrence (gist.science technical summary §2.1) and the reading y_t = H_tᵀ q_t
make easy: a transposed W, the gate's two branches swapped, the rank-1 term
dropped, the readout taken before the update, and in the backward a dropped
f_t in the carry of G, a missing tanh derivative, the sign of df, dq from the
previous state and a transposed W in the carry.
"""
import subprocess

import pytest

import test_oracle_pins as pins
from oracle import oracle

MUTANTS = {
    "transposed_W": ("s += Hprev[(size_t)i * V + l] * W[(size_t)l * V + c];",
                     "s += Hprev[(size_t)i * V + l] * W[(size_t)c * V + l];"),
    "gate_swapped": ("Hn[e] = ft * Hp[e] + (1.0 - ft) * tanh(A[e]);",
                     "Hn[e] = (1.0 - ft) * Hp[e] + ft * tanh(A[e]);"),
    "rank1_dropped": ("A[(size_t)i * V + c] = s + kt[i] * vt[c];", "A[(size_t)i * V + c] = s;"),
    "readout_before_update": ("for (int i = 0; i < K; ++i) s += Hn[(size_t)i * V + c] * qt[i];",
                              "for (int i = 0; i < K; ++i) s += Hp[(size_t)i * V + c] * qt[i];"),
    "carry_without_f": ("A[(size_t)i * V + l] = ft * G[(size_t)i * V + l] + s;",
                        "A[(size_t)i * V + l] = G[(size_t)i * V + l] + s;"),
    "no_tanh_derivative": ("dA[e] = (1.0 - ft) * G[e] * (1.0 - z * z);", "dA[e] = (1.0 - ft) * G[e];"),
    "df_sign": ("dft += G[e] * (Hp[e] - z);", "dft += G[e] * (z - Hp[e]);"),
    "dq_from_previous_state": ("for (int c = 0; c < V; ++c) s += Hn[(size_t)i * V + c] * dyt[c];",
                               "for (int c = 0; c < V; ++c) s += Hp[(size_t)i * V + c] * dyt[c];"),
    "carry_W_transposed": ("for (int c = 0; c < V; ++c) s += dA[(size_t)i * V + c] * W[(size_t)l * V + c];",
                           "for (int c = 0; c < V; ++c) s += dA[(size_t)i * V + c] * W[(size_t)c * V + l];"),
}

PINS = [
    pins.test_closed_form_W0_f0, pins.test_f1_keeps_initial_state, pins.test_ema_closed_form_W0_constant_gate,
    pins.test_f0_rows_are_torch_elman_rnns, pins.test_f0_backward_matches_torch_autograd,
    pins.test_convex_blend_bound, pins.test_row_permutation_equivariance,
    pins.test_column_permutation_equivariance, pins.test_two_by_two_written_out,
    lambda: pins.test_backward_finite_differences(3, 4), pins.test_backward_closed_form_f1,
    pins.test_backward_closed_form_W0_f0,
]


@pytest.fixture
def swap_oracle():
    saved = (oracle._LIB_PATH, oracle._lib)

    def use(path):
        oracle._LIB_PATH, oracle._lib = path, None
    yield use
    oracle._LIB_PATH, oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, tmp_path, swap_oracle):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    c_file, so_file = tmp_path / "mutant.c", tmp_path / "libmutant.so"
    c_file.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                           str(c_file), "-o", str(so_file), "-lpthread", "-lm"])
    swap_oracle(str(so_file))
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, "no pin catches %s" % name


def test_the_real_oracle_passes_every_pin_listed_here():
    for pin in PINS:
        pin()
