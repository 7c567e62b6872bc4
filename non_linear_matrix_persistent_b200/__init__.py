"""B200-native (sm_100a) M²RNN recurrence: Z_t = tanh(H_{t-1}W + k_t v_tᵀ),
H_t = f_t H_{t-1} + (1 - f_t) Z_t, y_t = H_tᵀ q_t, behind the C ABI of
include/m2rnn.h (libm2rnn.so).  ``api`` holds the torch-tensor binding,
``inputs`` the seeded synthetic workloads.
"""
import importlib

from .inputs import WORKLOADS, Workload, make_inputs  # noqa: F401

_API_NAMES = ("forward", "backward", "step", "device_status", "set_wait_limit_ns", "decay_logit_bias")


def __getattr__(name):
    # The CUDA binding is imported on first use so that the input generator
    # stays importable on machines without the built library.
    if name == "api" or name in _API_NAMES:
        mod = importlib.import_module(__name__ + ".api")
        return mod if name == "api" else getattr(mod, name)
    raise AttributeError(name)
