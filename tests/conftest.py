import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


@pytest.fixture(autouse=True)
def _restore_test_hooks():
    """Leave the library's process-wide test hooks (forced kernels, stalled
    chunk, wait limit) at their defaults after every test, however the test
    ended, so that no later call runs on a hook a failed test left set."""
    yield
    api = sys.modules.get("kalman_linear_attention_b200.api")
    lib = getattr(api, "_lib", None) if api is not None else None
    if lib is not None:
        lib.kla_debug_force_forward_kernel(0)
        lib.kla_debug_force_backward_kernel(0)
        lib.kla_debug_stall_chunk(-1)
        lib.kla_set_wait_limit_ns(1_000_000_000)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (seconds to minutes)")
