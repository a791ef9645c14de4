import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (runs on a B200)")
    config.addinivalue_line("markers", "slow: long-running")


@pytest.fixture(scope="session")
def oracle_default():
    import oracle
    return oracle.default()


@pytest.fixture(autouse=True)
def _no_kernel_wait_ran_out(request):
    """After every GPU test: no kernel of the library gave up a bounded wait
    (the device error word stays clear)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from bit_error_compensated_echo_b200 import abi
    torch.cuda.synchronize()
    flags = abi.echo_device_error_get(0, clear=True)
    assert flags == 0, "a kernel's bounded wait ran out (device error word %#x)" % flags
