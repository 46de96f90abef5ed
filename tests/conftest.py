import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


# Parity figures recorded by the GPU tests (test, quantity, value, bound),
# printed after the run so the literal errors are visible beside the bars.
PARITY = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    if not PARITY:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity with the fp64 oracle (literal figures)")
    for test, what, value, bound in PARITY:
        tr.write_line(f"{test:<70} {what:<34} {value:.3e}  (bar {bound})")


@pytest.fixture(scope="session")
def cuda_lib():
    """The compiled C-ABI library, loaded through the Python binding."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotated_w4_linear_b200 import binding
    return binding.lib()
