import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Print the parameter-gradient errors measured by the parity tests."""
    stats = sys.modules.get("parity")
    stats = getattr(stats, "PARAM_GRAD_STATS", None) if stats else None
    if not stats:
        return
    terminalreporter.write_line("parameter gradients: workload name rel_l2 cancellation "
                                "rounding-sigma/|ref|")
    for row in stats:
        terminalreporter.write_line("  %s %s %.3e %.3e %.3e" % row)
