import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# One line per full-shape parity check (max errors, near ties), printed at the end of the
# session, so that a quiet run still shows the measured errors.
PARITY_LINES: list[str] = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-shape case, minutes of CPU work")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if PARITY_LINES:
        terminalreporter.write_sep("-", "parity report")
        for line in PARITY_LINES:
            terminalreporter.write_line(line)


@pytest.fixture(scope="session")
def parity_report():
    """Append a line to the end-of-session parity report."""
    return PARITY_LINES.append


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
