import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case (minutes)")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # noqa: BLE001
        return False


@pytest.fixture(scope="session")
def gpu():
    if not cuda_available():
        pytest.fail("a gpu-marked test ran without a CUDA device")
    import torch
    return torch.device("cuda", 0)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the rel-L2 of every attention comparison made against the oracle."""
    try:
        import _parity
    except ImportError:
        return
    if not _parity.RECORDS:
        return
    terminalreporter.write_sep("-", "attention parity against the fp64 oracle")
    for label, r, mx, mn, gate in _parity.RECORDS:
        terminalreporter.write_line(f"{label}: rel-L2 {r:.3e} (gate {gate:g}), max-abs {mx:.2e}, mean-abs {mn:.2e}")
