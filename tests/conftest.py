import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")
    config.addinivalue_line("markers", "slow: oracle runs that take tens of seconds on CPU")


def cuda_ok() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library through the thin Python binding (fails loudly if unbuilt)."""
    from context_attention_dit_b200 import binding

    return binding.load()


_PARITY_LINES = []


@pytest.fixture
def parity_report():
    """Record a line for the session's parity summary (printed even under -q)."""
    return _PARITY_LINES.append


def pytest_terminal_summary(terminalreporter):
    if _PARITY_LINES:
        terminalreporter.section("parity summary")
        for line in _PARITY_LINES:
            terminalreporter.write_line(line)
