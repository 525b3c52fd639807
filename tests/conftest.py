import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    from packed_cache_decode_b200 import binding
    return binding.load()


def pytest_terminal_summary(terminalreporter):
    """Near-threshold code statistics of every packed-cache comparison with the oracle in
    this run: coordinates compared, how many lie within 1e-6 of a decision threshold, and
    how many of those the CUDA encoder coded differently (only those may differ)."""
    try:
        from tests import parity_util
    except Exception:
        return
    s = parity_util.NEAR_STATS
    if s["coords"]:
        terminalreporter.write_line(
            f"packed codes vs oracle: {s['coords']} coordinates compared, {s['near']} within 1e-6 of a "
            f"threshold, {s['near_coded_differently']} of those coded differently, 0 elsewhere")
