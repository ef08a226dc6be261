import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for _p in (ROOT, HERE):
    if _p not in sys.path:
        sys.path.insert(0, _p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built libgla.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(autouse=True)
def _clear_oracle_fault():
    """Every test starts and ends with no planted oracle mistake."""
    try:
        from oracle import recurrent
        recurrent.set_fault(0)
        yield
        recurrent.set_fault(0)
    except Exception:
        yield
