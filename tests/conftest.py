import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def root():
    return ROOT


def pytest_sessionfinish(session, exitstatus):
    """With PARITY_REPORT=<path> set, write the error records of every parity run of the
    session (rel, per-head and element-wise measures; see gpu_util) to that file."""
    path = os.environ.get("PARITY_REPORT")
    mod = sys.modules.get("gpu_util")
    if path and mod is not None and mod.REPORT:
        mod.write_report(path)
