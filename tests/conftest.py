import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def repo_root():
    return ROOT


def pytest_sessionfinish(session, exitstatus):
    """With RESS_PARITY_REPORT=<file>, writes the mask agreement and attention error of
    every full-layer GPU parity check of the session to that JSON file."""
    path = os.environ.get("RESS_PARITY_REPORT")
    if not path:
        return
    mod = sys.modules.get("parity")
    if mod is None or not getattr(mod, "REPORT", None):
        return
    import json
    with open(path, "w") as f:
        json.dump(mod.REPORT, f, indent=1)
