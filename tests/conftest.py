import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def repo_root():
    return ROOT


def pytest_sessionfinish(session, exitstatus):
    """Write the error figures every GPU parity comparison recorded (plain
    max-abs, envelope-scaled max-abs, rel-L2, share within the plain bound)
    to tests/results/parity_errors.json, or to $LH_PARITY_REPORT."""
    import json
    try:
        import torch
        from tests.parity import RECORDS
    except Exception:
        return
    if not RECORDS or not torch.cuda.is_available():
        return
    path = os.environ.get("LH_PARITY_REPORT",
                          os.path.join(ROOT, "tests", "results", "parity_errors.json"))
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump({"device": torch.cuda.get_device_name(0), "exitstatus": int(exitstatus),
                   "records": RECORDS}, f, indent=1)
