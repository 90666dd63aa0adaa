import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


def pytest_sessionfinish(session, exitstatus):
    """Write the near-margin counts of the selection checks (tests/parity.py)
    to the file named by ADASPARK_PARITY_RECORD, when set."""
    path = os.environ.get("ADASPARK_PARITY_RECORD")
    if not path:
        return
    try:
        from tests import parity
    except Exception:  # the GPU helpers could not be imported: nothing recorded
        return
    if parity.RECORD:
        import json
        with open(path, "w") as f:
            json.dump(parity.RECORD, f, indent=0)
