import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle():
    from oracle import coda_oracle
    return coda_oracle


def pytest_sessionfinish(session, exitstatus):
    """Write the measured error ratios of the parity checks (if any ran)."""
    try:
        from tests import _util
    except Exception:
        return
    if not _util.RESULTS:
        return
    import json
    # opt-in: the directory named by CODA_PARITY_REPORT_DIR receives parity_errors.json
    out = os.environ.get("CODA_PARITY_REPORT_DIR", "")
    if out and os.path.isdir(out):
        path = os.path.join(out, "parity_errors.json")
        prev = {}
        if os.path.exists(path):
            try:
                prev = json.load(open(path))
            except ValueError:
                prev = {}
        prev.update(_util.RESULTS)
        with open(path, "w") as f:
            json.dump(prev, f, indent=1, sort_keys=True)
