import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def pytest_sessionfinish(session, exitstatus):
    """With ENT_PARITY_REPORT=<path>, write the worst |dO| beyond bf16 storage
    rounding seen per workload (tests/parity.py O_REPORT) as JSON."""
    path = os.environ.get("ENT_PARITY_REPORT")
    if not path:
        return
    try:
        from parity import O_REPORT
    except ImportError:
        return
    import json
    with open(path, "w") as f:
        json.dump(dict(sorted(O_REPORT.items())), f, indent=1)
