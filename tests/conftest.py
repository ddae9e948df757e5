import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


def pytest_sessionfinish(session, exitstatus):
    """With LARD_PARITY_REPORT=<path>, write every parity comparison's observed
    error and bound (worst ratio first) as JSON."""
    path = os.environ.get("LARD_PARITY_REPORT")
    if not path:
        return
    try:
        import parity_util
    except ImportError:
        return
    import json
    rows = sorted(parity_util.ERRORS, key=lambda r: -(r[1] / r[2] if r[2] > 0 else 0))
    with open(path, "w") as f:
        json.dump([{"what": w, "err": e, "bound": b, "ratio": (e / b if b > 0 else None)}
                   for w, e, b in rows], f, indent=1)
