import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_sessionfinish(session, exitstatus):
    """With MOE_PARITY_REPORT=<path>, write every recorded error (normwise and element-wise, per
    case and tensor) as JSON."""
    path = os.environ.get("MOE_PARITY_REPORT")
    if not path:
        return
    from tests import parity
    if parity.REPORT:
        import json
        with open(path, "w") as f:
            json.dump(parity.REPORT, f, indent=1)
