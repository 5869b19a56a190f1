import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_sessionfinish(session, exitstatus):
    """Write the parity records of the GPU tests (plain max-abs / mean-abs per compared tensor) to the
    file named by SAP_PARITY_REPORT, when that variable is set."""
    path = os.environ.get("SAP_PARITY_REPORT")
    if not path:
        return
    helpers = sys.modules.get("gpu_helpers")
    records = list(getattr(helpers, "PARITY_RECORDS", [])) if helpers else []
    import json
    d = os.path.dirname(path)
    if d:
        os.makedirs(d, exist_ok=True)
    with open(path, "w") as f:
        json.dump({"exitstatus": int(exitstatus), "records": records}, f, indent=1)
