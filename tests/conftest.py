import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionfinish(session, exitstatus):
    """Write the GPU tests' per-case parity records (largest absolute and
    relative error against the oracle) to $PKV_PARITY_REPORT, one JSON line
    per comparison, when that variable is set."""
    path = os.environ.get("PKV_PARITY_REPORT")
    mod = sys.modules.get("tests.gpu_helpers")
    if not path or mod is None:
        return
    import json
    with open(path, "w") as f:
        for rec in mod.PARITY_LOG:
            f.write(json.dumps(rec) + "\n")
