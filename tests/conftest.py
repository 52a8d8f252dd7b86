import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionfinish(session, exitstatus):
    """Write every parity check's maximum error to $FATTN_PARITY_JSON (when set), with a
    per-(test, quantity kind) summary of the worst case."""
    path = os.environ.get("FATTN_PARITY_JSON")
    if not path:
        return
    from tests import parity
    worst = {}
    for r in parity.RECORDS:
        key = (r["test"], r["kind"])
        if key not in worst or r["frac_of_bound"] > worst[key]["frac_of_bound"]:
            worst[key] = r
    summary = sorted(worst.values(), key=lambda r: (r["test"], r["kind"]))
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump({"checks": len(parity.RECORDS), "worst_per_test": summary}, f, indent=1)
