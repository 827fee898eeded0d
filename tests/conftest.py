import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workload)")


def pytest_sessionfinish(session, exitstatus):
    """Writes the parity margins (max|err|/RMS per compared tensor) of this session to the file
    named by KDA_MARGINS_FILE, one JSON object per line."""
    path = os.environ.get("KDA_MARGINS_FILE")
    if not path:
        return
    try:
        from tests.kda_check import MARGINS
    except ImportError:
        return
    if not MARGINS:
        return
    import json
    with open(path, "a") as f:
        for m in MARGINS:
            f.write(json.dumps(m) + "\n")
