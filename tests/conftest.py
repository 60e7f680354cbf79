import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


def read_golden(name):
    """Non-comment lines of a fixture under tests/golden/."""
    path = os.path.join(ROOT, "tests", "golden", name)
    with open(path) as f:
        return [l.split("#")[0].strip() for l in f if l.split("#")[0].strip()]
