import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def load_golden(name: str) -> dict:
    """Parse tests/golden/<name>: `key = value  # citation` lines."""
    out = {}
    path = os.path.join(ROOT, "tests", "golden", name)
    with open(path) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            parts = [float(v) for v in val.split(",")]
            out[key] = parts[0] if len(parts) == 1 else tuple(parts)
    return out


@pytest.fixture(scope="session")
def golden():
    return load_golden("worked_example.txt")
