import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built liblfm3.so")
    config.addinivalue_line("markers", "slow: long CPU-side oracle work")


def read_golden(name):
    """key = value lines of a tests/golden fixture (comments after '#')."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = (t.strip() for t in line.split("=", 1))
                out[k] = float(v) if any(c in v for c in ".e") else int(v)
    return out
