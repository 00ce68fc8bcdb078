import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


def read_golden(name):
    """Parse a golden fixture: '#' lines are citations/comments, every other
    line is 'key value...'.  Returns {key: [tokens...]}, with repeated keys
    (e.g. 'table') collected in order under key -> list of token lists."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            out.setdefault(key, []).append(rest)
    return out
