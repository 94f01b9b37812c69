import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def read_golden(name):
    """Lines of a golden fixture with comments and blank lines removed."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.rstrip("\n") for ln in f if ln.strip() and not ln.startswith("#")]


def parse_segments(line):
    # "segments 0 2 0 | 2 3 1 | ..."
    body = line.split(None, 1)[1]
    return [tuple(int(x) for x in part.split()) for part in body.split("|")]
