import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


GOLDEN = os.path.join(ROOT, "tests", "golden")


def read_golden(name):
    """Parse a golden fixture: 'key: values' lines grouped into 'case:' ... 'end' blocks."""
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            key = key.strip()
            val = val.strip()
            if key == "case":
                cur = {"case": val}
            elif key == "end":
                cases.append(cur)
                cur = None
            else:
                cur[key] = val
    return cases


def ints(s):
    return [int(v) for v in s.replace("|", " ").split()]


def floats(s):
    return [float(v) for v in s.split()]
