import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


GOLDEN = os.path.join(ROOT, "tests", "golden")


def load_mask_fixture(name):
    """Returns ((T, c, F, tf), rows as a list of lists of 0/1)."""
    lines = [l.strip() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]
    desc = tuple(int(x) for x in lines[0].split())
    mat = [[int(ch) for ch in l] for l in lines[1:]]
    return desc, mat
