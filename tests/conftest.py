import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def load_golden(name):
    """Parse a tests/golden/*.txt fixture: '#' comments, 'key v v v' lines and
    bare numeric rows collected under the last bare key."""
    path = os.path.join(ROOT, "tests", "golden", name)
    out, cur = {}, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0][0].isalpha():
                key, vals = parts[0], parts[1:]
                if vals:
                    out[key] = [int(v) for v in vals]
                    cur = None
                else:
                    out[key] = []
                    cur = key
            else:
                out[cur].append([int(v) for v in parts])
    return out


@pytest.fixture
def golden():
    return load_golden
