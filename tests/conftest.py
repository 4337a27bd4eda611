import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libmedusa.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def read_golden(name):
    """Parse a golden fixture: 'key: value' lines, '#' comments, and a block
    of rows after a 'key:' line with an empty value."""
    out = {}
    cur = None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.rstrip("\n")
            if not line.strip() or line.lstrip().startswith("#"):
                continue
            if ":" in line and not line[0].isdigit() and not line.startswith("-"):
                k, v = line.split(":", 1)
                k = k.strip()
                v = v.strip()
                if v:
                    out[k] = v
                    cur = None
                else:
                    out[k] = []
                    cur = k
            elif cur is not None:
                out[cur].append(line.strip())
            else:
                out.setdefault("_rows", []).append(line.strip())
    return out


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False
