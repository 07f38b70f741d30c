import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes of oracle time)")


def read_golden(name):
    """Parse a golden fixture: 'key: v v v' lines and 'key:' followed by a matrix block."""
    out, key, rows = {}, None, []
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].rstrip()
            if not line.strip():
                continue
            if ":" in line:
                if key is not None and rows:
                    out[key] = rows
                k, v = line.split(":", 1)
                key, rows = k.strip(), []
                if v.strip():
                    out[key] = [float(t) for t in v.split()]
                    key = None
            else:
                rows.append([float(t) for t in line.split()])
    if key is not None and rows:
        out[key] = rows
    return out


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle
