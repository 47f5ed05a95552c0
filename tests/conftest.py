import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a golden fixture: '#' lines are comments; 'key v1 v2 ...' header lines
    become a dict entry; purely numeric lines become rows."""
    header, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            try:
                rows.append([float(x) if "." in x else int(x) for x in parts])
            except ValueError:
                vals = [float(x) if "." in x else int(x) for x in parts[1:]]
                header[parts[0]] = vals[0] if len(vals) == 1 else vals
    return header, rows


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import oracle
    return oracle.lib()
