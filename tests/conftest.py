import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    # Build libpa_b200.so in-tree if its sources changed (no-op otherwise).
    from paged_kv_cache_356_b200 import build
    build.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a); run with -m gpu")
    config.addinivalue_line("markers", "slow: full-size workload on the GPU")


def load_golden(name):
    """Parse a tests/golden fixture: '# ...' comment lines, then 'key value...' lines."""
    path = os.path.join(ROOT, "tests", "golden", name)
    fields, rows = {}, []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "block":
                rows.append(tuple(int(v) for v in vals))
            else:
                v = vals[0]
                fields[key] = float(v) if "." in v else int(v)
    fields["blocks"] = rows
    return fields


@pytest.fixture
def golden():
    return load_golden
