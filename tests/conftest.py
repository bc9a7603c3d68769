import os
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: `key: numbers` lines; ';' separates rows."""
    import numpy as np

    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            rows = [[float(v) for v in r.split()] for r in val.split(";")]
            out[key.strip()] = np.array(rows if len(rows) > 1 else rows[0], dtype=np.float64)
    return out
