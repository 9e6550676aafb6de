"""Reader for the small text fixtures under tests/golden/ ('key = row ; row' lines)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (p.strip() for p in line.split("=", 1))
            rows = [[float(t) for t in r.split()] for r in val.split(";")]
            a = np.array(rows, np.float64)
            if a.size == 1:
                out[key] = float(a[0, 0])
            else:
                out[key] = a[0] if a.shape[0] == 1 else a
    return out
