"""Parser for the hand-worked text fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    """Return {key: [list of float rows]} for a fixture file."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            out.setdefault(key, []).append([float(v) for v in vals])
    return out


def scalar(fx, key):
    return fx[key][0][0]


def matrix(fx, key):
    return np.array(fx[key], dtype=np.float64)
