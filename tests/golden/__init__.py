"""Text fixtures with their citations; `load(name)` parses one."""
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(_HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            arr = np.array([float(v) for v in vals])
            out[key] = int(arr[0]) if key in ("N", "H") else arr
    return out
