"""Reader for the hand-worked fixtures under tests/golden (text, '#' comments)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    out = {}
    multi = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            key, val = key.strip(), val.strip()
            if key in out:
                multi.setdefault(key, [out[key]]).append(val)
            out[key] = val
    for k, v in multi.items():
        out[k] = v
    return out


def mat(s, dtype=np.float64):
    """'1 2 | 3 4' -> [[1, 2], [3, 4]]; '1 2' -> [1, 2]."""
    if "|" in s:
        return np.array([[float(x) for x in row.split()] for row in s.split("|")], dtype=dtype)
    return np.array([float(x) for x in s.split()], dtype=dtype)


def ints(s):
    return [int(x) for x in s.split()] if s.strip() else []
