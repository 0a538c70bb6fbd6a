"""Reader for the hand-worked fixtures under tests/golden/.

Format: '#' comments; 'name = value' lines; matrices use ';' between rows;
entries may be fractions 'a/b' or 'ln3'.
"""
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(tok: str) -> float:
    if tok == "ln3":
        return math.log(3.0)
    return float(Fraction(tok))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            rows = [r.split() for r in val.split(";")]
            arr = np.array([[_num(t) for t in r] for r in rows], dtype=np.float64)
            if arr.shape[0] == 1:
                arr = arr[0]
                if arr.shape[0] == 1:
                    arr = arr[0]
            out[key] = arr
    return out
