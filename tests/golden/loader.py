"""Reads the small text fixtures in this folder (``key v1 v2 ...`` lines, ``#`` comments)."""
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(_HERE, name), encoding="utf-8") as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = np.array([float(v) for v in vals])
    return out
