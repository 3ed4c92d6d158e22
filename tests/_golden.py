"""Readers for the text fixtures under tests/golden (each fixture cites its source)."""
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def _val(tok: str) -> float:
    if tok == "nan":
        return math.nan
    return float.fromhex(tok) if "0x" in tok else float(tok)


def e2m1_table() -> np.ndarray:
    """16 E2M1 values indexed by code (OCP MX v1.0)."""
    t = np.zeros(16)
    for code, v in _rows("e2m1_values.txt"):
        t[int(code)] = float(v)
    return t


def e8m0_points():
    return [(int(e), _val(v)) for e, v in _rows("e8m0_values.txt")]


def e4m3_points():
    return [(int(c, 16), _val(v)) for c, v in _rows("e4m3_values.txt")]


def kv(name):
    return {k: int(v) for k, v in _rows(name)}
