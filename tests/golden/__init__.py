"""Readers for the golden fixtures: values printed on the pages, each file citing its source."""
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _lines(name):
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def read_band(name):
    """Returns (T, W, mask) where mask[i, j] is True when query i may attend key j."""
    T = W = None
    rows = []
    for tok in _lines(name):
        if tok[0] == "T":
            T = int(tok[1])
        elif tok[0] == "W":
            W = int(tok[1])
        else:
            rows.append([t in ("1", ".") for t in tok])
    mask = np.array(rows, dtype=bool)
    assert mask.shape == (T, T)
    return T, W, mask


def read_moving_average(name="nnx_moving_average.txt"):
    """Returns dict with W, x [T,2], y [T,2], changed_row (index, values), unchanged_from."""
    out = {"x": [], "y": []}
    for tok in _lines(name):
        if tok[0] == "W":
            out["W"] = int(tok[1])
        elif tok[0] in ("x", "y"):
            out[tok[0]].append([float(t) for t in tok[1:]])
        elif tok[0] == "changed_row":
            out["changed_row"] = (int(tok[1]), [float(t) for t in tok[2:]])
        elif tok[0] == "unchanged_from":
            out["unchanged_from"] = int(tok[1])
    out["x"] = np.array(out["x"])
    out["y"] = np.array(out["y"])
    return out
