"""Reader for the small text fixtures under tests/golden/.

Format: '#' lines are the citation; every other line is ``name = values``;
values are whitespace-separated numbers, rows separated by ';'.
"""

from __future__ import annotations

import os

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(__file__), "golden")


def _num(tok):
    try:
        return int(tok)
    except ValueError:
        return float(tok)


def load(name):
    out = {}
    with open(os.path.join(GOLDEN_DIR, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            if ";" in val:
                out[key] = np.array([[_num(t) for t in row.split()] for row in val.split(";")])
            else:
                toks = val.split()
                out[key] = _num(toks[0]) if len(toks) == 1 else np.array([_num(t) for t in toks])
    return out
