"""Readers for the hand-written fixtures under tests/golden/ (plain text)."""

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln.split()


def code_table(name):
    """[(code, value)] from a 'code value' fixture."""
    return [(int(c, 16), float(v)) for c, v in _lines(name)]


def rounding_cases():
    return [(fmt, np.float32(float(x)), int(c, 16)) for fmt, x, c in _lines("rounding_cases.txt")]


def keyed(name):
    d = {}
    for parts in _lines(name):
        d[parts[0]] = parts[1:]
    return d
