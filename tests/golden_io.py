"""Parser for the hand-worked fixtures under tests/golden/ (plain text)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _mat(text):
    rows = [r.split() for r in text.split("|")]
    return np.array([[float(x) for x in r] for r in rows], dtype=np.float64)


def load(name):
    """Returns (inputs: dict of 2-D arrays, cases: list of (gamma, expected dict))."""
    inputs, cases, cur = {}, [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case "):
                cur = {}
                cases.append((float(line.split("=", 1)[1]), cur))
                continue
            key, val = line.split(":", 1)
            (cur if cur is not None else inputs)[key.strip()] = _mat(val)
    return inputs, cases
