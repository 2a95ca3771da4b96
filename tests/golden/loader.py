"""Reads the hand-derived worked examples in ``worked_examples.txt``."""

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _parse_matrix(text):
    rows = [r.split() for r in text.split(";")]
    return np.array([[float(x) for x in r] for r in rows], dtype=np.float64)


def load_worked_examples(path=None):
    path = path or os.path.join(HERE, "worked_examples.txt")
    cases = {}
    cur = None
    with open(path) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("["):
                cur = {}
                cases[line.strip("[]")] = cur
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            if key == "scale":
                cur[key] = float(val)
            elif key in ("k", "v"):
                cur[key] = _parse_matrix(val)
            else:
                cur[key] = np.array([float(x) for x in val.split()], dtype=np.float64)
    return cases
