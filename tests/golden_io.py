"""Readers for the hand-derived text fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                yield k.strip(), v.strip()


def _nums(v, dtype=float):
    return np.array([dtype(x) for x in v.split()])


def _rows(v, dtype=float):
    return [np.array([dtype(x) for x in part.split()]) for part in v.split("|")]


def read_kv(name):
    return dict(_lines(name))


def read_cases(name):
    cases, cur = [], None
    for k, v in _lines(name):
        if k == "case":
            cur = {"case": v}
            cases.append(cur)
        else:
            cur[k] = v
    return cases


nums, rows = _nums, _rows
