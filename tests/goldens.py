"""Reader for the hand-derived fixtures under tests/golden/ (blocks of `key: value` lines)."""
import math
import os

import numpy as np

_NS = {"ln": math.log, "exp": math.exp, "inf": math.inf, "nan": math.nan, "__builtins__": {}}


def _num(expr: str) -> float:
    return float(eval(expr.strip(), _NS))  # fixtures are trusted test data, not user input


def nums(s: str):
    return [_num(x) for x in s.split(",") if x.strip()]


def rows(s: str):
    """'a, b | c, d' -> 2-D array (rows separated by '|')."""
    return np.array([nums(r) for r in s.split("|")], dtype=np.float64)


def load(name: str):
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    blocks, cur = [], {}
    with open(path) as f:
        for line in f:
            line = line.rstrip("\n")
            if not line.strip():
                if cur:
                    blocks.append(cur)
                    cur = {}
                continue
            if line.lstrip().startswith("#"):
                continue
            k, _, v = line.partition(":")
            cur[k.strip()] = v.strip()
    if cur:
        blocks.append(cur)
    return blocks
