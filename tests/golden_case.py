"""Loader of the worked example in tests/golden/ (hand-derived exact answers).

Entries are numbers, "ln X" (natural log of X) or "a/b" (a fraction); the
loader turns them into float64. It holds no attention arithmetic."""

import json
import math
import os
from fractions import Fraction

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
PATH = os.path.join(HERE, "golden", "paged_attention_worked_example.json")


def value(x):
    if isinstance(x, (int, float)):
        return float(x)
    s = x.strip()
    if s.startswith("ln "):
        return math.log(float(s[3:]))
    return float(Fraction(s))


def array(xs):
    if isinstance(xs, list):
        return np.array([array(x) for x in xs], dtype=np.float64)
    return value(xs)


def load():
    with open(PATH) as f:
        g = json.load(f)
    shape = (g["num_blocks"], g["num_kv_heads"], g["block_size"], g["head_dim"])
    k = np.full(shape, g["sentinel"], dtype=np.float64)
    v = np.full(shape, g["sentinel"], dtype=np.float64)
    for r in g["rows"]:
        k[r["block"], :, r["row"], :] = array(r["k"])
        v[r["block"], :, r["row"], :] = array(r["v"])
    return g, k, v
