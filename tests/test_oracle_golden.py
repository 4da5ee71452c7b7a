"""Pins the oracle to the hand-worked example in tests/golden (every number
there was derived by hand from the pages' equations)."""
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_layer.txt")


def _parse():
    d = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = v.split()
    return d


def _num(tok, sc1):
    if tok.endswith("*sc1"):
        return float(np.float32(float(tok[:-4]) * sc1))
    if "/" in tok:
        a, b = tok.split("/")
        return float(Fraction(a) / Fraction(b))
    return float(Fraction(tok))


def test_hand_worked_layer():
    d = _parse()
    K, G = int(d["K"][0]), int(d["G"][0])
    sc1 = 1101 / 131072   # FP16 0x204D, see the fixture's derivation
    W = np.array([[_num(t, sc1) for t in d["W0"]], [_num(t, sc1) for t in d["W1"]]], np.float32)
    X = np.array([[float(t) for t in d["X0"]]], np.float16)
    r = oracle.linear(X, W, G)
    ints = lambda key: [int(t, 0) for t in d[key]]
    assert list(r["s_c"]) == ints("s_c_bits")
    assert list(r["W8"][0]) == ints("W8_0") and list(r["W8"][1]) == ints("W8_1")
    assert list(r["s_g"].ravel()) == ints("s_g")
    assert list(r["z"].ravel()) == ints("z")
    assert list(r["zs"].ravel()) == ints("zs")
    assert list(r["q"][0]) == ints("q_0") and list(r["q"][1]) == ints("q_1")
    assert list(r["W8hat"][0]) == ints("W8hat_0") and list(r["W8hat"][1]) == ints("W8hat_1")
    assert list(r["s_x"]) == ints("s_x_bits")
    assert list(r["X8"][0]) == ints("X8_0")
    assert list(r["acc"][0]) == ints("acc")
    assert list(r["Y"][0]) == ints("Y_bits")
    assert K == W.shape[1]
