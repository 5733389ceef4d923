"""The oracle against the stored golden fixtures of tests/golden/: exact rational results
of the plain definitions (Eq. 14 / Eq. 15 of section 3.3 and the conv of section 3.4),
written by tests/golden/make_golden.py with Python fractions.  The paper prints no worked
example, so these are the closest stored values: computed outside the oracle and
outside the CUDA path, from the definitions alone."""
import json
import os
from fractions import Fraction

import numpy as np

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f(x):
    return float(Fraction(x))


def _arr(m):
    return np.array([[_f(x) for x in row] for row in m], dtype=np.float64)


def test_kda_exact_fixture():
    d = json.load(open(os.path.join(GOLD, "kda_exact.json")))
    alpha, k, q, v = _arr(d["alpha"]), _arr(d["k"]), _arr(d["q"]), _arr(d["v"])
    T, dk = alpha.shape
    dv = v.shape[1]
    beta = np.array([_f(b) for b in d["beta"]])
    o, ST = O.kda_forward(q.reshape(1, T, 1, dk), k.reshape(1, T, 1, dk), v.reshape(1, T, 1, dv),
                          np.log(alpha).reshape(1, T, 1, dk), beta.reshape(1, T, 1),
                          _arr(d["S0"]).reshape(1, 1, dk, dv))
    o_ref, S_ref = _arr(d["o"]), _arr(d["S_T"])
    assert np.abs(o[0, :, 0] - o_ref).max() <= 1e-13 * np.abs(o_ref).max()
    assert np.abs(ST[0, 0] - S_ref).max() <= 1e-13 * np.abs(S_ref).max()


def test_conv_exact_fixture():
    d = json.load(open(os.path.join(GOLD, "conv_exact.json")))
    xt, xi, xv = d["text"]["x"], d["image"]["x"], d["video"]["x"]
    flat = xt + [x for row in xi for x in row] + [x for fr in xv for row in fr for x in row]
    T = len(flat)
    x = np.array(flat, dtype=np.float64).reshape(1, T, 1)
    segs = [(O.MOD_TEXT, 0, 1, 1, 5, 0), (O.MOD_IMAGE, 5, 1, 3, 3, 0), (O.MOD_VIDEO, 14, 2, 2, 2, 0)]
    wt = np.array(d["text"]["w"], dtype=np.float32).reshape(1, 1, 4)
    wi = np.array(d["image"]["w"], dtype=np.float32).reshape(1, 1, 3, 3)
    wv = np.array(d["video"]["w"], dtype=np.float32).reshape(1, 1, 3, 3, 3)
    y = O.mshortconv(x, segs, 4, wt, wi, wv)[0, :, 0]
    want = d["text"]["y"] + [v for row in d["image"]["y"] for v in row] + \
        [v for fr in d["video"]["y"] for row in fr for v in row]
    assert np.array_equal(y, np.array(want, dtype=np.float64))
