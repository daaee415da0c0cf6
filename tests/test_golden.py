"""The oracle reproduces its stored fixture (tests/golden/tiny_wave.txt).

The fixture was written by tests/golden/make_golden.py from the oracle alone;
this guards the oracle against unreviewed drift.
"""
import os

import numpy as np

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_fixture():
    qk, o = {}, {}
    with open(os.path.join(HERE, "tiny_wave.txt")) as f:
        for line in f:
            if line.startswith("#"):
                continue
            p = line.split()
            if p[0] == "qk":
                qk[(int(p[1]), int(p[2]))] = (
                    np.array([int(b, 16) for b in p[3].split(",")], np.uint16),
                    np.array([int(b, 16) for b in p[4].split(",")], np.uint16))
            elif p[0] == "o":
                o[(int(p[1]), int(p[2]))] = (float(p[3]),
                                             np.array([float(t) for t in p[4].split(",")]))
    return qk, o


def test_oracle_reproduces_fixture():
    import sys
    sys.path.insert(0, HERE)
    import make_golden
    w, qo, ko, rows, heads, o, lse = make_golden.compute()
    qk, fo = load_fixture()
    for (n, h), (q_bits, k_bits) in qk.items():
        assert np.array_equal(qo[n, h], q_bits) and np.array_equal(ko[n, h], k_bits)
    for i in range(len(rows)):
        l0, o0 = fo[(int(rows[i]), int(heads[i]))]
        assert abs(lse[i] - l0) <= 1e-13
        assert np.allclose(o[i], o0, rtol=0, atol=1e-14)
