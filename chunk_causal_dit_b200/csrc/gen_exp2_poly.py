"""Fit the FMA-pipe exp2 polynomial used by the attention kernel and write exp2_poly.h.

    python chunk_causal_dit_b200/csrc/gen_exp2_poly.py

Method (Cody-Waite split + Remez): 2^x = 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2].  2^f is approximated by the degree-N polynomial that
minimises the maximum RELATIVE error on [-1/2, 1/2], found with the Remez
exchange algorithm (equioscillation of p(f)/2^f - 1 at N+2 points).  The
coefficients are then rounded to float32 and the error re-measured on a dense
grid in float64; the header records that bound.  Everything here is derived
from the definition of 2^f; no library exp constants are used.
"""
from __future__ import annotations

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(deg: int, iters: int = 60):
    n = deg + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i   for coefficients c_0..c_deg and E
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign run
        s = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(s))[0] + 1, [len(grid)]))
        ext = [a + int(np.argmax(np.abs(err[a:b]))) for a, b in zip(idx[:-1], idx[1:])]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitudes
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x_new = grid[ext]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    return c


def measured_bound(c32):
    grid = np.linspace(LO, HI, 2000001)
    p = np.zeros_like(grid)
    for cc in c32[::-1]:               # Horner in float64 on the float32 coefficients
        p = p * grid + float(cc)
    return float(np.max(np.abs(p / 2.0 ** grid - 1.0)))


def main(path=os.path.join(HERE, "exp2_poly.h")):
    c = remez_relative(DEGREE)
    c32 = np.asarray(c, np.float32)
    bound = measured_bound(c32)
    lines = [
        "// exp2_poly.h -- written by gen_exp2_poly.py; do not edit by hand.",
        "// 2^f on [-1/2, 1/2] by a degree-%d polynomial, minimax in relative error" % DEGREE,
        "// (Remez exchange), coefficients rounded to float32.",
        "// Max relative error on [-1/2, 1/2] with float32 coefficients: %.3e" % bound,
        "#pragma once",
        "namespace wf {",
        "constexpr int kExp2PolyDegree = %d;" % DEGREE,
        "constexpr float kExp2PolyRelErr = %.9ef;" % bound,
    ]
    for i, v in enumerate(c32):
        lines.append("constexpr float kExp2C%d = %sf;" % (i, repr(float(v))))
    lines.append("}  // namespace wf")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")
    print("degree %d, max rel err %.3e -> %s" % (DEGREE, bound, path), file=sys.stderr)
    return c32, bound


if __name__ == "__main__":
    main()
