"""The FMA-pipe exp2 (Cody-Waite split + Remez cubic) meets its stated bound.

The coefficients come from chunk_causal_dit_b200/csrc/exp2_poly.h (written by
gen_exp2_poly.py).  Here the kernel's float32 steps are replayed in numpy:
j = round(x) via the 1.5*2^23 shift, f = x - j, Horner in float32, scale by 2^j;
the result is compared with exp2 in float64 over x in [-126, 8], the range the
softmax feeds it (scores minus a running maximum that is at most 2^8 stale).
The attention kernel sends a third of the exponential pairs through this path
(the rest through MUFU ex2.approx); this checks its error bound.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "chunk_causal_dit_b200", "csrc", "exp2_poly.h")


def coeffs():
    text = open(HDR).read()
    c = [float(m) for m in re.findall(r"kExp2C\d = ([-0-9.e]+)f;", text)]
    bound = float(re.search(r"kExp2PolyRelErr = ([-0-9.e]+)f;", text).group(1))
    return np.array(c, np.float32), bound


def exp2_fma_f32(x):
    c0, c1, c2, c3 = coeffs()[0]
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    jf = (t - shift).astype(np.float32)
    f = (x - jf).astype(np.float32)
    q = np.float32(c3)
    q = (q * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_bound_is_consistent_with_degree():
    c, bound = coeffs()
    assert len(c) == 4 and 1e-5 < bound < 1e-4   # a cubic on [-1/2, 1/2]


def test_relative_error_over_softmax_range():
    _, bound = coeffs()
    # above -125 the result is a normal float; at the clamp (x <= -126) the
    # kernel only promises a tiny positive value (next test)
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001),
                        np.arange(-125, 8, dtype=np.float64) + 0.5])   # rounding ties
    x = x.astype(np.float32)
    got = exp2_fma_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    # float32 Horner adds a few ulps (2^-24 each) on top of the minimax bound
    assert rel.max() <= bound + 8 * 2.0 ** -24


def test_clamp_below_range():
    got = exp2_fma_f32(np.array([-200.0, -np.inf], np.float32))
    assert np.all(got > 0) and np.all(got < 2.0 ** -125)   # tiny, never wraps sign
