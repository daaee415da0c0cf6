"""Helpers shared by the GPU parity tests: device set-up of one wave round and
the comparison rules.  The oracle side sees only bf16 bit patterns."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from chunk_causal_dit_b200 import inputs as wi

# Attention parity bar on unit-scale data (fp32 accumulation, bf16 output).
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3


def bf16_quantum(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (normal range)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def pair_norm(f64: np.ndarray) -> np.ndarray:
    """|(y_2i, y_2i+1)| of every RoPE pair, repeated onto both members."""
    n = np.hypot(f64[..., 0::2], f64[..., 1::2])
    return np.repeat(n, 2, axis=-1)


def assert_within_one_ulp(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str,
                          ref_f64: np.ndarray = None):
    """GPU bf16 vs the oracle's RNE bf16: at most one bf16 quantum apart.

    With ref_f64 (the oracle's unrounded values) the bar adds the fp32 error of
    the GPU's rotation, 2^-20 * |pair|: x0*cos - x1*sin carries an absolute
    error of a few fp32 ulps of |pair|, which exceeds a bf16 quantum when the
    two products nearly cancel."""
    g = wi.from_bits(gpu_bits).double().numpy()
    r = wi.from_bits(ref_bits).double().numpy()
    diff = np.abs(g - r)
    tol = bf16_quantum(r) * 1.0000001
    if ref_f64 is not None:
        tol = tol + 2.0 ** -20 * pair_norm(ref_f64)
    bad = diff > tol
    assert not bad.any(), "%s: %d of %d values differ by more than 1 bf16 ulp (max %g)" % (
        what, int(bad.sum()), bad.size, float(diff.max()))
    return float((gpu_bits != ref_bits).mean())


def assert_attention_close(o_gpu: np.ndarray, o_ref: np.ndarray, what: str):
    d = np.abs(o_gpu.astype(np.float64) - o_ref)
    mx, mean = float(d.max()), float(d.mean())
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, \
        "%s: max abs %.3g (bar %g), mean abs %.3g (bar %g)" % (what, mx, ATTN_MAX_ABS, mean,
                                                            ATTN_MEAN_ABS)
    return mx, mean


def assert_attention_within_rounding(o_gpu: np.ndarray, o_ref: np.ndarray, v_absmax: float,
                                     what: str):
    """Elementwise bound for rows that see very few keys, where rounding errors
    do not average out: P is rounded to bf16 before the PV product (relative
    error <= 2^-9 per weight, so <= 2^-9 * max|V| on O) and O is rounded to
    bf16 once (<= 2^-9 * |O|); 2^-8 leaves room for the fp32 sums."""
    d = np.abs(o_gpu.astype(np.float64) - o_ref)
    bound = 2.0 ** -8 * (v_absmax + np.abs(o_ref)) + 1e-6
    assert np.all(d <= bound), "%s: %d values exceed the rounding bound (worst excess %.3g)" % (
        what, int((d > bound).sum()), float((d - bound).max()))


def assert_attention_close_scaled(o_gpu: np.ndarray, o_ref: np.ndarray, v_absmax: float,
                                  what: str):
    """The 1e-2 / 1e-3 bar on unit-scale outputs, a relative bar above them.

    Elements with |O| <= 1 must be within ATTN_MAX_ABS, and all elements
    together within ATTN_MEAN_ABS on average.  Elements with |O| > 1 (a row
    pulled onto one large V row) are held to the rounding bound of
    assert_attention_within_rounding instead: there one bf16 rounding of O
    alone can exceed 1e-2."""
    d = np.abs(o_gpu.astype(np.float64) - o_ref)
    unit = np.abs(o_ref) <= 1.0
    if unit.any():
        mx = float(d[unit].max())
        assert mx <= ATTN_MAX_ABS, "%s: max abs %.3g on |O| <= 1 (bar %g)" % (what, mx,
                                                                             ATTN_MAX_ABS)
    if (~unit).any():
        assert_attention_within_rounding(o_gpu[~unit], o_ref[~unit], v_absmax,
                                         what + " (|O| > 1)")
    assert float(d.mean()) <= ATTN_MEAN_ABS, "%s: mean abs %.3g (bar %g)" % (
        what, float(d.mean()), ATTN_MEAN_ABS)


def rand_bf16(shape, seed, device="cuda"):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(device)


def sample_rows(L: int, W: int, n_random: int, seed: int):
    """Wave rows at chunk and 128-row tile boundaries plus seeded random rows."""
    rows = set()
    for c in range(W):
        base = c * L
        for r in (0, 1, L - 2, L - 1):
            rows.add(base + r)
        for t in range(128, L, 128):
            rows.update((base + t - 1, base + t))
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, W * L, n_random))
    return np.array(sorted(r for r in rows if 0 <= r < W * L), np.int64)


def oracle_rows(cache: "oracle.OracleCache", round_, W, Hh, q_bits, rows, heads):
    o, lse = oracle.round_attention(cache, round_, W, Hh, q_bits, rows, heads)
    return o, lse
