"""Pins for the oracle's E4M3 codec, its quantization rule and its FP8-Q.K attention.

E4M3 (the 8-bit float with 4 exponent bits, bias 7, 3 mantissa bits, no
infinities, S.1111.111 = NaN, largest finite 448) is pinned to values the
format definition fixes, to round trips, to ties-to-even at several binades and
to PyTorch's own float8_e4m3fn cast (an independent library implementation) on
in-range inputs.  The FP8 attention route is pinned to the bf16 oracle on inputs
whose quantization is exact up to fp32 scale rounding, with a different scale in
every key tile and head, so a scale read from the wrong tile, head or row fails.
"""
import numpy as np
import pytest
import torch

import oracle


def test_e4m3_published_values():
    codes = np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0x3C, 0x40, 0x77, 0x7E, 0xFE],
                     np.uint8)
    want = [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.5, 2.0, 240.0, 448.0, -448.0]
    got = oracle.e4m3_decode(codes)
    assert list(got) == want
    assert np.signbit(got[1])
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_round_trip_and_order():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals)
    assert np.array_equal(back, codes)
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)           # strictly increasing over the finite codes


def test_e4m3_ties_to_even_and_saturation():
    cases = {
        1.0 + 1 / 16: 0x38,             # midway 1.0 / 1.125 -> even mantissa 0
        1.0 + 3 / 16: 0x3A,             # midway 1.125 / 1.25 -> even mantissa 2
        2.0 ** -10: 0x00,               # midway 0 / 2^-9 -> 0
        3 * 2.0 ** -10: 0x02,           # midway 1 / 2 (x 2^-9) -> 2
        2.0 ** -6 - 2.0 ** -10: 0x08,   # midway largest subnormal / smallest normal -> normal (even)
        232.0: 0x76,                    # midway 224 / 240 -> 224 (mantissa 6)
        448.0: 0x7E, 463.9: 0x7E, 464.0: 0x7E, 1e6: 0x7E,   # saturation
        -1e6: 0xFE,
    }
    x = np.array(list(cases.keys()))
    assert list(oracle.e4m3_encode(x)) == list(cases.values())


def test_e4m3_matches_library_cast():
    g = np.random.default_rng(7)
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.uniform(-4, 2.5, 20000),
                        g.uniform(-447.9, 447.9, 5000)]).astype(np.float32)
    x = x[np.abs(x) < 448.0]              # the library cast does not saturate; compare in range
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(ours, lib)


def test_quantize_rows_rule_and_error_bound():
    g = np.random.default_rng(3)
    x = (g.standard_normal((50, 3, 64)) * 10.0 ** g.uniform(-3, 3, (50, 3, 1))).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)       # truncate to bf16
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    codes, scale = oracle.quantize_rows_fp8(bits)
    assert scale.shape == (3, 50) and scale.dtype == np.float32
    amax = np.abs(x).max(axis=2)
    assert np.array_equal(scale.T, (amax / np.float32(448.0)).astype(np.float32))
    # codes are E4M3 of the fp32 product x * (448 / amax)
    inv = (np.float32(448.0) / amax).astype(np.float32)
    want = oracle.e4m3_encode((x * inv[..., None]).astype(np.float32).astype(np.float64))
    assert np.array_equal(codes, want)
    # the largest magnitude of every row lands on the largest code
    top = np.take_along_axis(codes & 0x7F, np.abs(x).argmax(axis=2)[..., None], axis=2)
    assert (top == 0x7E).all()
    deq = oracle.e4m3_decode(codes) * scale.T[..., None]
    err = np.abs(deq - x)
    # half a unit in the last place: 2^-4 relative in the normal range, 2^-10 * scale below it
    # (plus the fp32 roundings of 448 / amax, of the product and of amax / 448)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scale.T[..., None] * 2.0 ** -10) * (1 + 1e-6) + \
        np.abs(x) * 2.0 ** -21
    assert (err <= bound).all()


def test_quantize_tiles_scales_per_tile_and_head():
    g = np.random.default_rng(4)
    L, H, D = 300, 2, 16
    x = g.standard_normal((L, H, D)).astype(np.float32)
    x[128:256, 1] *= 50.0                 # tile 1 of head 1 is larger
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = oracle.quantize_tiles_fp8(bits)
    assert scales.shape == (3, H)
    xs = (bits.astype(np.uint32) << 16).view(np.float32)
    for t in range(3):
        sl = slice(128 * t, min(L, 128 * (t + 1)))
        for h in range(H):
            assert scales[t, h] == np.float32(np.abs(xs[sl, h]).max()) / np.float32(448.0)
    assert scales[1, 1] > 20 * scales[1, 0]
    zero = np.zeros((5, 1, 8), np.uint16)
    c0, s0 = oracle.quantize_tiles_fp8(zero)
    assert (c0 == 0).all() and (s0 == 1.0).all()


def _pow2_bits(g, shape, exps):
    """bf16 bits of +-2^e with e drawn from `exps` (exactly representable in E4M3
    after scaling by a power-of-two ratio of the group maximum)."""
    e = g.choice(exps, size=shape)
    sgn = g.choice([-1.0, 1.0], size=shape)
    x = (sgn * np.exp2(e)).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("L,W,Hh,H,D,r", [(150, 3, 1, 2, 32, 2), (260, 2, 2, 3, 16, 5)])
def test_fp8qk_attention_equals_bf16_route_on_exact_inputs(L, W, Hh, H, D, r):
    g = np.random.default_rng(L + D)
    R = W + Hh
    q = _pow2_bits(g, (W * L, H, D), [-3, -2, -1, 0])
    ks = [_pow2_bits(g, (L, H, D), [-4, -3, -2]) for _ in range(R)]
    # give every key tile and head its own range, so every tile scale differs
    for b in range(R):
        kk = (ks[b].astype(np.uint32) << 16).view(np.float32).copy()
        for t in range((L + 127) // 128):
            for h in range(H):
                kk[128 * t:128 * (t + 1), h] *= 2.0 ** ((b + 2 * t + 3 * h) % 5)
        ks[b] = (kk.view(np.uint32) >> 16).astype(np.uint16)
    vs = [(g.standard_normal((L, H, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
          for _ in range(R)]
    cache = oracle.OracleCache(L)
    cache8 = oracle.OracleCacheFP8(L)
    for gid in range(r - min(Hh, r), r + W):
        cache.put(gid, ks[gid % R], vs[gid % R])
        cache8.put_bf16(gid, ks[gid % R], vs[gid % R])
    q8, qs = oracle.quantize_rows_fp8(q)
    rows = np.repeat(np.arange(W * L), H)
    heads = np.tile(np.arange(H), W * L)
    ref, lse_ref = oracle.round_attention(cache, r, W, Hh, q, rows, heads)
    got, lse = oracle.round_attention_fp8qk(cache8, r, W, Hh, q8, qs, rows, heads)
    # quantization is exact here up to the fp32 rounding of each scale (2^-24 relative)
    assert np.max(np.abs(got - ref)) < 1e-5
    assert np.max(np.abs(lse - lse_ref)) < 1e-5
