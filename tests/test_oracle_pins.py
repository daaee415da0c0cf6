"""Pins for the CPU fp64 oracle: every check here comes from outside the oracle.

The pages print no worked example, so the oracle is pinned by IEEE definitions
(hand-derived bf16 rounding cases), library routines on special cases (torch's
float32->bf16 conversion, scaled_dot_product_attention, rms_norm, numpy complex
rotation), a second brute-force route (dense explicit chunk mask) and
invariants of chunk-causal attention stated in the "Wave Forcing" abstract
(later chunks see earlier chunks and their own chunk, never a later one).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import inputs as wi

# ----------------------------------------------------------------------------
# bf16 conversions
# ----------------------------------------------------------------------------

# (value, expected bf16 bits): derived by hand from IEEE 754 round-to-nearest-even
# with 8 significand bits.
RNE_CASES = [
    (1.0, 0x3F80),
    (1.0 + 2.0 ** -8, 0x3F80),                 # halfway 1 .. 1+2^-7 -> even (1.0)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),             # halfway 1+2^-7 .. 1+2^-6 -> even
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),    # just above halfway -> up
    (1.0 + 2.0 ** -8 - 2.0 ** -40, 0x3F80),    # just below halfway -> down
    (-2.5, 0xC020),
    (0.0, 0x0000),
    (-0.0, 0x8000),
    ((2 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),    # largest finite bf16
    ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),    # halfway to 2^128, odd -> up -> inf
    (2.0 ** -133, 0x0001),                     # smallest subnormal
    (2.0 ** -134, 0x0000),                     # halfway 0 .. 2^-133 -> even (0)
    (3 * 2.0 ** -134, 0x0002),                 # halfway 1..2 quanta -> even (2)
    (2.0 ** -126, 0x0080),                     # smallest normal
    (float("inf"), 0x7F80),
    (-float("inf"), 0xFF80),
]


@pytest.mark.parametrize("x,bits", RNE_CASES)
def test_f64_to_bf16_hand_cases(x, bits):
    assert int(oracle.f64_to_bf16(np.array([x]))[0]) == bits


def test_f64_to_bf16_matches_torch_on_float32_values():
    # For float32-representable inputs torch's float32->bf16 (RNE) is a library
    # reference; include values near every rounding boundary.
    g = torch.Generator().manual_seed(123)
    x = torch.randn(200000, generator=g, dtype=torch.float32) * torch.exp2(
        torch.randint(-40, 40, (200000,), generator=g).float())
    u = x.view(torch.int32)
    ties = ((u & ~0xFFFF) | 0x8000).view(torch.float32)   # exact halfway points
    x = torch.cat([x, ties, ties.nextafter(torch.tensor(float("inf")))])
    want = wi.bits(x.to(torch.bfloat16))
    got = oracle.f64_to_bf16(x.double().numpy())
    assert np.array_equal(got, want)


def test_bf16_to_f64_all_patterns():
    pats = np.arange(65536, dtype=np.uint16)
    got = oracle.bf16_to_f64(pats)
    want = wi.from_bits(pats).double().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


# ----------------------------------------------------------------------------
# positions
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("r,W,F,gh,gw", [(0, 3, 2, 4, 4), (7, 5, 3, 3, 5), (2, 1, 1, 2, 3)])
def test_positions_structure(r, W, F, gh, gw):
    pos = oracle.positions(r, W, F, gh, gw)
    L = F * gh * gw
    assert pos.shape == (W * L, 3)
    # independent route: numpy index grids in (chunk, frame, row, col) raster order
    c, f, y, x = np.indices((W, F, gh, gw)).reshape(4, -1)
    assert np.array_equal(pos[:, 1], y) and np.array_equal(pos[:, 2], x)
    # time: F consecutive frames per chunk, chunks consecutive, round r starts at r*F
    t = pos[:, 0].reshape(W, L)
    assert t.min() == r * F and t.max() == (r + W) * F - 1
    assert np.all(np.diff(np.unique(t)) == 1)
    # next round shifts time by exactly F, nothing else
    nxt = oracle.positions(r + 1, W, F, gh, gw)
    assert np.array_equal(nxt - pos, np.tile([F, 0, 0], (W * L, 1)))


# ----------------------------------------------------------------------------
# RMSNorm
# ----------------------------------------------------------------------------

def test_rms_norm_matches_torch_library():
    rng = np.random.default_rng(0)
    for D in (64, 128):
        x = rng.standard_normal(D) * 3.0
        g = 1 + 0.1 * rng.standard_normal(D)
        want = torch.nn.functional.rms_norm(torch.from_numpy(x), (D,), torch.from_numpy(g),
                                            eps=1e-6).numpy()
        assert np.allclose(oracle.rms_norm(x, g, 1e-6), want, rtol=1e-14, atol=1e-14)


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128)
    ones = np.ones(128)
    y = oracle.rms_norm(x, ones, 1e-6)
    ms = np.mean(x * x)
    assert math.isclose(np.sqrt(np.mean(y * y)), math.sqrt(ms / (ms + 1e-6)), rel_tol=1e-14)
    # with eps = 0 the norm is scale invariant exactly up to rounding
    assert np.allclose(oracle.rms_norm(4.0 * x, ones, 0.0), oracle.rms_norm(x, ones, 0.0),
                       rtol=0, atol=1e-14)
    # the gain multiplies channel-wise
    g = np.arange(1, 129, dtype=np.float64)
    assert np.allclose(oracle.rms_norm(x, g, 1e-6), y * g, rtol=1e-14)


# ----------------------------------------------------------------------------
# 3D RoPE
# ----------------------------------------------------------------------------

def _complex_rope(x, pos, split, theta):
    """Independent route: each pair as a complex number times exp(i*pos*omega)."""
    out = np.empty_like(x)
    off = 0
    for a, da in enumerate(split):
        z = x[off:off + da:2] + 1j * x[off + 1:off + da:2]
        omega = theta ** (-np.arange(da // 2) * 2.0 / da)
        z = z * np.exp(1j * pos[a] * omega)
        out[off:off + da:2], out[off + 1:off + da:2] = z.real, z.imag
        off += da
    return out


@pytest.mark.parametrize("D", [64, 128])
def test_rope_matches_complex_rotation(D):
    rng = np.random.default_rng(2)
    split = oracle.default_rope_split(D)
    assert sum(split) == D and all(s % 2 == 0 for s in split)
    for pos in ([0, 0, 0], [5, 3, 7], [1234, 29, 51], [-3, 1, 0]):
        x = rng.standard_normal(D)
        got = oracle.rope_3d(x, pos, split, 10000.0)
        assert np.allclose(got, _complex_rope(x, pos, split, 10000.0), rtol=0, atol=1e-12)


def test_rope_split_and_invariants():
    assert oracle.default_rope_split(128) == (44, 42, 42)
    assert oracle.default_rope_split(64) == (24, 20, 20)
    rng = np.random.default_rng(3)
    D = 128
    x = rng.standard_normal(D)
    # position 0 is the identity
    assert np.array_equal(oracle.rope_3d(x, [0, 0, 0]), x)
    # each pair keeps its length
    y = oracle.rope_3d(x, [17, 4, 9])
    assert np.allclose(np.hypot(y[0::2], y[1::2]), np.hypot(x[0::2], x[1::2]), rtol=1e-14)
    # axis blocks are independent: moving h leaves the t and w blocks untouched
    y2 = oracle.rope_3d(x, [17, 11, 9])
    assert np.array_equal(y[:44], y2[:44]) and np.array_equal(y[86:], y2[86:])
    # pair 0 of each axis turns by exactly pos radians; pair 11 of the t block
    # (width 44) by pos * theta^(-1/2) = pos / 100
    e0 = np.zeros(D)
    e0[0] = 1.0
    r = oracle.rope_3d(e0, [3, 0, 0])
    assert math.isclose(r[0], math.cos(3.0), abs_tol=1e-15)
    assert math.isclose(r[1], math.sin(3.0), abs_tol=1e-15)
    e22 = np.zeros(D)
    e22[22] = 1.0
    r = oracle.rope_3d(e22, [50, 0, 0])
    assert math.isclose(r[22], math.cos(0.5), abs_tol=1e-14)
    assert math.isclose(r[23], math.sin(0.5), abs_tol=1e-14)


def test_rope_relative_position_property():
    rng = np.random.default_rng(4)
    D = 128
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    d1 = np.dot(oracle.rope_3d(q, [10, 3, 40]), oracle.rope_3d(k, [4, 1, 33]))
    d2 = np.dot(oracle.rope_3d(q, [106, 22, 47]), oracle.rope_3d(k, [100, 20, 40]))
    assert math.isclose(d1, d2, rel_tol=1e-11, abs_tol=1e-11)


# ----------------------------------------------------------------------------
# fused append
# ----------------------------------------------------------------------------

def test_append_composition_and_rounding():
    w = wi.WORKLOADS["tiny"]
    x = wi.wave_inputs(w, seed=0)
    pos = oracle.positions(0, w.n_wave, w.F, w.gh, w.gw)
    qb, kb, vb = wi.bits(x.q), wi.bits(x.k), wi.bits(x.v)
    qo, ko, vo, q64, k64 = oracle.append(qb, kb, vb, pos, x.gamma_q.numpy(),
                                         x.gamma_k.numpy(), want_f64=True)
    assert np.array_equal(vo, vb)                 # V is copied bit-exactly
    # the bf16 outputs are within half a bf16 quantum of the f64 values
    for o, f in ((qo, q64), (ko, k64)):
        ov = wi.from_bits(o).double().numpy()
        quantum = np.exp2(np.floor(np.log2(np.abs(f))) - 7)
        assert np.all(np.abs(ov - f) <= 0.5 * quantum * (1 + 1e-12))
    # spot-check the composition norm -> rope through the single-vector helpers
    for n, h in ((0, 0), (37, 1), (95, 0)):
        xq = wi.from_bits(qb[n, h]).double().numpy()
        want = oracle.rope_3d(oracle.rms_norm(xq, x.gamma_q[h].double().numpy()), pos[n])
        assert np.allclose(q64[n, h], want, rtol=0, atol=1e-13)
        # and against a torch fp64 restatement (library rms_norm + complex rotation)
        tn = torch.nn.functional.rms_norm(torch.from_numpy(xq), (w.D,),
                                          x.gamma_q[h].double(), eps=1e-6).numpy()
        assert np.allclose(q64[n, h], _complex_rope(tn, pos[n], (24, 20, 20), 1e4),
                           rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# chunk-causal attention
# ----------------------------------------------------------------------------

def _rand_bits(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return wi.bits(torch.randn(shape, generator=g).to(torch.bfloat16))


def _dense_masked(q, qids, k, v, kids, L):
    """Second route: explicit boolean mask over all (query, key) pairs, fp64."""
    Q = wi.from_bits(q).double().numpy()
    K = wi.from_bits(k).double().numpy()
    V = wi.from_bits(v).double().numpy()
    T, H, D = Q.shape
    M = np.asarray(kids)[np.arange(K.shape[0]) // L][None, :] <= \
        np.asarray(qids)[np.arange(T) // L][:, None]
    O = np.empty((T, H, D))
    lse = np.empty((T, H))
    for h in range(H):
        S = Q[:, h] @ K[:, h].T / math.sqrt(D)
        S = np.where(M, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        Z = E.sum(axis=1, keepdims=True)
        O[:, h] = (E / Z) @ V[:, h]
        lse[:, h] = (m + np.log(Z))[:, 0]
    return O, lse, M


def _all_rows(T, H):
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    return rows, heads


@pytest.mark.parametrize("W,Hh,L,H,D", [(3, 0, 32, 2, 64), (3, 1, 8, 2, 64),
                                        (4, 2, 5, 3, 128), (2, 3, 7, 1, 64)])
def test_attention_matches_dense_mask(W, Hh, L, H, D):
    T = W * L
    r = 10
    q = _rand_bits((T, H, D), 1)
    k = _rand_bits(((Hh + W) * L, H, D), 2)
    v = _rand_bits(((Hh + W) * L, H, D), 3)
    kids = np.arange(r - Hh, r + W)
    qids = np.arange(r, r + W)
    rows, heads = _all_rows(T, H)
    o, lse = oracle.chunk_causal_attn_rows(q, qids, k, v, kids, L, rows, heads)
    O, LSE, _ = _dense_masked(q, qids, k, v, kids, L)
    assert np.allclose(o.reshape(T, H, D), O, rtol=0, atol=1e-12)
    assert np.allclose(lse.reshape(T, H), LSE, rtol=0, atol=1e-12)


def test_attention_key_chunk_order_is_irrelevant():
    # visibility is by absolute chunk id, not by position in the key array
    W, Hh, L, H, D = 3, 2, 6, 2, 64
    q = _rand_bits((W * L, H, D), 4)
    k = _rand_bits(((Hh + W) * L, H, D), 5)
    v = _rand_bits(((Hh + W) * L, H, D), 6)
    kids = np.arange(5 - Hh, 5 + W)
    perm = np.array([3, 0, 4, 2, 1])
    kp = k.reshape(Hh + W, L, H, D)[perm].reshape(k.shape)
    vp = v.reshape(Hh + W, L, H, D)[perm].reshape(v.shape)
    rows, heads = _all_rows(W * L, H)
    qids = np.arange(5, 5 + W)
    o1, _ = oracle.chunk_causal_attn_rows(q, qids, k, v, kids, L, rows, heads)
    o2, _ = oracle.chunk_causal_attn_rows(q, qids, kp, vp, kids[perm], L, rows, heads)
    O, _, _ = _dense_masked(q, qids, kp, vp, kids[perm], L)
    assert np.allclose(o1, o2, rtol=0, atol=1e-13)
    assert np.allclose(o2.reshape(W * L, H, D), O, rtol=0, atol=1e-12)


def test_single_chunk_equals_full_attention_library():
    # one chunk, no history: plain bidirectional softmax attention
    L, H, D = 40, 3, 128
    q, k, v = (_rand_bits((L, H, D), s) for s in (7, 8, 9))
    rows, heads = _all_rows(L, H)
    o, _ = oracle.chunk_causal_attn_rows(q, [0], k, v, [0], L, rows, heads)
    Q, K, V = (wi.from_bits(a).double().permute(1, 0, 2) for a in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V).permute(1, 0, 2)
    assert np.allclose(o.reshape(L, H, D), want.numpy(), rtol=0, atol=1e-12)


def test_one_hot_values_closed_form():
    # K == 0 makes every visible score equal; V[j] = one-hot(key chunk of j)
    # gives O[n] = 1/(visible chunks) on each visible chunk's column, 0 elsewhere.
    W, Hh, L, H, D = 4, 2, 3, 1, 64
    nk = (Hh + W) * L
    q = _rand_bits((W * L, H, D), 10)
    k = np.zeros((nk, H, D), np.uint16)
    vf = np.zeros((nk, H, D))
    for j in range(nk):
        vf[j, 0, j // L] = 1.0
    v = oracle.f64_to_bf16(vf)
    rows, heads = _all_rows(W * L, H)
    o, _ = oracle.chunk_causal_attn_rows(q, np.arange(2, 2 + W), k, v,
                                         np.arange(0, Hh + W), L, rows, heads)
    for i, n in enumerate(rows):
        c = n // L
        nvis = Hh + c + 1
        want = np.zeros(D)
        want[:nvis] = 1.0 / nvis
        assert np.allclose(o[i], want, rtol=0, atol=1e-15)
        assert np.all(o[i][nvis:] == 0.0)


def test_causality_perturbation_bit_identical():
    W, Hh, L, H, D = 4, 1, 9, 2, 64
    q = _rand_bits((W * L, H, D), 11)
    k = _rand_bits(((Hh + W) * L, H, D), 12)
    v = _rand_bits(((Hh + W) * L, H, D), 13)
    kids, qids = np.arange(0, Hh + W), np.arange(Hh, Hh + W)
    rows, heads = _all_rows(W * L, H)
    base, _ = oracle.chunk_causal_attn_rows(q, qids, k, v, kids, L, rows, heads)
    for j in range(W):
        k2, v2 = k.copy(), v.copy()
        sl = slice((Hh + j) * L, (Hh + j + 1) * L)
        k2[sl] = _rand_bits(k2[sl].shape, 100 + j)
        v2[sl] = _rand_bits(v2[sl].shape, 200 + j)
        pert, _ = oracle.chunk_causal_attn_rows(q, qids, k2, v2, kids, L, rows, heads)
        before = rows < j * L
        assert np.array_equal(pert[before], base[before])     # bit-identical
        assert not np.array_equal(pert[~before], base[~before])


def test_softmax_normalisation_and_lse():
    W, Hh, L, H, D = 3, 2, 5, 2, 64
    q = _rand_bits((W * L, H, D), 14)
    k = _rand_bits(((Hh + W) * L, H, D), 15)
    ones = oracle.f64_to_bf16(np.ones(((Hh + W) * L, H, D)))
    kids, qids = np.arange(0, Hh + W), np.arange(Hh, Hh + W)
    rows, heads = _all_rows(W * L, H)
    o, lse = oracle.chunk_causal_attn_rows(q, qids, k, ones, kids, L, rows, heads)
    assert np.allclose(o, 1.0, rtol=0, atol=1e-15)           # weights sum to one
    Q = wi.from_bits(q).double().numpy()
    K = wi.from_bits(k).double().numpy()
    for i, (n, h) in enumerate(zip(rows, heads)):
        nvis = (Hh + n // L + 1) * L
        s = K[:nvis, h] @ Q[n, h] / math.sqrt(D)
        assert math.isclose(np.exp(s - lse[i]).sum(), 1.0, rel_tol=1e-14)


def test_useful_flops_by_brute_force_count():
    for (W, Hh, L, H, D, r) in [(3, 0, 32, 2, 64, 0), (5, 2, 7, 3, 128, 2),
                                (5, 2, 7, 3, 128, 1), (6, 3, 4, 2, 128, 9)]:
        hv = min(Hh, r)
        kids = np.arange(r - hv, r + W)
        qids = np.arange(r, r + W)
        M = kids[np.arange((hv + W) * L) // L][None, :] <= qids[np.arange(W * L) // L][:, None]
        assert oracle.useful_flops(L, W, Hh, H, D, r) == 4.0 * H * D * M.sum()


def test_oracle_cache_round_keys():
    L, H, D = 2, 1, 64
    cache = oracle.OracleCache(L)
    for i in range(0, 12):
        kv = np.full((L, H, D), i, np.uint16)
        cache.put(i, kv, kv + 1)
    k, v, ids = cache.round_keys(0, 3, 2)
    assert list(ids) == [0, 1, 2]                     # nothing before the first round
    k, v, ids = cache.round_keys(1, 3, 2)
    assert list(ids) == [0, 1, 2, 3]                  # pipeline filling: one history chunk
    k, v, ids = cache.round_keys(7, 3, 2)
    assert list(ids) == [5, 6, 7, 8, 9]
    assert np.array_equal(k[:, 0, 0], np.repeat(ids, L).astype(np.uint16))
    assert np.array_equal(v[:, 0, 0], np.repeat(ids, L).astype(np.uint16) + 1)
