"""Pins for the oracle of the synthetic DiT block (oracle/block.py).

Each pin ties the oracle to something other than itself:
* linear: identity and permutation weights (exact), a weight of zeros (the bias
  alone), and an exactly rounded brute-force sum (math.fsum) on tiny shapes;
* GELU (tanh form): PyTorch's own implementation in fp64 and the identity
  gelu(x) - gelu(-x) = x that the tanh form satisfies because tanh is odd;
* gated residual: gate 0 returns the residual bit for bit, and a one-hot gate
  table shows which modulation row every token takes;
* LayerNorm + modulation: PyTorch's layer_norm in fp64, constant rows (x_hat = 0
  so the output is the shift itself), per-chunk modulation rows;
* QKV projection with the fused norm/RoPE/append: with W = [I; I; I] it must
  reduce bit for bit to the (separately pinned) append oracle applied to x, and
  permuting W's heads permutes the outputs' heads;
* the composed block: zero gates return the input bit for bit, and with the
  feed-forward gate zero the block is the gated attention half of its parts.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.block as ob


def _bits(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    return oracle.f64_to_bf16(x.astype(np.float64))


def _rand_bits(g, shape, scale=1.0):
    return _bits(g.standard_normal(shape) * scale)


def test_linear_identity_permutation_and_bias_only():
    g = np.random.default_rng(1)
    x = _rand_bits(g, (9, 16))
    eye = _bits(np.eye(16))
    assert np.array_equal(ob.linear(x, eye), x)
    perm = g.permutation(16)
    assert np.array_equal(ob.linear(x, eye[perm]), x[:, perm])
    bias = g.standard_normal(16).astype(np.float32)
    got = ob.linear(x, np.zeros((16, 16), np.uint16), bias)
    assert np.array_equal(got, np.broadcast_to(_bits(bias), got.shape))


def test_linear_brute_force_exact_sum():
    g = np.random.default_rng(2)
    M, N, K = 3, 4, 37
    x, w = _rand_bits(g, (M, K)), _rand_bits(g, (N, K))
    bias = g.standard_normal(N).astype(np.float32)
    xf, wf = oracle.bf16_to_f64(x), oracle.bf16_to_f64(w)
    y = ob.linear_f64(x, w, bias)
    for m in range(M):
        for n in range(N):
            exact = math.fsum([float(xf[m, k]) * float(wf[n, k]) for k in range(K)] +
                              [float(bias[n])])
            assert abs(y[m, n] - exact) <= 1e-14 * max(1.0, abs(exact))


def test_gelu_tanh_library_and_odd_identity():
    x = np.linspace(-12.0, 12.0, 2001)
    lib = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.max(np.abs(ob.gelu_tanh(x) - lib)) <= 1e-15 * 12
    assert np.max(np.abs(ob.gelu_tanh(x) - ob.gelu_tanh(-x) - x)) <= 1e-14
    assert ob.gelu_tanh(np.array([0.0]))[0] == 0.0


def test_gated_residual_gate_zero_and_group_rows():
    g = np.random.default_rng(3)
    M, N, K, rpg = 12, 8, 16, 4
    x, w, r = _rand_bits(g, (M, K)), _rand_bits(g, (N, K)), _rand_bits(g, (M, N))
    zero_gate = np.zeros((3, N), np.float32)
    assert np.array_equal(ob.linear(x, w, None, "gated_residual", zero_gate, r, rpg), r)
    gate = np.zeros((3, N), np.float32)
    gate[1] = 1.0                        # only the second group of rows gets the product
    y = ob.linear_f64(x, w, None, "gated_residual", gate, r, rpg)
    prod = oracle.bf16_to_f64(x) @ oracle.bf16_to_f64(w).T
    res = oracle.bf16_to_f64(r)
    assert np.array_equal(y[:4], res[:4]) and np.array_equal(y[8:], res[8:])
    assert np.array_equal(y[4:8], res[4:8] + prod[4:8])


def test_layer_norm_modulate_library_constant_rows_and_groups():
    g = np.random.default_rng(4)
    M, C, rpg = 10, 48, 5
    x = _rand_bits(g, (M, C), 3.0)
    x[7] = x[7, 0]                       # a constant row: x_hat = 0
    shift = g.standard_normal((2, C)).astype(np.float32)
    scale = g.standard_normal((2, C)).astype(np.float32)
    y = ob.layer_norm_modulate_f64(x, shift, scale, rpg)
    xt = torch.from_numpy(oracle.bf16_to_f64(x))
    ln = torch.nn.functional.layer_norm(xt, (C,), eps=ob.LN_EPS).numpy()
    grp = np.arange(M) // rpg
    want = ln * (1.0 + scale[grp].astype(np.float64)) + shift[grp].astype(np.float64)
    assert np.max(np.abs(y - want)) <= 1e-12
    assert np.array_equal(y[7], shift[1].astype(np.float64))
    z = ob.layer_norm_modulate_f64(x, np.zeros(C, np.float32), np.zeros(C, np.float32), M)
    keep = [i for i in range(M) if i != 7]
    assert np.max(np.abs(z[keep].mean(axis=1))) <= 1e-12
    var = oracle.bf16_to_f64(x)[keep].var(axis=1)
    assert np.allclose(z[keep].var(axis=1), var / (var + ob.LN_EPS), rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,D", [(2, 64), (3, 128)])
def test_qkv_identity_reduces_to_append(H, D):
    g = np.random.default_rng(H * D)
    T, C = 40, H * D
    x = _rand_bits(g, (T, C))
    eye = np.eye(C)
    w = _bits(np.concatenate([eye, eye, eye], axis=0))
    pos = oracle.positions(3, 2, 2, 2, 5)
    gq = (1 + 0.1 * g.standard_normal((H, D))).astype(np.float32)
    gk = (1 + 0.1 * g.standard_normal((H, D))).astype(np.float32)
    q, k, v = ob.qkv_project_append(x, w, None, pos, gq, gk, H, D)
    xh = x.reshape(T, H, D)
    rq, rk, rv = oracle.append(xh, xh, xh, pos, gq, gk)
    assert np.array_equal(q, rq) and np.array_equal(k, rk) and np.array_equal(v, rv)


def test_qkv_head_permutation():
    g = np.random.default_rng(6)
    T, H, D, C = 20, 3, 64, 96
    x = _rand_bits(g, (T, C))
    w = _rand_bits(g, (3 * H * D, C), 0.1)
    bias = g.standard_normal(3 * H * D).astype(np.float32)
    pos = oracle.positions(0, 1, 1, 4, 5)
    gq = (1 + 0.1 * g.standard_normal((H, D))).astype(np.float32)
    gk = (1 + 0.1 * g.standard_normal((H, D))).astype(np.float32)
    perm = np.array([2, 0, 1])
    rows = np.arange(3 * H * D).reshape(3, H, D)[:, perm].reshape(-1)
    q, k, v = ob.qkv_project_append(x, w, bias, pos, gq, gk, H, D)
    pq, pk, pv = ob.qkv_project_append(x, w[rows], bias[rows], pos, gq[perm], gk[perm], H, D)
    assert np.array_equal(pq, q[:, perm]) and np.array_equal(pk, k[:, perm])
    assert np.array_equal(pv, v[:, perm])


def _block_case(seed, F=1, gh=2, gw=8, W=2, Hh=1, H=2, D=64, ffn=96, r=1):
    g = np.random.default_rng(seed)
    L = F * gh * gw
    T, C = W * L, H * D
    wts = dict(w_qkv=_rand_bits(g, (3 * C, C), 0.1), w_o=_rand_bits(g, (C, C), 0.1),
               w_1=_rand_bits(g, (ffn, C), 0.1), w_2=_rand_bits(g, (C, ffn), 0.1),
               b_qkv=g.standard_normal(3 * C).astype(np.float32) * 0.02,
               b_o=g.standard_normal(C).astype(np.float32) * 0.02,
               b_1=g.standard_normal(ffn).astype(np.float32) * 0.02,
               b_2=g.standard_normal(C).astype(np.float32) * 0.02,
               gamma_q=(1 + 0.1 * g.standard_normal((H, D))).astype(np.float32),
               gamma_k=(1 + 0.1 * g.standard_normal((H, D))).astype(np.float32))
    mod = (0.1 * g.standard_normal((6, W, C))).astype(np.float32)
    x = _rand_bits(g, (T, C))
    cache = oracle.OracleCache(L)
    for j in range(min(Hh, r)):
        cache.put(r - 1 - j, _rand_bits(g, (L, H, D)), _rand_bits(g, (L, H, D)))
    pos = oracle.positions(r, W, F, gh, gw)
    return x, wts, mod, pos, cache, dict(round_=r, n_wave=W, n_hist=Hh, H=H, D=D, L=L)


def test_block_forward_zero_gates_return_the_input():
    x, wts, mod, pos, cache, kw = _block_case(11)
    mod[2] = 0.0
    mod[5] = 0.0
    x2, inter = ob.block_forward(x, wts, mod, pos, cache, **kw)
    assert np.array_equal(x2, x) and np.array_equal(inter["x1"], x)


def test_block_forward_attention_half_matches_its_parts():
    """With the feed-forward gate zero, the block is x + gate * (o W_o^T + b_o) of
    the chunk-causal attention over the fused projection's q/k/v (the parts
    pinned separately), and the ring holds the wave's K/V under their ids."""
    x, wts, mod, pos, cache, kw = _block_case(12)
    mod[5] = 0.0
    x2, inter = ob.block_forward(x, wts, mod, pos, cache, **kw)
    L, H, D, W, r = kw["L"], kw["H"], kw["D"], kw["n_wave"], kw["round_"]
    h = ob.layer_norm_modulate(x, mod[0], mod[1], L)
    q, k, v = ob.qkv_project_append(h, wts["w_qkv"], wts["b_qkv"], pos, wts["gamma_q"],
                                    wts["gamma_k"], H, D)
    for c in range(W):
        assert np.array_equal(cache.chunks[r + c][0], k[c * L:(c + 1) * L])
    T = W * L
    rows, heads = np.repeat(np.arange(T), H), np.tile(np.arange(H), T)
    o64, _ = oracle.round_attention(cache, r, W, kw["n_hist"], q, rows, heads)
    o = oracle.f64_to_bf16(o64).reshape(T, H * D)
    want = ob.linear(o, wts["w_o"], wts["b_o"], "gated_residual", mod[2], x, L)
    assert np.array_equal(x2, want)
