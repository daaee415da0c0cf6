"""CPU fp64 oracle for the synthetic DiT block around the wave-round path.

TEST INFRASTRUCTURE ONLY (the same rule as the rest of ``oracle/``): only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` call it.

"Wave Forcing: Towards Speed-of-Light Streaming Video Generation" (abstract)
runs every wave chunk through the layers of Wan2.1-T2V-1.3B in one forward
pass; the attention of that pass is the chunk-causal wave attention, and the
layers around it are the linear projections and the feed-forward network of a
DiT block.  The pages print none of these layers' formulas.  The readings taken
here (each one a plain definition):

* A linear layer is ``y = x W^T + b`` with ``W`` stored ``[out, in]``; the
  product of the bf16 operands is formed exactly (fp64 holds every bf16 x bf16
  product and the sums at these sizes to ~1e-16 relative) and the epilogue's
  result is rounded once to bf16 (round to nearest, ties to even).
* Epilogues: ``store`` (y), ``gelu_tanh`` (the tanh form of GELU,
  0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))), ``gated_residual``
  (``resid + gate * y``, the gated residual of an adaLN block).
* The wave's chunks sit at different denoising steps, so every chunk carries
  its own modulation: row ``n`` of a wave takes row ``n // rows_per_group`` of
  ``shift``, ``scale`` and ``gate`` (``rows_per_group`` = chunk tokens).
* The pre-attention and pre-FFN norms are LayerNorm without a learned affine,
  eps 1e-6, followed by the modulation ``x_hat * (1 + scale) + shift``.
* The QKV projection is one linear layer of ``3 H D`` outputs: rows
  ``[0, HD)`` of ``W`` make q, ``[HD, 2HD)`` k and ``[2HD, 3HD)`` v, each
  head-major (output ``h*D + d``).  The per-head RMSNorm and 3D RoPE of the
  append (the wave-round path) act on the exact projection (bias included),
  and q, k and v are each rounded once to bf16.

Pins: ``tests/test_block_pins.py``.
"""
from __future__ import annotations

import math

import numpy as np

from . import (DEFAULT_EPS, DEFAULT_THETA, _load, _p, bf16_to_f64, default_rope_split,
               f64_to_bf16)

LN_EPS = 1e-6
EPILOGUES = ("store", "gelu_tanh", "gated_residual")


def gelu_tanh(y: np.ndarray) -> np.ndarray:
    """Tanh form of GELU in fp64."""
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * y * (1.0 + np.tanh(c * (y + 0.044715 * y * y * y)))


def _group_rows(mod: np.ndarray, M: int, rows_per_group: int) -> np.ndarray:
    """Per-row view of a per-group modulation table [G, N] (row n -> group n // rpg)."""
    mod = np.asarray(mod, dtype=np.float64)
    if mod.ndim == 1:
        mod = mod[None, :]
    g = np.arange(M) // rows_per_group
    if g.size and g.max() >= mod.shape[0]:
        raise ValueError("modulation table has %d groups, rows need %d"
                         % (mod.shape[0], g.max() + 1))
    return mod[g]


def linear_f64(x_bits, w_bits, bias=None, epilogue="store", gate=None, resid_bits=None,
               rows_per_group=None):
    """Exact ``x W^T + b`` followed by the epilogue, in fp64 (not rounded).

    x_bits [M, K], w_bits [N, K], resid_bits [M, N]: bf16 bit patterns;
    bias [N] fp32; gate [G, N] fp32 (row n uses group n // rows_per_group).
    """
    if epilogue not in EPILOGUES:
        raise ValueError("unknown epilogue %r" % (epilogue,))
    x = bf16_to_f64(x_bits)
    w = bf16_to_f64(w_bits)
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    if epilogue == "gelu_tanh":
        y = gelu_tanh(y)
    elif epilogue == "gated_residual":
        M = y.shape[0]
        g = _group_rows(np.asarray(gate, np.float32), M, rows_per_group or M)
        y = bf16_to_f64(resid_bits) + g * y
    return y


def linear(x_bits, w_bits, bias=None, epilogue="store", gate=None, resid_bits=None,
           rows_per_group=None):
    """bf16 bits of :func:`linear_f64` (one rounding)."""
    return f64_to_bf16(linear_f64(x_bits, w_bits, bias, epilogue, gate, resid_bits,
                                  rows_per_group))


def layer_norm_modulate_f64(x_bits, shift, scale, rows_per_group, eps=LN_EPS):
    """LayerNorm over the last axis (no affine), then x_hat * (1 + scale) + shift."""
    x = bf16_to_f64(x_bits)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    xh = (x - mu) / np.sqrt(var + eps)
    M = x.shape[0]
    sc = _group_rows(np.asarray(scale, np.float32), M, rows_per_group)
    sh = _group_rows(np.asarray(shift, np.float32), M, rows_per_group)
    return xh * (1.0 + sc) + sh


def layer_norm_modulate(x_bits, shift, scale, rows_per_group, eps=LN_EPS):
    return f64_to_bf16(layer_norm_modulate_f64(x_bits, shift, scale, rows_per_group, eps))


def qk_norm_rope_f64(x, pos, gamma, eps=DEFAULT_EPS, split=None, theta=DEFAULT_THETA):
    """Per-head RMSNorm (gain gamma[h]) and 3D RoPE of fp64 rows x [T, H, D]."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, H, D = x.shape
    dt, dh, dw = split or default_rope_split(D)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    y = np.empty_like(x)
    lib = _load()
    rc = lib.wfo_qk_norm_rope_f64(T, H, D, _p(x), _p(pos), _p(g), float(eps), dt, dh, dw,
                                  float(theta), _p(y))
    if rc != 0:
        raise ValueError("oracle norm/rope: bad RoPE split %r for D=%d" % ((dt, dh, dw), D))
    return y


def qkv_project_append(x_bits, w_bits, bias, pos, gamma_q, gamma_k, H, D,
                       eps=DEFAULT_EPS, split=None, theta=DEFAULT_THETA, want_f64=False):
    """QKV projection with the append's norm and RoPE fused after it.

    x_bits [T, C], w_bits [3HD, C] bf16 bits; bias [3HD] fp32 or None;
    pos [T, 3] int32; gammas [H, D] fp32.  Returns bf16 bits (q_out, k, v), each
    [T, H, D] (k and v are what the ring slots receive), plus their fp64 values
    if want_f64.
    """
    y = linear_f64(x_bits, w_bits, bias)
    T = y.shape[0]
    y = y.reshape(T, 3, H, D)
    q = qk_norm_rope_f64(y[:, 0], pos, gamma_q, eps, split, theta)
    k = qk_norm_rope_f64(y[:, 1], pos, gamma_k, eps, split, theta)
    v = np.ascontiguousarray(y[:, 2])
    out = (f64_to_bf16(q), f64_to_bf16(k), f64_to_bf16(v))
    if want_f64:
        return out + (q, k, v)
    return out


def block_forward(x_bits, wts, mod, pos, cache, round_, n_wave, n_hist, H, D, L,
                  eps=DEFAULT_EPS, split=None, theta=DEFAULT_THETA):
    """One DiT block over a wave (reading s16 of the block's layers), composed from
    the functions above; every intermediate the GPU stores is rounded once to bf16.

    x_bits [T, C]; wts: dict of bf16 bits w_qkv, w_o, w_1, w_2 and fp32 b_qkv, b_o,
    b_1, b_2, gamma_q, gamma_k; mod [6, n_wave, C] fp32 (shift, scale, gate of the
    attention half, then of the feed-forward half; chunk c's tokens take row c);
    pos [T, 3]; cache: an ``oracle.OracleCache`` holding the visible history
    chunks (the wave's K/V are added here, under their absolute ids).
    Returns the block's output x2 (bf16 bits [T, C]) and the intermediates.
    """
    from . import round_attention
    T, C = x_bits.shape
    h = layer_norm_modulate(x_bits, mod[0], mod[1], L)
    q, k, v = qkv_project_append(h, wts["w_qkv"], wts["b_qkv"], pos, wts["gamma_q"],
                                 wts["gamma_k"], H, D, eps, split, theta)
    cache.put_wave(round_, k, v)
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    o64, _ = round_attention(cache, round_, n_wave, n_hist, q, rows, heads)
    o = f64_to_bf16(o64).reshape(T, H * D)
    x1 = linear(o, wts["w_o"], wts["b_o"], "gated_residual", mod[2], x_bits, L)
    h2 = layer_norm_modulate(x1, mod[3], mod[4], L)
    f = linear(h2, wts["w_1"], wts["b_1"], "gelu_tanh")
    x2 = linear(f, wts["w_2"], wts["b_2"], "gated_residual", mod[5], x1, L)
    return x2, dict(h=h, q=q, k=k, v=v, o=o, x1=x1, h2=h2, f=f)
