"""CPU fp64 oracle for the Wave Forcing wave-round hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The CUDA
library never loads it and shares no code with it; the only thing both sides
take is the seeded input arrays from ``chunk_causal_dit_b200.inputs``.

The arithmetic lives in ``wf_oracle.c`` (plain loops, IEEE double, OpenMP over
rows).  This module compiles it with gcc, loads it with ctypes and adds the
oracle's own model of the K/V history: a dictionary keyed by absolute chunk id,
with no ring and no physical slots, so that the CUDA ring-buffer indexing is
checked against something that does not share its arithmetic.

Readings taken where the pages ("Wave Forcing: Towards Speed-of-Light Streaming
Video Generation", abstract; airadar.tv summary, usage notes) are silent:
history holds the last ``n_hist`` clean (refresh) chunks and a round that comes
before the pipeline is full sees ``min(n_hist, round)`` of them; the wave's
refresh chunk is wave chunk 0 (oldest, cleanest); softmax scale ``1/sqrt(D)``;
RMSNorm ``eps = 1e-6`` per head over D; RoPE theta 10000 with the channel
split ``dt = D - 4*(D//6)``, ``dh = dw = 2*(D//6)``.

The synthetic DiT block around the path (projections, feed-forward, norms) is
in ``oracle/block.py``.

Parity pins: ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wf_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwf_oracle.so")

DEFAULT_EPS = 1e-6
DEFAULT_THETA = 10000.0


def default_rope_split(D: int) -> Tuple[int, int, int]:
    """(dt, dh, dw) channel widths of the t/h/w RoPE blocks for head_dim D."""
    dh = 2 * (D // 6)
    return D - 2 * dh, dh, dh


def build(force: bool = False) -> str:
    """Compile wf_oracle.c into a shared library next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        Dd = ctypes.c_double
        lib.wfo_bf16_to_f64.argtypes = [P, P, L]
        lib.wfo_f64_to_bf16.argtypes = [P, P, L]
        lib.wfo_positions.argtypes = [L, I, I, I, I, P]
        lib.wfo_rms_norm.argtypes = [P, P, I, Dd, P]
        lib.wfo_rope_3d.argtypes = [P, I, I, I, I, Dd, P, P]
        lib.wfo_append.argtypes = [I, I, I, P, P, P, P, P, P, Dd, I, I, I, Dd,
                                   P, P, P, P, P]
        lib.wfo_append.restype = I
        lib.wfo_chunk_causal_attn_rows.argtypes = [I, I, I, P, P, P, P, P, I,
                                                   I, P, P, P, P]
        lib.wfo_e4m3_encode.argtypes = [P, P, L]
        lib.wfo_e4m3_decode.argtypes = [P, P, L]
        lib.wfo_chunk_causal_attn_rows_fp8qk.argtypes = [I, I, I, I, P, P, P, P, P, P, P, I,
                                                         I, P, P, P, P]
        lib.wfo_qk_norm_rope_f64.argtypes = [I, I, I, P, P, P, Dd, I, I, I, Dd, P]
        lib.wfo_qk_norm_rope_f64.restype = I
        lib.wfo_chunk_causal_attn_rows.restype = I
        lib.wfo_num_threads.restype = I
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().wfo_num_threads())


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().wfo_bf16_to_f64(_p(bits), _p(out), bits.size)
    return out


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().wfo_f64_to_bf16(_p(x), _p(out), x.size)
    return out


def positions(round_: int, n_wave: int, F: int, gh: int, gw: int) -> np.ndarray:
    """(t, h, w) int32 [n_wave*F*gh*gw, 3] of the wave tokens of one round."""
    out = np.empty((n_wave * F * gh * gw, 3), dtype=np.int32)
    _load().wfo_positions(int(round_), n_wave, F, gh, gw, _p(out))
    return out


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float = DEFAULT_EPS) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(gamma, dtype=np.float64)
    y = np.empty_like(x)
    _load().wfo_rms_norm(_p(x), _p(g), x.size, eps, _p(y))
    return y


def rope_3d(x: np.ndarray, pos_thw: Sequence[int], split=None,
            theta: float = DEFAULT_THETA) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    D = x.size
    dt, dh, dw = split or default_rope_split(D)
    pos = np.asarray(pos_thw, dtype=np.int32)
    y = np.empty_like(x)
    _load().wfo_rope_3d(_p(x), D, dt, dh, dw, theta, _p(pos), _p(y))
    return y


def append(q, k, v, pos, gamma_q, gamma_k, eps=DEFAULT_EPS, split=None,
           theta=DEFAULT_THETA, want_f64=False):
    """Per-head RMSNorm + 3D RoPE on q and k, rounded once to bf16; v copied.

    q, k, v: uint16 bf16 bits [T, H, D]; pos: int32 [T, 3]; gammas: float32 [H, D].
    Returns (q_out, k_out, v_out) bf16 bits, plus (q_f64, k_f64) if want_f64.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    gq = np.ascontiguousarray(gamma_q, dtype=np.float32)
    gk = np.ascontiguousarray(gamma_k, dtype=np.float32)
    T, H, D = q.shape
    dt, dh, dw = split or default_rope_split(D)
    qo, ko, vo = (np.empty_like(q), np.empty_like(k), np.empty_like(v))
    q64 = np.empty(q.shape, np.float64) if want_f64 else None
    k64 = np.empty(k.shape, np.float64) if want_f64 else None
    rc = _load().wfo_append(T, H, D, _p(q), _p(k), _p(v), _p(pos), _p(gq), _p(gk),
                            eps, dt, dh, dw, theta, _p(qo), _p(ko), _p(vo),
                            _p(q64), _p(k64))
    if rc != 0:
        raise ValueError("oracle append: bad RoPE split %r for D=%d" % ((dt, dh, dw), D))
    if want_f64:
        return qo, ko, vo, q64, k64
    return qo, ko, vo


def chunk_causal_attn_rows(q, q_chunk_ids, k, v, k_chunk_ids, L, rows, heads,
                           want_lse=True):
    """Chunk-causal softmax attention for the given (row, head) pairs.

    q: uint16 [Tq, H, D] queries; query row n lies in chunk n // L whose absolute
    id is q_chunk_ids[n // L].  k, v: uint16 [n_kchunks*L, H, D], key chunk b has
    absolute id k_chunk_ids[b].  Key j is visible to query n iff
    id(j) <= id(n).  Returns (o [n_sel, D] float64, lse [n_sel] float64).
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    qid = np.ascontiguousarray(q_chunk_ids, dtype=np.int64)
    kid = np.ascontiguousarray(k_chunk_ids, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    _, H, D = q.shape
    assert k.shape[0] == kid.size * L and v.shape == k.shape
    n_sel = rows.size
    o = np.empty((n_sel, D), np.float64)
    lse = np.empty(n_sel, np.float64) if want_lse else None
    rc = _load().wfo_chunk_causal_attn_rows(H, D, L, _p(q), _p(qid), _p(k), _p(v),
                                            _p(kid), kid.size, n_sel, _p(rows),
                                            _p(heads), _p(o), _p(lse))
    if rc != 0:
        raise ValueError("oracle attention: a query row sees no key")
    return o, lse


class OracleCache:
    """The oracle's K/V history: absolute chunk id -> (K, V) bf16 [L, H, D].

    No ring, no slots: the CUDA library's ring buffer is checked against this.
    """

    def __init__(self, L: int):
        self.L = L
        self.chunks: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}

    def put(self, chunk_id: int, k: np.ndarray, v: np.ndarray) -> None:
        assert k.shape[0] == self.L and v.shape == k.shape
        self.chunks[int(chunk_id)] = (np.array(k, np.uint16), np.array(v, np.uint16))

    def put_wave(self, round_: int, k_wave: np.ndarray, v_wave: np.ndarray) -> None:
        """Store the K/V of every wave chunk of a round (wave chunk c = id round+c)."""
        W = k_wave.shape[0] // self.L
        for c in range(W):
            sl = slice(c * self.L, (c + 1) * self.L)
            self.put(round_ + c, k_wave[sl], v_wave[sl])

    def round_keys(self, round_: int, n_wave: int, n_hist: int):
        """Concatenated [history | wave] keys of a round and their chunk ids.

        History = the min(n_hist, round) chunks just before the wave, oldest
        first; wave = chunks round .. round+n_wave-1.
        """
        h_valid = min(n_hist, round_)
        ids = list(range(round_ - h_valid, round_ + n_wave))
        k = np.concatenate([self.chunks[i][0] for i in ids], axis=0)
        v = np.concatenate([self.chunks[i][1] for i in ids], axis=0)
        return k, v, np.asarray(ids, np.int64)


def round_attention(cache: OracleCache, round_: int, n_wave: int, n_hist: int,
                    q_wave: np.ndarray, rows, heads):
    """Attention of the given wave (row, head) pairs of one round."""
    k, v, ids = cache.round_keys(round_, n_wave, n_hist)
    qids = np.arange(round_, round_ + n_wave, dtype=np.int64)
    return chunk_causal_attn_rows(q_wave, qids, k, v, ids, cache.L, rows, heads)


# ---- FP8 (E4M3) quantized Q.K^T ------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes -> float64 values (S.1111.111 decodes to NaN)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().wfo_e4m3_decode(_p(c), _p(out), c.size)
    return out


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 codes: round to nearest, ties to even, +-448 saturation."""
    a = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(a.shape, np.uint8)
    _load().wfo_e4m3_encode(_p(a), _p(out), a.size)
    return out


def _bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _fp8_scale(amax: np.ndarray) -> np.ndarray:
    """Per-group dequantization scale in fp32: amax / 448 (IEEE fp32 division), 1 for
    an all-zero group."""
    amax = np.asarray(amax, np.float32)
    return np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)


def _fp8_inv(amax: np.ndarray) -> np.ndarray:
    """Per-group quantization multiplier in fp32: 448 / amax (IEEE fp32 division), 1
    for an all-zero group."""
    amax = np.asarray(amax, np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    return np.where(amax > 0, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)


def _fp8_codes(x32: np.ndarray, inv32: np.ndarray) -> np.ndarray:
    # the product is formed in fp32 (IEEE multiply), then rounded once to E4M3
    return e4m3_encode((x32 * inv32).astype(np.float32).astype(np.float64))


def quantize_rows_fp8(bits: np.ndarray):
    """bf16 [N, H, D] -> (E4M3 codes [N, H, D], fp32 scales [H, N]); one group per
    (row, head): codes = E4M3(x * (448 / amax)), scale = amax / 448, so the group's
    largest magnitude maps to 448 and code * scale approximates x."""
    x = _bf16_bits_to_f32(bits)
    amax = np.abs(x).max(axis=2)                       # [N, H]
    s = _fp8_scale(amax)
    return _fp8_codes(x, _fp8_inv(amax)[:, :, None]), np.ascontiguousarray(s.T)


def quantize_tiles_fp8(bits: np.ndarray, tile: int = 128):
    """bf16 [L, H, D] of one chunk -> (E4M3 codes [L, H, D], fp32 scales [ceil(L/tile), H]);
    one scale per (tile of `tile` rows, head)."""
    x = _bf16_bits_to_f32(bits)
    L, H, _ = x.shape
    nt = (L + tile - 1) // tile
    scales = np.empty((nt, H), np.float32)
    codes = np.empty(x.shape, np.uint8)
    for t in range(nt):
        sl = slice(t * tile, min(L, (t + 1) * tile))
        amax = np.abs(x[sl]).max(axis=(0, 2))
        scales[t] = _fp8_scale(amax)
        codes[sl] = _fp8_codes(x[sl], _fp8_inv(amax)[None, :, None])
    return codes, scales


class OracleCacheFP8:
    """Absolute chunk id -> (K codes [L,H,D], K scales [nt,H], V bf16 [L,H,D])."""

    def __init__(self, L: int):
        self.L = L
        self.chunks: Dict[int, Tuple[np.ndarray, np.ndarray, np.ndarray]] = {}

    def put(self, chunk_id: int, k8: np.ndarray, k_scale: np.ndarray, v: np.ndarray) -> None:
        self.chunks[int(chunk_id)] = (np.array(k8, np.uint8), np.array(k_scale, np.float32),
                                      np.array(v, np.uint16))

    def put_bf16(self, chunk_id: int, k_bits: np.ndarray, v_bits: np.ndarray) -> None:
        """Quantize a bf16 K chunk by the per-tile rule and store it."""
        k8, ks = quantize_tiles_fp8(k_bits)
        self.put(chunk_id, k8, ks, v_bits)


def round_attention_fp8qk(cache: OracleCacheFP8, round_: int, n_wave: int, n_hist: int,
                          q8: np.ndarray, q_scale: np.ndarray, rows, heads):
    """Attention of the given (row, head) pairs of one round with E4M3 q and k
    (dequantized exactly by their fp32 scales) and bf16 v."""
    h_valid = min(n_hist, round_)
    ids = list(range(round_ - h_valid, round_ + n_wave))
    k8 = np.ascontiguousarray(np.concatenate([cache.chunks[i][0] for i in ids], axis=0))
    ks = np.ascontiguousarray(np.stack([cache.chunks[i][1] for i in ids], axis=0))
    v = np.ascontiguousarray(np.concatenate([cache.chunks[i][2] for i in ids], axis=0))
    kid = np.asarray(ids, np.int64)
    qid = np.arange(round_, round_ + n_wave, dtype=np.int64)
    q8 = np.ascontiguousarray(q8, np.uint8)
    q_scale = np.ascontiguousarray(q_scale, np.float32)
    rows = np.ascontiguousarray(rows, np.int32)
    heads = np.ascontiguousarray(heads, np.int32)
    Tq, H, D = q8.shape
    o = np.empty((rows.size, D), np.float64)
    lse = np.empty(rows.size, np.float64)
    rc = _load().wfo_chunk_causal_attn_rows_fp8qk(H, D, cache.L, Tq, _p(q8), _p(q_scale), _p(qid),
                                                  _p(k8), _p(ks), _p(v), _p(kid), kid.size,
                                                  rows.size, _p(rows), _p(heads), _p(o), _p(lse))
    if rc != 0:
        raise ValueError("oracle attention: a query row sees no key")
    return o, lse


def useful_flops(L: int, n_wave: int, n_hist: int, H: int, D: int, round_: int) -> float:
    """QK^T and PV multiply-adds (x2) over visible, unpadded (query, key) pairs."""
    h_valid = min(n_hist, round_)
    pairs = sum((h_valid + c + 1) * L * L for c in range(n_wave))
    return 4.0 * H * D * pairs
