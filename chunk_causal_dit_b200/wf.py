"""ctypes binding of libwf.so with the C ABI's names (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module only
turns torch tensors (or raw integers) into pointers and status codes into
exceptions.  Loading fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
# WF_LIB_VARIANT=check selects the bounds-checked debug build (build.py --check)
LIB_PATH = os.path.join(HERE, "libwf_check.so" if os.environ.get("WF_LIB_VARIANT") == "check"
                        else "libwf.so")

WF_OK = 0
WF_ERR_INVALID_ARG = 1
WF_ERR_UNSUPPORTED = 2
WF_ERR_CUDA = 3
WF_ERR_TIMEOUT = 4
WF_ERR_NO_DEVICE = 5
WF_ERR_DEVICE = 6
WF_ERR_BOUNDS = 7

# attention kernel variants (wf_plan_set_attn_kernel)
WF_ATTN_AUTO = 0
WF_ATTN_SINGLE = 1
WF_ATTN_PAIR = 2

# epilogues of wf_linear
WF_EPI_STORE = 0
WF_EPI_GELU_TANH = 1
WF_EPI_GATED_RESIDUAL = 2

# Every function include/wf.h declares: name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_long
SIGNATURES = {
    "wf_plan": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
    "wf_plan_set_rope": (_I, [_P, _I, _I, _I, ctypes.c_double]),
    "wf_plan_set_rope_split": (_I, [_P, _I, _I, _I]),
    "wf_plan_set_norm_eps": (_I, [_P, ctypes.c_double]),
    "wf_plan_set_wait_limit": (_I, [_P, ctypes.c_ulonglong]),
    "wf_plan_set_withhold_q": (_I, [_P, _I]),
    "wf_plan_set_attn_kernel": (_I, [_P, _I]),
    "wf_plan_set_head_block": (_I, [_P, _I]),
    "wf_plan_head_block": (_I, [_P, _L, _I]),
    "wf_attn_head_block": (_I, [_I, _I, _I, _I, _I, _I, ctypes.c_longlong, _I]),
    "wf_plan_destroy": (None, [_P]),
    "wf_cache_bytes": (ctypes.c_size_t, [_P]),
    "wf_useful_flops": (ctypes.c_double, [_P, _L]),
    "wf_qk_norm_rope_append": (_I, [_P, _L, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "wf_chunk_causal_attn": (_I, [_P, _L, _P, _P, _P, _P, _P, _P]),
    "wf_sync_status": (_I, [_P, _P]),
    "wf_plan_debug_ranges": (_I, [_P, _L, _P, _I]),
    "wf_status_string": (ctypes.c_char_p, [_I]),
    "wf_chunk_causal_attn_noalloc": (_I, [_I, _I, _I, _I, _I, _L, _P, _P, _P, _P, _P, _P]),
    "wf_noalloc_debug_fill_scratch": (_I, [ctypes.c_uint]),
    "wf_noalloc_sync_status": (_I, [_P]),
    "wf_quantize_q_fp8": (_I, [_P, _P, _P, _P, _P]),
    "wf_qk_norm_rope_append_fp8q": (_I, [_P, _L, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                         _P]),
    "wf_quantize_k_fp8": (_I, [_P, _L, _I, _P, _P, _P, _P]),
    "wf_chunk_causal_attn_fp8qk": (_I, [_P, _L, _P, _P, _P, _P, _P, _P, _P, _P]),
    "wf_linear": (_I, [_P, _I, _I, _I, _P, _P, _P, _I, _P, _P, _I, _P, _P]),
    "wf_qkv_proj_norm_rope_append": (_I, [_P, _L, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "wf_layer_norm_modulate": (_I, [_P, _I, _I, _P, _P, _P, _I, _P, _P]),
    "wf_causal_conv3d": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "wf_rms_norm_silu": (_I, [_P, _I, _I, _P, _P, _P, _P]),
}

_lib = None


class WFError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


def load() -> ctypes.CDLL:
    """Load libwf.so (built in-tree by chunk_causal_dit_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libwf.so not built: run `python -m chunk_causal_dit_b200.build` "
                              "(expected at %s)" % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().wf_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != WF_OK:
        raise WFError(status, what)


def _ptr(x) -> Optional[int]:
    """torch tensor / int / None -> raw pointer value."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Plan:
    """Owns a wf_plan_t; mirrors wf_plan / wf_plan_set_* / wf_plan_destroy."""

    def __init__(self, chunk_tokens: int, n_wave_chunks: int, n_hist_chunks: int, heads: int,
                 head_dim: int):
        self.L, self.W, self.Hh, self.H, self.D = (chunk_tokens, n_wave_chunks, n_hist_chunks,
                                                   heads, head_dim)
        self.R = n_hist_chunks + n_wave_chunks
        self.T = chunk_tokens * n_wave_chunks
        h = ctypes.c_void_p()
        _check(load().wf_plan(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim,
                              ctypes.byref(h)), "wf_plan")
        self.handle = h.value

    def set_rope(self, frames_per_chunk: int, grid_h: int, grid_w: int, theta: float = 10000.0):
        _check(load().wf_plan_set_rope(self.handle, frames_per_chunk, grid_h, grid_w, theta),
               "wf_plan_set_rope")
        return self

    def set_rope_split(self, d_t: int, d_h: int, d_w: int):
        _check(load().wf_plan_set_rope_split(self.handle, d_t, d_h, d_w), "wf_plan_set_rope_split")
        return self

    def set_norm_eps(self, eps: float):
        _check(load().wf_plan_set_norm_eps(self.handle, eps), "wf_plan_set_norm_eps")
        return self

    def set_wait_limit(self, cycles: int):
        _check(load().wf_plan_set_wait_limit(self.handle, cycles), "wf_plan_set_wait_limit")
        return self

    def set_withhold_q(self, on: bool):
        """Test hook: make the attention kernel's first Q wait expire (see wf.h)."""
        _check(load().wf_plan_set_withhold_q(self.handle, int(bool(on))), "wf_plan_set_withhold_q")
        return self

    def set_attn_kernel(self, kind: int):
        """WF_ATTN_AUTO, WF_ATTN_SINGLE or WF_ATTN_PAIR (see wf.h)."""
        _check(load().wf_plan_set_attn_kernel(self.handle, int(kind)), "wf_plan_set_attn_kernel")
        return self

    def set_head_block(self, heads: int):
        """Heads per block of the attention's unit order; 0 = chosen per call (see wf.h)."""
        _check(load().wf_plan_set_head_block(self.handle, int(heads)), "wf_plan_set_head_block")
        return self

    def head_block(self, round_: int, fp8_keys: bool = False) -> int:
        """Heads per block that round `round_`'s attention call uses."""
        return int(load().wf_plan_head_block(self.handle, round_, int(bool(fp8_keys))))

    def destroy(self):
        if self.handle:
            load().wf_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.destroy()


def wf_plan(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim) -> Plan:
    return Plan(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim)


def wf_attn_head_block(heads, n_wave_chunks, h_valid, chunk_tokens, head_dim, key_bytes,
                       l2_bytes, n_ctas) -> int:
    return int(load().wf_attn_head_block(heads, n_wave_chunks, h_valid, chunk_tokens, head_dim,
                                         key_bytes, l2_bytes, n_ctas))


def wf_cache_bytes(plan: Plan) -> int:
    return int(load().wf_cache_bytes(plan.handle))


def wf_useful_flops(plan: Plan, round_: int) -> float:
    return float(load().wf_useful_flops(plan.handle, round_))


def wf_qk_norm_rope_append(plan: Plan, round_: int, q, k, v, pos_thw, gamma_q, gamma_k, q_out,
                           k_cache, v_cache, stream=None) -> None:
    _check(load().wf_qk_norm_rope_append(plan.handle, round_, _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(pos_thw), _ptr(gamma_q), _ptr(gamma_k),
                                         _ptr(q_out), _ptr(k_cache), _ptr(v_cache),
                                         _stream(stream)), "wf_qk_norm_rope_append")


def wf_chunk_causal_attn(plan: Plan, round_: int, q_out, k_cache, v_cache, o, lse=None,
                         stream=None) -> None:
    _check(load().wf_chunk_causal_attn(plan.handle, round_, _ptr(q_out), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(o), _ptr(lse), _stream(stream)),
           "wf_chunk_causal_attn")


def wf_quantize_q_fp8(plan: Plan, q_out, q8, q_scale, stream=None) -> None:
    """q_out [T,H,D] bf16 -> q8 [T,H,D] uint8 E4M3 codes, q_scale [H,T] float32."""
    _check(load().wf_quantize_q_fp8(plan.handle, _ptr(q_out), _ptr(q8), _ptr(q_scale),
                                    _stream(stream)), "wf_quantize_q_fp8")


def wf_qk_norm_rope_append_fp8q(plan: Plan, round_: int, q, k, v, pos_thw, gamma_q, gamma_k,
                                q_out, q8, q_scale, k_cache, v_cache, stream=None) -> None:
    """wf_qk_norm_rope_append that also writes the E4M3 codes q8 [T,H,D] uint8 and
    row scales q_scale [H,T] float32 of its bf16 q'; q_out may be None."""
    _check(load().wf_qk_norm_rope_append_fp8q(
        plan.handle, round_, _ptr(q), _ptr(k), _ptr(v), _ptr(pos_thw), _ptr(gamma_q),
        _ptr(gamma_k), _ptr(q_out), _ptr(q8), _ptr(q_scale), _ptr(k_cache), _ptr(v_cache),
        _stream(stream)), "wf_qk_norm_rope_append_fp8q")


def wf_quantize_k_fp8(plan: Plan, first_chunk: int, n_chunks: int, k_cache, k8_cache, k_scale,
                      stream=None) -> None:
    """K of chunks first_chunk.. (ring slots chunk mod R) -> E4M3 codes in k8_cache
    [R,L,H,D] uint8 and per-tile scales k_scale [R, ceil(L/128), H] float32."""
    _check(load().wf_quantize_k_fp8(plan.handle, first_chunk, n_chunks, _ptr(k_cache),
                                    _ptr(k8_cache), _ptr(k_scale), _stream(stream)),
           "wf_quantize_k_fp8")


def wf_chunk_causal_attn_fp8qk(plan: Plan, round_: int, q8, q_scale, k8_cache, k_scale, v_cache,
                               o, lse=None, stream=None) -> None:
    _check(load().wf_chunk_causal_attn_fp8qk(plan.handle, round_, _ptr(q8), _ptr(q_scale),
                                             _ptr(k8_cache), _ptr(k_scale), _ptr(v_cache),
                                             _ptr(o), _ptr(lse), _stream(stream)),
           "wf_chunk_causal_attn_fp8qk")


def wf_linear(plan: Plan, x, w, y, bias=None, epilogue=WF_EPI_STORE, gate=None, resid=None,
              rows_per_group=1, stream=None) -> None:
    """y [M,N] = epilogue(x [M,K] @ w[N,K]^T + bias), bf16 in and out (see wf.h)."""
    M, K = x.shape
    N = w.shape[0]
    _check(load().wf_linear(plan.handle, M, N, K, _ptr(x), _ptr(w), _ptr(bias), epilogue,
                            _ptr(gate), _ptr(resid), rows_per_group, _ptr(y), _stream(stream)),
           "wf_linear")


def wf_qkv_proj_norm_rope_append(plan: Plan, round_: int, x, w_qkv, b_qkv, gamma_q, gamma_k,
                                 q_out, k_cache, v_cache, stream=None) -> None:
    """x [T,hidden] @ w_qkv[3HD,hidden]^T + b_qkv, then the append's norm/RoPE/ring write."""
    _check(load().wf_qkv_proj_norm_rope_append(plan.handle, round_, x.shape[1], _ptr(x),
                                               _ptr(w_qkv), _ptr(b_qkv), _ptr(gamma_q),
                                               _ptr(gamma_k), _ptr(q_out), _ptr(k_cache),
                                               _ptr(v_cache), _stream(stream)),
           "wf_qkv_proj_norm_rope_append")


def wf_layer_norm_modulate(plan: Plan, x, shift, scale, rows_per_group, y, stream=None) -> None:
    """y = LayerNorm(x) * (1 + scale[g]) + shift[g], g = row // rows_per_group."""
    M, C = x.shape
    _check(load().wf_layer_norm_modulate(plan.handle, M, C, _ptr(x), _ptr(shift), _ptr(scale),
                                         rows_per_group, _ptr(y), _stream(stream)),
           "wf_layer_norm_modulate")


def wf_sync_status(plan: Plan, stream=None) -> int:
    """Returns the status code (WF_OK or WF_ERR_TIMEOUT ...) without raising."""
    return int(load().wf_sync_status(plan.handle, _stream(stream)))


def wf_plan_debug_ranges(plan: Plan, round_: int):
    """List of (wave chunk, logical index, absolute chunk id, ring slot) in visiting order."""
    lib = load()
    n = lib.wf_plan_debug_ranges(plan.handle, round_, None, 0)
    if n < 0:
        raise WFError(WF_ERR_INVALID_ARG, "wf_plan_debug_ranges")
    buf = (ctypes.c_int32 * (4 * max(n, 1)))()
    lib.wf_plan_debug_ranges(plan.handle, round_, buf, n)
    return [tuple(buf[4 * i:4 * i + 4]) for i in range(n)]


def wf_chunk_causal_attn_noalloc(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim,
                                 round_, q_out, k_cache, v_cache, o, lse=None,
                                 stream=None) -> None:
    """Attention without a plan, for callers that must not allocate device memory
    (see include/wf.h): the kernel's scratch lives in a block compiled into the
    library, shared by every call on the device."""
    _check(load().wf_chunk_causal_attn_noalloc(chunk_tokens, n_wave_chunks, n_hist_chunks,
                                               heads, head_dim, round_, _ptr(q_out),
                                               _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                               _stream(stream)), "wf_chunk_causal_attn_noalloc")


def wf_causal_conv3d(plan: Plan, x, x_hist, w, bias, resid, y, stream=None) -> None:
    """Causal 3x3x3 convolution of one chunk: x [T,H,W,Cin] bf16, x_hist [2,H,W,Cin]
    or None (start of the video), w [Cout,3,3,3,Cin] bf16, bias [Cout] f32 or None,
    resid [T,H,W,Cout] or None, y [T,H,W,Cout] bf16."""
    T, H, W, Cin = x.shape
    Cout = w.shape[0]
    _check(load().wf_causal_conv3d(plan.handle, T, H, W, Cin, Cout, _ptr(x), _ptr(x_hist),
                                   _ptr(w), _ptr(bias), _ptr(resid), _ptr(y), _stream(stream)),
           "wf_causal_conv3d")


def wf_rms_norm_silu(plan: Plan, x, gamma, y, stream=None) -> None:
    """Per-pixel RMSNorm over the last axis with gain gamma, then SiLU (bf16 in/out)."""
    C = x.shape[-1]
    M = x.numel() // C
    _check(load().wf_rms_norm_silu(plan.handle, M, C, _ptr(x), _ptr(gamma), _ptr(y),
                                   _stream(stream)), "wf_rms_norm_silu")
