"""C-ABI checks that need no GPU: symbols, argument validation, host-side logic.

The ring/visibility arithmetic that wf_plan_debug_ranges reports is the same
function the attention kernel calls; here it is checked against the oracle's
cache model, which keys chunks by absolute id and has no ring.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from chunk_causal_dit_b200 import build as wf_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    mod.load()
    return mod


def header_functions():
    text = open(os.path.join(ROOT, "include", "wf.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wf_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(wf):
    names = header_functions()
    assert len(names) >= 13
    lib = ctypes.CDLL(wf.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(wf.SIGNATURES), "binding and header disagree"


def test_plan_argument_validation(wf):
    lib = wf.load()
    h = ctypes.c_void_p()
    bad = [(0, 5, 2, 12, 128), (4680, 0, 2, 12, 128), (4680, 5, -1, 12, 128),
           (4680, 5, 2, 0, 128)]
    for args in bad:
        assert lib.wf_plan(*args, ctypes.byref(h)) == wf.WF_ERR_INVALID_ARG
        assert h.value is None
    assert lib.wf_plan(4680, 5, 2, 12, 96, ctypes.byref(h)) == wf.WF_ERR_UNSUPPORTED
    # too large for 32-bit element indexing of one [T,H,D] tensor
    assert lib.wf_plan(1 << 20, 64, 0, 64, 128, ctypes.byref(h)) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_plan(4680, 5, 2, 12, 128, None) == wf.WF_ERR_INVALID_ARG


def test_plan_setters_validate(wf):
    p = wf.Plan(4680, 5, 2, 12, 128)
    with pytest.raises(wf.WFError):
        p.set_rope(3, 30, 51)              # 3*30*51 != 4680
    p.set_rope(3, 30, 52)
    with pytest.raises(wf.WFError):
        p.set_rope_split(44, 42, 40)       # sum != D
    with pytest.raises(wf.WFError):
        p.set_rope_split(43, 43, 42)       # odd widths
    p.set_rope_split(44, 42, 42)
    with pytest.raises(wf.WFError):
        p.set_norm_eps(-1.0)
    p.set_norm_eps(1e-5)
    for kind in (wf.WF_ATTN_SINGLE, wf.WF_ATTN_PAIR, wf.WF_ATTN_AUTO):
        p.set_attn_kernel(kind)
    with pytest.raises(wf.WFError):
        p.set_attn_kernel(3)
    p.destroy()
    p64 = wf.Plan(32, 3, 0, 2, 64)
    p64.set_attn_kernel(wf.WF_ATTN_SINGLE)
    with pytest.raises(wf.WFError) as e:
        p64.set_attn_kernel(wf.WF_ATTN_PAIR)   # the pair kernel is head_dim 128 only
    assert e.value.status == wf.WF_ERR_UNSUPPORTED
    p64.destroy()


@pytest.mark.parametrize("L,W,Hh,H,D", [(32, 3, 0, 2, 64), (4680, 5, 2, 12, 128),
                                        (4680, 6, 3, 12, 128), (4680, 5, 3, 40, 128),
                                        (100, 4, 7, 3, 64)])
def test_useful_flops_and_cache_bytes(wf, L, W, Hh, H, D):
    p = wf.Plan(L, W, Hh, H, D)
    for r in (0, 1, 2, 3, 10):
        assert wf.wf_useful_flops(p, r) == oracle.useful_flops(L, W, Hh, H, D, r)
    assert wf.wf_cache_bytes(p) == (Hh + W) * L * H * D * 2
    p.destroy()


def test_useful_flops_headline_value(wf):
    # 12 heads x 128, 4680-token chunks, 5-chunk wave, 2 history chunks: 3.364 TFLOP
    p = wf.Plan(4680, 5, 2, 12, 128)
    assert abs(wf.wf_useful_flops(p, 2) - 3.3644e12) < 0.001e12
    p.destroy()


@pytest.mark.parametrize("W,Hh", [(3, 0), (5, 2), (6, 3), (2, 5)])
def test_debug_ranges_match_oracle_cache_model(wf, W, Hh):
    L, H = 4, 1
    p = wf.Plan(L, W, Hh, H, 64)
    R = W + Hh
    cache = oracle.OracleCache(L)
    for r in range(0, 2 * R + 3):
        got = wf.wf_plan_debug_ranges(p, r)
        # oracle: ids visible to wave chunk c are the round's history then chunks r..r+c
        for i in range(r - min(Hh, r), r + W):
            cache.put(i, np.zeros((L, H, 64), np.uint16), np.zeros((L, H, 64), np.uint16))
        _, _, ids = cache.round_keys(r, W, Hh)
        hv = len(ids) - W
        want = []
        for c in range(W):
            for b, cid in enumerate(ids[:hv + c + 1]):
                want.append((c, b, int(cid), int(cid) % R))
        assert got == want
        # within one round every visible chunk has its own slot
        slots = {s for (_, _, _, s) in got}
        assert len(slots) == len(ids)


def test_hot_calls_without_device(wf):
    import torch
    if torch.cuda.is_available():
        pytest.skip("device present")
    p = wf.Plan(32, 3, 0, 2, 64)
    lib = wf.load()
    fake = 1 << 20   # never dereferenced: the call fails before any launch
    assert lib.wf_chunk_causal_attn(p.handle, 0, fake, fake, fake, fake, None, None) == \
        wf.WF_ERR_NO_DEVICE
    assert lib.wf_qk_norm_rope_append(p.handle, 0, fake, fake, fake, None, fake, fake, fake,
                                      fake, fake, None) == wf.WF_ERR_INVALID_ARG  # no geometry
    p.set_rope(2, 4, 4)
    assert lib.wf_qk_norm_rope_append(p.handle, 0, fake, fake, fake, None, fake, fake, fake,
                                      fake, fake, None) == wf.WF_ERR_NO_DEVICE
    # misaligned pointers are rejected before the device check
    assert lib.wf_chunk_causal_attn(p.handle, 0, fake + 2, fake, fake, fake, None, None) == \
        wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn(p.handle, -1, fake, fake, fake, fake, None, None) == \
        wf.WF_ERR_INVALID_ARG
    p.destroy()


def test_fp8_calls_validate_before_the_device(wf):
    """The FP8 entry points: argument checks (NULL, alignment, chunk range,
    head_dim) come before any device access; with valid arguments and no GPU the
    calls report WF_ERR_NO_DEVICE."""
    import torch
    lib = wf.load()
    fake = 1 << 20
    p = wf.Plan(300, 4, 2, 3, 128)
    # head_dim 64 is unsupported by the FP8 attention, whatever the pointers
    p64 = wf.Plan(32, 3, 0, 2, 64)
    assert lib.wf_chunk_causal_attn_fp8qk(p64.handle, 0, fake, fake, fake, fake, fake, fake,
                                          None, None) == wf.WF_ERR_UNSUPPORTED
    assert lib.wf_chunk_causal_attn_fp8qk(p.handle, 0, None, fake, fake, fake, fake, fake,
                                          None, None) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn_fp8qk(p.handle, 0, fake + 8, fake, fake, fake, fake, fake,
                                          None, None) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn_fp8qk(p.handle, 0, fake, fake + 2, fake, fake, fake, fake,
                                          None, None) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_quantize_q_fp8(p.handle, fake, fake + 4, fake, None) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_quantize_k_fp8(p.handle, 0, 7, fake, fake, fake, None) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_quantize_k_fp8(p.handle, -1, 1, fake, fake, fake, None) == wf.WF_ERR_INVALID_ARG
    if not torch.cuda.is_available():
        assert lib.wf_quantize_q_fp8(p.handle, fake, fake, fake, None) == wf.WF_ERR_NO_DEVICE
        assert lib.wf_quantize_k_fp8(p.handle, 3, 6, fake, fake, fake, None) == \
            wf.WF_ERR_NO_DEVICE
        assert lib.wf_chunk_causal_attn_fp8qk(p.handle, 0, fake, fake, fake, fake, fake, fake,
                                              None, None) == wf.WF_ERR_NO_DEVICE
    p.destroy()
    p64.destroy()


def test_status_strings(wf):
    assert wf.status_string(0) == "ok"
    assert "timed out" in wf.status_string(wf.WF_ERR_TIMEOUT)
    assert wf.status_string(999) == "unknown status"


def test_block_calls_validate_before_the_device(wf):
    """wf_linear, wf_qkv_proj_norm_rope_append and wf_layer_norm_modulate: sizes,
    epilogue codes, NULL and misaligned pointers, a missing RoPE grid and shapes the
    kernels do not cover are reported before any device access; valid calls on a
    machine without a GPU report WF_ERR_NO_DEVICE."""
    import torch
    lib = wf.load()
    f = 1 << 20
    p = wf.Plan(32, 1, 0, 1, 64)
    E = wf.WF_ERR_INVALID_ARG
    lin = lib.wf_linear
    assert lin(p.handle, 10, 48, 64, f, f, None, 0, None, None, 1, f, None) == E   # N % 32
    assert lin(p.handle, 10, 64, 60, f, f, None, 0, None, None, 1, f, None) == E   # K % 8
    assert lin(p.handle, -1, 64, 64, f, f, None, 0, None, None, 1, f, None) == E
    assert lin(p.handle, 10, 64, 64, f, f, None, 3, None, None, 1, f, None) == E   # epilogue
    assert lin(p.handle, 10, 64, 64, f + 8, f, None, 0, None, None, 1, f, None) == E
    assert lin(p.handle, 10, 64, 64, f, f, f + 4, 0, None, None, 1, f, None) == E  # bias align
    assert lin(p.handle, 10, 64, 64, f, f, None, 2, None, f, 1, f, None) == E      # no gate
    assert lin(p.handle, 10, 64, 64, f, f, None, 2, f, f, 0, f, None) == E         # rows/group
    qkv = lib.wf_qkv_proj_norm_rope_append
    pg = wf.Plan(300, 3, 1, 2, 128)                       # no grid set yet
    assert qkv(pg.handle, 0, 256, f, f, None, f, f, f, f, f, None) == E
    pg.set_rope(2, 6, 25)
    assert qkv(pg.handle, 0, 250, f, f, None, f, f, f, f, f, None) == E             # hidden % 8
    assert qkv(pg.handle, -1, 256, f, f, None, f, f, f, f, f, None) == E
    assert qkv(pg.handle, 0, 256, f, f, None, f, None, f, f, f, None) == E
    p1 = wf.Plan(64, 2, 0, 1, 64).set_rope(1, 8, 8)      # H*D = 64: not a multiple of 128
    assert qkv(p1.handle, 0, 64, f, f, None, f, f, f, f, f, None) == wf.WF_ERR_UNSUPPORTED
    big = wf.Plan(64 * 64, 1, 0, 2, 64).set_rope(1, 64, 64)   # 12 + 640 + 640 entries: fits
    wide = wf.Plan(1 * 4000, 1, 0, 2, 64).set_rope(1, 1, 4000)  # w table 4000 * 5 > 3072
    assert qkv(wide.handle, 0, 64, f, f, None, f, f, f, f, f, None) == wf.WF_ERR_UNSUPPORTED
    ln = lib.wf_layer_norm_modulate
    assert ln(p.handle, 10, 12, f, f, f, 1, f, None) == E                          # C % 8
    assert ln(p.handle, 10, 6152, f, f, f, 1, f, None) == wf.WF_ERR_UNSUPPORTED
    assert ln(p.handle, 10, 64, f, f, f, 0, f, None) == E
    assert ln(p.handle, 10, 64, f, f + 4, f, 1, f, None) == E
    if not torch.cuda.is_available():
        N = wf.WF_ERR_NO_DEVICE
        assert lin(p.handle, 10, 64, 64, f, f, None, 0, None, None, 1, f, None) == N
        assert lin(p.handle, 10, 64, 64, f, f, f, 2, f, f, 3, f, None) == N
        assert qkv(pg.handle, 0, 256, f, f, None, f, f, f, f, f, None) == N
        assert qkv(big.handle, 0, 64, f, f, f, f, f, f, f, f, None) == N
        assert ln(p.handle, 10, 64, f, f, f, 1, f, None) == N
    for q in (p, pg, p1, big, wide):
        q.destroy()


def test_debug_build_exports_the_same_abi():
    """libwf_check.so (the WF_CHECK variant) loads without a GPU, exports every
    function the header declares, and names the status its checks report."""
    import ctypes
    import re
    from chunk_causal_dit_b200 import build as wf_build
    path = wf_build.build(check=True)
    lib = ctypes.CDLL(path)
    with open(os.path.join(ROOT, "include", "wf.h")) as f:
        names = set(re.findall(r"WF_API\s+[^()]*?\b(wf_[a-z0-9_]+)\s*\(", f.read()))
    assert names and all(hasattr(lib, n) for n in names)
    lib.wf_status_string.restype = ctypes.c_char_p
    assert b"bounds" in lib.wf_status_string(7)
