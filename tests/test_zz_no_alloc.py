"""wf_chunk_causal_attn_noalloc through the C ABI: against the fp64 oracle and
against the plan API, and without allocating.

The no-alloc entry point is for callers that must not allocate device memory
(a serving loop whose memory belongs to a caching allocator or was reserved up
front): it takes the shape directly and keeps the kernel's scratch in a block
compiled into the library.  On two calls in a row (the second reuses the
scratch the first one left behind) its output must
- match the oracle's chunk-causal attention on sampled rows (chunk and tile
  boundaries plus random rows) within the attention bar, and lse within 1e-3;
- match wf_plan + wf_chunk_causal_attn on every row within the same bar;
and every call after the first must leave the device's free memory and
PyTorch's allocator statistics unchanged.  A call after the scratch block was
left dirty (every word set, through the library's test hook, as a timed-out
call leaves status, timeout site and work counter) must still match the oracle.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_attention_close, rand_bf16, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    mod.load()
    return mod


CASES = [
    # L, W, Hh, H, D, round
    (300, 4, 2, 3, 128, 5),
    (200, 3, 1, 2, 64, 7),
    (4680 // 4, 5, 2, 4, 128, 2),
]


def _inputs(L, W, Hh, H, D, seed):
    R = Hh + W
    return (rand_bf16((W * L, H, D), seed), rand_bf16((R, L, H, D), seed + 1),
            rand_bf16((R, L, H, D), seed + 2))


def _oracle_cache(kc, vc, round_, W, Hh):
    """The oracle's absolute-id view of the ring (slot g mod R holds chunk g)."""
    R, L = kc.shape[0], kc.shape[1]
    cache = oracle.OracleCache(L)
    kb, vb = wi.bits(kc.cpu()), wi.bits(vc.cpu())
    for g in range(round_ - min(Hh, round_), round_ + W):
        cache.put(g, kb[g % R], vb[g % R])
    return cache


def _alloc_state():
    torch.cuda.synchronize()
    free, _ = torch.cuda.mem_get_info()
    st = torch.cuda.memory_stats()
    keys = ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current")
    return free, {k: st.get(k, 0) for k in keys}


@pytest.mark.parametrize("L,W,Hh,H,D,r", CASES)
def test_noalloc_matches_oracle_and_plan_api_twice(wf, L, W, Hh, H, D, r):
    lib = wf.load()
    q, kc, vc = _inputs(L, W, Hh, H, D, seed=L + D)
    T = W * L

    # the oracle on sampled rows, every head
    rows_s = sample_rows(L, W, n_random=24, seed=L)
    rows = np.repeat(rows_s, H)
    heads = np.tile(np.arange(H), rows_s.size)
    cache = _oracle_cache(kc, vc, r, W, Hh)
    o_orc, lse_orc = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)

    # the plan API on the same inputs
    plan = wf.Plan(L, W, Hh, H, D)
    o_ref = torch.empty_like(q)
    wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o_ref, None)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()
    ref = o_ref.double().cpu().numpy().reshape(-1, D)

    stream = torch.cuda.current_stream().cuda_stream
    # outputs allocated before the first call; nothing is allocated in the loop
    outs = [torch.full_like(q, float("nan")) for _ in range(2)]
    lses = [torch.full((H, T), float("nan"), dtype=torch.float32, device=q.device)
            for _ in range(2)]
    for call in range(2):
        o, lse = outs[call], lses[call]
        before = _alloc_state()
        rc = lib.wf_chunk_causal_attn_noalloc(L, W, Hh, H, D, r, q.data_ptr(), kc.data_ptr(),
                                              vc.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                              stream)
        assert rc == wf.WF_OK, wf.status_string(rc)
        after = _alloc_state()
        if call > 0:
            # the first call may load the module's code; later calls change nothing
            assert after == before, "no-alloc call %d changed device memory: %r -> %r" % (
                call, before, after)
        got = o.cpu().float().numpy().reshape(T, H, D)   # no device temporaries
        assert np.isfinite(got).all()
        what = "no-alloc call %d L=%d W=%d Hh=%d D=%d r=%d" % (call, L, W, Hh, D, r)
        assert_attention_close(got[rows, heads], o_orc, what + " vs oracle")
        lse_got = lse.cpu().numpy()[heads, rows]
        assert float(np.abs(lse_got - lse_orc).max()) <= 1e-3
        assert_attention_close(got.reshape(-1, D), ref, what + " vs plan API")


def test_noalloc_after_a_dirty_scratch_block(wf):
    """A call after one that left the scratch block dirty (status and timeout
    site set, the work counter past the last unit: what a timed-out call
    leaves) clears what must start at zero and matches the oracle."""
    lib = wf.load()
    L, W, Hh, H, D, r = 300, 4, 2, 3, 128, 5
    q, kc, vc = _inputs(L, W, Hh, H, D, seed=99)
    T = W * L
    rows_s = sample_rows(L, W, n_random=24, seed=5)
    rows = np.repeat(rows_s, H)
    heads = np.tile(np.arange(H), rows_s.size)
    cache = _oracle_cache(kc, vc, r, W, Hh)
    o_orc, lse_orc = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    stream = torch.cuda.current_stream().cuda_stream
    for word in (0xFFFFFFFF, 0x7FFFFFFF, 1):
        torch.cuda.synchronize()
        assert lib.wf_noalloc_debug_fill_scratch(word) == wf.WF_OK
        o = torch.full_like(q, float("nan"))
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=q.device)
        rc = lib.wf_chunk_causal_attn_noalloc(L, W, Hh, H, D, r, q.data_ptr(), kc.data_ptr(),
                                              vc.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                              stream)
        assert rc == wf.WF_OK, wf.status_string(rc)
        got = o.cpu().float().numpy().reshape(T, H, D)
        assert np.isfinite(got).all(), "fill %#x: rows left unwritten" % word
        assert_attention_close(got[rows, heads], o_orc, "after fill %#x vs oracle" % word)
        assert float(np.abs(lse.cpu().numpy()[heads, rows] - lse_orc).max()) <= 1e-3
        assert lib.wf_noalloc_sync_status(stream) == wf.WF_OK


def test_noalloc_status_query(wf):
    """wf_noalloc_sync_status maps the block's status word the way wf_sync_status
    maps a plan's: the timeout bit to WF_ERR_TIMEOUT, the bounds bit to
    WF_ERR_BOUNDS (the words are planted through the test hook; no kernel is
    made to time out), and a call that ran clean to WF_OK."""
    lib = wf.load()
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    for word, want in ((1, wf.WF_ERR_TIMEOUT), (2, wf.WF_ERR_BOUNDS), (3, wf.WF_ERR_TIMEOUT),
                       (0, wf.WF_OK)):
        assert lib.wf_noalloc_debug_fill_scratch(word) == wf.WF_OK
        assert lib.wf_noalloc_sync_status(stream) == want, word
    # a call clears the status left behind
    assert lib.wf_noalloc_debug_fill_scratch(1) == wf.WF_OK
    L, W, Hh, H, D, r = 200, 3, 1, 2, 64, 7
    q, kc, vc = _inputs(L, W, Hh, H, D, seed=3)
    o = torch.empty_like(q)
    rc = lib.wf_chunk_causal_attn_noalloc(L, W, Hh, H, D, r, q.data_ptr(), kc.data_ptr(),
                                          vc.data_ptr(), o.data_ptr(), None, stream)
    assert rc == wf.WF_OK
    assert lib.wf_noalloc_sync_status(stream) == wf.WF_OK


def test_noalloc_rejects_what_the_plan_rejects(wf):
    lib = wf.load()
    fake = 1 << 20          # never dereferenced: each call fails before any launch
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.wf_chunk_causal_attn_noalloc(300, 4, 2, 3, 96, 0, fake, fake, fake, fake, None,
                                            stream) == wf.WF_ERR_UNSUPPORTED
    assert lib.wf_chunk_causal_attn_noalloc(1 << 20, 64, 0, 64, 128, 0, fake, fake, fake, fake,
                                            None, stream) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn_noalloc(300, 4, 2, 3, 128, -1, fake, fake, fake, fake, None,
                                            stream) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn_noalloc(300, 4, 2, 3, 128, 0, fake + 8, fake, fake, fake,
                                            None, stream) == wf.WF_ERR_INVALID_ARG
    assert lib.wf_chunk_causal_attn_noalloc(300, 4, 2, 3, 128, 0, fake, fake, fake, fake,
                                            ctypes.c_void_p(fake + 2), stream) == \
        wf.WF_ERR_INVALID_ARG
