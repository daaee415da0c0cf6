"""wf_chunk_causal_attn_noalloc against the plan API, through the C ABI.

The no-alloc entry point is for callers that must not allocate device memory
(a serving loop whose memory belongs to a caching allocator or was reserved up
front): it takes the shape directly and keeps the kernel's scratch in a block
compiled into the library.  Its result must match wf_plan + wf_chunk_causal_attn
on the same inputs, within the attention tolerance, on two calls in a row (the
second call reuses the scratch the first one left behind).

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from chunk_causal_dit_b200 import build as wf_build
from tests.wfcase import assert_attention_close, rand_bf16

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


@pytest.mark.parametrize("L,W,Hh,H,D,r", CASES)
def test_noalloc_matches_plan_api_twice(wf, L, W, Hh, H, D, r):
    lib = wf.load()
    q, kc, vc = _inputs(L, W, Hh, H, D, seed=L + D)
    T = W * L
    plan = wf.Plan(L, W, Hh, H, D)
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((H, T), dtype=torch.float32, device=q.device)
    wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o_ref, lse_ref)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()
    ref = o_ref.double().cpu().numpy().reshape(-1, D)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=q.device)
        rc = lib.wf_chunk_causal_attn_noalloc(L, W, Hh, H, D, r, q.data_ptr(), kc.data_ptr(),
                                              vc.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                              stream)
        assert rc == wf.WF_OK, wf.status_string(rc)
        torch.cuda.synchronize()
        got = o.float().cpu().numpy().reshape(-1, D)
        assert np.isfinite(got).all()
        assert_attention_close(got, ref, "no-alloc call %d" % call)
        assert float((lse - lse_ref).abs().max()) <= 1e-3


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
