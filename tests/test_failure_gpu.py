"""Failure detection on the GPU without a fault.

Every mbarrier wait in the attention kernel is bounded.  The test hook
wf_plan_set_withhold_q makes the producer skip each CTA's first Q-tile copy, so
the MMA warp waits on a barrier phase that nothing will complete: the wait runs
out after the plan's limit (a short one here), the kernel drains its own
copies and MMAs, frees TMEM and returns, and wf_sync_status reports
WF_ERR_TIMEOUT.  Nothing traps or faults; the same context then computes the
next call correctly.
"""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_attention_close, rand_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


@pytest.mark.parametrize("kind", ["WF_ATTN_SINGLE", "WF_ATTN_PAIR"])
def test_expired_wait_reports_timeout_and_context_survives(wf, kind):
    L, W, Hh, H, D, r = 300, 4, 2, 3, 128, 5
    R = W + Hh
    q = rand_bf16((W * L, H, D), 1)
    kc = rand_bf16((R, L, H, D), 2)
    vc = rand_bf16((R, L, H, D), 3)
    o = torch.empty_like(q)
    plan = wf.Plan(L, W, Hh, H, D).set_attn_kernel(getattr(wf, kind))
    plan.set_wait_limit(1 << 24).set_withhold_q(True)    # ~10 ms of SM clock
    wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o, None)
    assert wf.wf_sync_status(plan) == wf.WF_ERR_TIMEOUT
    assert wf.wf_sync_status(plan) == wf.WF_OK           # reading clears the status
    # the same plan and context compute the next call correctly
    plan.set_withhold_q(False).set_wait_limit(0)
    wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o, None)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    cache = oracle.OracleCache(L)
    kb, vb = wi.bits(kc.cpu()), wi.bits(vc.cpu())
    for g in range(r - min(Hh, r), r + W):
        cache.put(g, kb[g % R], vb[g % R])
    rows = np.repeat(np.arange(W * L), H)
    heads = np.tile(np.arange(H), W * L)
    ref, _ = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    assert_attention_close(o.float().cpu().numpy().reshape(-1, D), ref, "after timeout")
    plan.destroy()
