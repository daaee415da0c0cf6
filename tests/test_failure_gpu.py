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


@pytest.mark.parametrize("call", ["linear", "qkv"])
def test_gemm_expired_wait_reports_timeout_and_context_survives(wf, call):
    """The CTA-pair GEMM's bounded waits: with the first K slice withheld the
    MMA's wait expires, both CTAs stop (copies drained, TMEM freed) and the call
    reports WF_ERR_TIMEOUT; the next call on the same plan is correct."""
    import oracle.block as ob
    dev = "cuda"
    F, gh, gw, W, Hh, H, D, C = 2, 6, 25, 3, 1, 2, 128, 256
    L, T = F * gh * gw, W * F * gh * gw
    x = wi.bf16_normal((T, C), 4, wi.STREAM_X)
    w_qkv = wi.bf16_weight(3 * H * D, C, 4)
    gq, gk = wi.gains(H, D, 4)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    q_out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((W + Hh, L, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    y = torch.empty((T, 3 * H * D), dtype=torch.bfloat16, device=dev)

    def run():
        if call == "linear":
            wf.wf_linear(plan, x.to(dev), w_qkv.to(dev), y)
        else:
            wf.wf_qkv_proj_norm_rope_append(plan, 1, x.to(dev), w_qkv.to(dev), None,
                                            gq.to(dev), gk.to(dev), q_out, kc, vc)

    plan.set_wait_limit(1 << 24).set_withhold_q(True)     # ~10 ms of SM clock
    run()
    assert wf.wf_sync_status(plan) == wf.WF_ERR_TIMEOUT
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.set_withhold_q(False).set_wait_limit(0)
    run()
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref = ob.linear_f64(wi.bits(x), wi.bits(w_qkv))
    if call == "linear":
        got = y.float().cpu().numpy()
    else:   # v is the projection itself, rounded once
        got = torch.cat([vc[(1 + c) % (W + Hh)] for c in range(W)]).float().cpu().numpy()
        got = got.reshape(T, H * D)
        ref = ref[:, 2 * H * D:]
    assert np.abs(got - ref).max() <= 2.0 ** -6     # bf16 rounding of values up to ~4
    plan.destroy()
