"""Wave Parallelism's per-rank decomposition on one GPU, without collectives.

Every rank's plan (its chunks as the wave, the global history plus the earlier
wave chunks as its history, round r + c0) runs the libwf kernels on its own
ring; device copies stand in for the one-way delivery (``incoming``), and no
kernel waits on another.  Each rank's output rows must equal, bit for bit, the
single-GPU round's rows of the same chunks: the append computes the same
positions, and the attention visits the same key tiles in the same order.  Two
consecutive rounds check that the refresh chunk delivered in the first is the
history of the second.
"""
import pytest
import torch

from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


@pytest.mark.parametrize("world,Hh", [(1, 2), (2, 2), (3, 2), (5, 2), (5, 0), (2, 0)])
def test_emulated_ranks_equal_single_wave(wf, world, Hh):
    from chunk_causal_dit_b200.wave_parallel import LibwfKernels, WaveParallelRound
    dev = "cuda"
    F, gh, gw, W, H, D = 2, 6, 25, 5, 2, 128
    L = F * gh * gw
    R = Hh + W
    rounds = 2
    gq, gk = (t.to(dev) for t in wi.gains(H, D, 1))
    xs = [tuple(wi.bf16_normal((W * L, H, D), 10 + i, s).to(dev) for s in range(3))
          for i in range(rounds)]
    hk = wi.bf16_normal((Hh, L, H, D), 7, 3).to(dev)
    hv = wi.bf16_normal((Hh, L, H, D), 7, 4).to(dev)
    r0 = Hh

    # the single-GPU round
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    kc = torch.zeros((R, L, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    for j in range(Hh):
        kc[(r0 - Hh + j) % R].copy_(hk[j])
        vc[(r0 - Hh + j) % R].copy_(hv[j])
    want = []
    for i in range(rounds):
        q, k, v = xs[i]
        q_out, o = torch.empty_like(q), torch.empty_like(q)
        wf.wf_qk_norm_rope_append(plan, r0 + i, q, k, v, None, gq, gk, q_out, kc, vc)
        wf.wf_chunk_causal_attn(plan, r0 + i, q_out, kc, vc, o)
        want.append(o)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()

    # the ranks, one after another
    kern = LibwfKernels(gq, gk)
    ranks = [WaveParallelRound(L, W, Hh, H, D, (F, gh, gw), kern, world=world, rank=k)
             for k in range(world)]
    rings = []
    for wp in ranks:
        rk = torch.zeros(wp.ring_shape(), dtype=torch.bfloat16, device=dev)
        rv = torch.zeros_like(rk)
        wp.prefill_history(r0, [(r0 - Hh + j, hk[j], hv[j]) for j in range(Hh)], rk, rv)
        rings.append((rk, rv))
    for i in range(rounds):
        r = r0 + i
        q, k, v = xs[i]
        q_outs = []
        for wp, (rk, rv) in zip(ranks, rings):
            rows = slice(wp.c0 * L, wp.c1 * L)
            q_out = torch.empty((wp.rows, H, D), dtype=torch.bfloat16, device=dev)
            kern.append(wp.plan, r + wp.c0, q[rows].contiguous(), k[rows].contiguous(),
                        v[rows].contiguous(), q_out, rk, rv)
            q_outs.append(q_out)
        for wp, (rk, rv) in zip(ranks, rings):                 # the one-way delivery
            for src, g in wp.incoming(r):
                sk, sv = rings[src]
                rk[wp.slot(g)].copy_(sk[ranks[src].slot(g)])
                rv[wp.slot(g)].copy_(sv[ranks[src].slot(g)])
        for wp, (rk, rv), q_out in zip(ranks, rings, q_outs):
            o = torch.empty_like(q_out)
            kern.attention(wp.plan, r + wp.c0, q_out, rk, rv, o)
            torch.cuda.synchronize()
            assert wf.wf_sync_status(wp.plan) == wf.WF_OK
            got = o.view(torch.int16)
            ref = want[i][wp.c0 * L:wp.c1 * L].view(torch.int16)
            assert torch.equal(got, ref), "world %d rank %d round %d" % (world, wp.rank, r)
    for wp in ranks:
        wp.destroy()
