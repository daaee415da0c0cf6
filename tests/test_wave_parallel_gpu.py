"""Wave Parallelism's per-rank decomposition on one GPU, without collectives.

Every rank's plan (its chunks as the wave, the global history plus the earlier
wave chunks as its history, round r + c0) runs the libwf kernels on its own
ring; device copies stand in for the one-way delivery (``incoming``), and no
kernel waits on another.  Each rank's output rows must
- match the fp64 oracle's round (its own append feeding its own attention, or
  its DiT block, over the whole wave, with its absolute-id cache) on sampled
  rows at chunk and tile boundaries plus random rows, within the parity bars;
- equal, bit for bit, the single-GPU round's rows of the same chunks: the
  append computes the same positions, and the attention visits the same key
  tiles in the same order.
Two consecutive rounds check that the refresh chunk delivered in the first is
the history of the second.  Starting at round 0 (no history yet) makes every
rank's window, min(Hh + c0, r + c0) chunks, fill up as the rounds advance.
"""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_attention_close, bf16_quantum, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def _bits(t):
    return wi.bits(t.cpu())


@pytest.mark.parametrize("world,Hh,r0", [(1, 2, 2), (2, 2, 2), (3, 2, 2), (5, 2, 2), (5, 0, 0),
                                         (2, 0, 0), (3, 2, 0), (5, 3, 1)])
def test_emulated_ranks_equal_single_wave(wf, world, Hh, r0):
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
    # history chunks that exist before round r0 (ids >= 0)
    hist = [(r0 - Hh + j, hk[j], hv[j]) for j in range(Hh) if r0 - Hh + j >= 0]

    # the oracle's rounds: its own append feeds its own attention
    cache = oracle.OracleCache(L)
    for g, kk, vv in hist:
        cache.put(g, _bits(kk), _bits(vv))
    sel = sample_rows(L, W, 24, seed=world + 7 * Hh + r0)
    rows = np.repeat(sel, H)
    heads = np.tile(np.arange(H), sel.size)
    o_orc = []
    for i in range(rounds):
        q, k, v = xs[i]
        pos = oracle.positions(r0 + i, W, F, gh, gw)
        qo, ko, vo = oracle.append(_bits(q), _bits(k), _bits(v), pos, gq.cpu().numpy(),
                                   gk.cpu().numpy())
        cache.put_wave(r0 + i, ko, vo)
        o_orc.append(oracle.round_attention(cache, r0 + i, W, Hh, qo, rows, heads)[0])

    # the single-GPU round
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    kc = torch.zeros((R, L, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    for g, kk, vv in hist:
        kc[g % R].copy_(kk)
        vc[g % R].copy_(vv)
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
        wp.prefill_history(r0, hist, rk, rv)
        rings.append((rk, rv))
    for i in range(rounds):
        r = r0 + i
        q, k, v = xs[i]
        q_outs = []
        for wp, (rk, rv) in zip(ranks, rings):
            own = slice(wp.c0 * L, wp.c1 * L)
            q_out = torch.empty((wp.rows, H, D), dtype=torch.bfloat16, device=dev)
            kern.append(wp.plan, r + wp.c0, q[own].contiguous(), k[own].contiguous(),
                        v[own].contiguous(), q_out, rk, rv)
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
            # against the oracle, on the sampled rows this rank owns
            mine = (rows >= wp.c0 * L) & (rows < wp.c1 * L)
            got_o = o.cpu().float().numpy()[rows[mine] - wp.c0 * L, heads[mine]]
            assert_attention_close(got_o, o_orc[i][mine],
                                   "world %d rank %d round %d vs oracle" % (world, wp.rank, r))
            # and bit for bit against the single-GPU round
            got = o.view(torch.int16)
            ref = want[i][wp.c0 * L:wp.c1 * L].view(torch.int16)
            assert torch.equal(got, ref), "world %d rank %d round %d" % (world, wp.rank, r)
    for wp in ranks:
        wp.destroy()


@pytest.mark.parametrize("world,r0", [(2, 2), (5, 2), (3, 0)])
def test_emulated_ranks_run_the_block_like_one_gpu(wf, world, r0):
    """The whole DiT block per rank (LayerNorm, fused QKV projection, delivery,
    attention, output projection, feed-forward), ranks emulated one after another
    with device copies for the delivery, over two rounds:
    - every rank's residual rows match oracle.block.block_forward over the whole
      wave (bar of the composed block: two bf16 quanta + 1e-2 per element, mean
      1e-3; the stored residual stream rounds twice and the attention's error
      reaches it through W_o and a gate of ~0.1);
    - and equal the single-GPU block's, bit for bit.  (Each GEMM element sums K
      in the same order whatever the row tiling; LayerNorm is per row; the
      attention visits the same key tiles.)"""
    import oracle.block as ob
    from chunk_causal_dit_b200.wave_parallel import LibwfKernels, WaveParallelRound
    dev = "cuda"
    F, gh, gw, W, Hh, H, D, C, FF = 2, 6, 25, 5, 2, 2, 128, 256, 512
    L, T, R = F * gh * gw, W * F * gh * gw, Hh + W
    s = 17
    w = {"w_qkv": wi.bf16_weight(3 * H * D, C, s, 1), "w_o": wi.bf16_weight(C, H * D, s, 2),
         "w_1": wi.bf16_weight(FF, C, s, 3), "w_2": wi.bf16_weight(C, FF, s, 4),
         "b_qkv": wi.f32_vector((3 * H * D,), 0.02, s, wi.STREAM_BIAS, 1),
         "b_o": wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 2),
         "b_1": wi.f32_vector((FF,), 0.02, s, wi.STREAM_BIAS, 3),
         "b_2": wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 4)}
    w = {k: t.to(dev) for k, t in w.items()}
    mod = wi.f32_vector((6, W, C), 0.1, s, wi.STREAM_MOD).to(dev)
    gq, gk = (t.to(dev) for t in wi.gains(H, D, s))
    xs = [wi.bf16_normal((T, C), s + i, wi.STREAM_X).to(dev) for i in range(2)]
    hk = wi.bf16_normal((Hh, L, H, D), s, 3).to(dev)
    hv = wi.bf16_normal((Hh, L, H, D), s, 4).to(dev)
    kern = LibwfKernels(gq, gk)
    hist = [(r0 - Hh + j, hk[j], hv[j]) for j in range(Hh) if r0 - Hh + j >= 0]

    # the oracle's blocks over the whole wave
    cache = oracle.OracleCache(L)
    for g, kk, vv in hist:
        cache.put(g, _bits(kk), _bits(vv))
    bw = {k: (_bits(t) if t.dtype == torch.bfloat16 else t.cpu().numpy()) for k, t in w.items()}
    bw["gamma_q"], bw["gamma_k"] = gq.cpu().numpy(), gk.cpu().numpy()
    x_orc = []
    for i in range(2):
        x2, _ = ob.block_forward(_bits(xs[i]), bw, mod.cpu().numpy(),
                                 oracle.positions(r0 + i, W, F, gh, gw), cache, r0 + i, W, Hh,
                                 H, D, L)
        x_orc.append(oracle.bf16_to_f64(x2))

    def buffers(rows, ring_shape):
        return {"h": torch.empty((rows, C), dtype=torch.bfloat16, device=dev),
                "q_out": torch.empty((rows, H, D), dtype=torch.bfloat16, device=dev),
                "o": torch.empty((rows, H, D), dtype=torch.bfloat16, device=dev),
                "f": torch.empty((rows, FF), dtype=torch.bfloat16, device=dev),
                "k_cache": torch.zeros(ring_shape, dtype=torch.bfloat16, device=dev),
                "v_cache": torch.zeros(ring_shape, dtype=torch.bfloat16, device=dev)}

    def prefill(wp, buf):
        wp.prefill_history(r0, hist, buf["k_cache"], buf["v_cache"])

    one = WaveParallelRound(L, W, Hh, H, D, (F, gh, gw), kern, world=1, rank=0)
    b1 = buffers(one.rows, one.ring_shape())
    prefill(one, b1)
    ranks = [WaveParallelRound(L, W, Hh, H, D, (F, gh, gw), kern, world=world, rank=k)
             for k in range(world)]
    bufs = [buffers(wp.rows, wp.ring_shape()) for wp in ranks]
    for wp, b in zip(ranks, bufs):
        prefill(wp, b)
    for i in range(2):
        r = r0 + i
        X1 = xs[i].clone()
        one.run_block(r, X1, w, mod, b1)
        Xs = [xs[i][wp.c0 * L:wp.c1 * L].clone() for wp in ranks]
        ms = [wp.mod_rows(mod) for wp in ranks]
        for wp, b, X, m in zip(ranks, bufs, Xs, ms):
            wp.norm_and_qkv(r, X, w, m, b)
        for wp, b in zip(ranks, bufs):                       # the one-way delivery
            for src, g in wp.incoming(r):
                sb = bufs[src]
                b["k_cache"][wp.slot(g)].copy_(sb["k_cache"][ranks[src].slot(g)])
                b["v_cache"][wp.slot(g)].copy_(sb["v_cache"][ranks[src].slot(g)])
        for wp, b, X, m in zip(ranks, bufs, Xs, ms):
            wp.attention_and_rest(r, X, w, m, b)
        torch.cuda.synchronize()
        for wp, X in zip(ranks, Xs):
            assert wf.wf_sync_status(wp.plan) == wf.WF_OK
            want = x_orc[i][wp.c0 * L:wp.c1 * L]
            diff = np.abs(X.cpu().double().numpy() - want)
            tol = 2.0 * bf16_quantum(want) + 1e-2
            assert not (diff > tol).any(), "world %d rank %d round %d: %d outside the bar" % (
                world, wp.rank, r, int((diff > tol).sum()))
            assert diff.mean() <= 1e-3, "world %d rank %d round %d: mean %g" % (
                world, wp.rank, r, diff.mean())
            ref = X1[wp.c0 * L:wp.c1 * L]
            assert torch.equal(X.view(torch.int16), ref.view(torch.int16)), \
                "world %d rank %d round %d" % (world, wp.rank, r)
    for wp in ranks + [one]:
        wp.destroy()
