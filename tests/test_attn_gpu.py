"""GPU parity of wf_chunk_causal_attn against the fp64 oracle.

Bars (unit-scale data, fp32 accumulation, bf16 output): max abs error <= 1e-2
and mean abs error <= 1e-3 per case; lse within 1e-3.  Chunk visibility and
ring indexing are exact: perturbing a later chunk leaves earlier chunks'
outputs bit-identical, and rounds that wrap the ring match the oracle's
absolute-id cache model.
"""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import (assert_attention_close, assert_attention_close_scaled,
                          assert_attention_within_rounding, rand_bf16, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def place_round(L, W, Hh, H, D, round_, seed):
    """Random q_out and a ring whose slot (g mod R) holds absolute chunk g."""
    R = Hh + W
    q = rand_bf16((W * L, H, D), seed)
    kc = rand_bf16((R, L, H, D), seed + 1)
    vc = rand_bf16((R, L, H, D), seed + 2)
    return q, kc, vc


def oracle_cache_from_ring(kc, vc, round_, W, Hh):
    """The oracle's absolute-id view of a ring laid out by the header contract."""
    L = kc.shape[1]
    R = kc.shape[0]
    cache = oracle.OracleCache(L)
    kb, vb = wi.bits(kc.cpu()), wi.bits(vc.cpu())
    for g in range(round_ - min(Hh, round_), round_ + W):
        cache.put(g, kb[g % R], vb[g % R])
    return cache


KERNELS = ["single", "pair"]


def make_plan(wf, L, W, Hh, H, D, kernel):
    kind = {"single": wf.WF_ATTN_SINGLE, "pair": wf.WF_ATTN_PAIR}[kernel]
    return wf.Plan(L, W, Hh, H, D).set_attn_kernel(kind)


def run_attn(wf, plan, round_, q, kc, vc, with_lse=True):
    T, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=q.device) if with_lse else None
    wf.wf_chunk_causal_attn(plan, round_, q, kc, vc, o, lse)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    return o, lse


SHAPES = [
    # L, W, Hh, H, D, round
    (300, 4, 2, 3, 128, 5),     # ragged chunk: 2 full tiles + 44 rows
    (200, 3, 1, 2, 64, 7),      # head_dim 64, ragged
    (128, 2, 0, 1, 128, 0),     # exactly one tile, no history
    (129, 3, 3, 2, 128, 1),     # one row past a tile; pipeline filling (1 of 3 history)
    (1, 3, 1, 2, 64, 4),        # one token per chunk
    (513, 2, 2, 1, 128, 9),     # 5 tiles, last with 1 row; odd number of query tiles
    (32, 3, 0, 2, 64, 0),       # the tiny wave shape
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("L,W,Hh,H,D,r", SHAPES)
def test_attention_all_rows(wf, L, W, Hh, H, D, r, kernel):
    if kernel == "pair" and D != 128:
        pytest.skip("the pair kernel is built for head_dim 128")
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=L + W + D)
    plan = make_plan(wf, L, W, Hh, H, D, kernel)
    o, lse = run_attn(wf, plan, r, q, kc, vc)
    cache = oracle_cache_from_ring(kc, vc, r, W, Hh)
    T = W * L
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    o_ref, lse_ref = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    o_gpu = o.float().cpu().numpy().reshape(T * H, D)
    what = "O L=%d W=%d Hh=%d D=%d r=%d" % (L, W, Hh, D, r)
    if L * (min(Hh, r) + 1) >= 32:
        assert_attention_close(o_gpu, o_ref, what)
    else:   # a handful of visible keys per row: the elementwise rounding bound
        v_absmax = float(vc.float().abs().max())
        assert_attention_within_rounding(o_gpu, o_ref, v_absmax, what)
    lse_gpu = lse.cpu().numpy().T.reshape(-1)
    assert np.max(np.abs(lse_gpu - lse_ref)) <= 1e-3
    plan.destroy()


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("L,H,D", [(300, 2, 128), (700, 1, 128), (200, 3, 64)])
def test_single_chunk_equals_bidirectional_attention(wf, L, H, D, kernel):
    """One wave chunk and no history: chunk-causal attention is plain
    bidirectional softmax attention over the chunk.  Checked against PyTorch's
    scaled_dot_product_attention in fp64 on the same bf16 values (a library
    route independent of the oracle) and against the oracle."""
    if kernel == "pair" and D != 128:
        pytest.skip("the pair kernel is built for head_dim 128")
    q, kc, vc = place_round(L, 1, 0, H, D, 0, seed=L + 7 * H)
    plan = make_plan(wf, L, 1, 0, H, D, kernel)
    o, lse = run_attn(wf, plan, 0, q, kc, vc)
    qd = q.cpu().double().permute(1, 0, 2)            # [H, L, D]
    kd = kc[0].cpu().double().permute(1, 0, 2)
    vd = vc[0].cpu().double().permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qd[None], kd[None], vd[None])[0]
    ref = ref.permute(1, 0, 2).reshape(L * H, D).numpy()
    got = o.float().cpu().numpy().reshape(L * H, D)
    assert_attention_close(got, ref, "single chunk vs sdpa L=%d D=%d" % (L, D))
    s_ = torch.einsum("hld,hmd->hlm", qd, kd) / np.sqrt(D)
    lse_ref = torch.logsumexp(s_, dim=-1).numpy()     # [H, L]
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= 1e-3
    plan.destroy()


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("D", [128, 64])
def test_score_jump_far_above_the_running_reference(wf, D, kernel):
    """Keys built to score far above everything a row saw before (by ~90-130
    log2 units), in the first and in the second half of a later key tile: the
    online softmax must move the row's reference and rescale O and l, with no
    overflow and no loss of the earlier tiles' weights."""
    if kernel == "pair" and D != 128:
        pytest.skip("the pair kernel is built for head_dim 128")
    L, W, Hh, H, r = 600, 2, 0, 2, 0
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=41)
    n1, n2, n3 = L + 5, L + 300, 17          # queries in chunk 1, 1 and 0
    big = 8.0
    # chunk 0, key tile 1, column 10 (first half): aligned with n1 and n3
    kc[0, 138, 0] = (big * q[n1, 0].float()).to(torch.bfloat16)
    kc[0, 140, 1] = (big * q[n3, 1].float()).to(torch.bfloat16)
    # chunk 1, key tile 3, column 100 (second half): aligned with n2 and n1
    kc[1, 484, 0] = (big * q[n2, 0].float()).to(torch.bfloat16)
    kc[1, 490, 1] = (big * q[n1, 1].float()).to(torch.bfloat16)
    plan = make_plan(wf, L, W, Hh, H, D, kernel)
    o, lse = run_attn(wf, plan, r, q, kc, vc)
    cache = oracle_cache_from_ring(kc, vc, r, W, Hh)
    T = W * L
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    ref, lse_ref = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    got = o.float().cpu().numpy().reshape(T * H, D)
    assert np.isfinite(got).all()
    targets = ((n1, 0, (0, 138)), (n2, 0, (1, 484)), (n1, 1, (1, 490)), (n3, 1, (0, 140)))
    hit = np.zeros(T * H, bool)
    for n, h, _ in targets:
        hit[n * H + h] = True
    # The big keys also pull rows that merely correlate with the targeted
    # queries towards a single V row, so |O| reaches ~4.5 where one bf16
    # rounding alone exceeds the 1e-2 max-abs bar: elements with |O| > 1 are
    # held to the elementwise rounding bound, the rest to the 1e-2 bar, and
    # all together to the mean bar.
    v_absmax = float(vc.float().abs().max())
    assert_attention_close_scaled(got, ref, v_absmax, "score jump D=%d" % D)
    for n, h, key in targets:
        v = vc[key[0], key[1], h].float().cpu().numpy()
        assert np.max(np.abs(o[n, h].float().cpu().numpy() - v)) <= 2.0 ** -6 * np.abs(v).max()
    lse_gpu = lse.cpu().numpy().T.reshape(-1)
    assert np.max(np.abs(lse_gpu - lse_ref)) <= 1e-3
    plan.destroy()


@pytest.mark.parametrize("kernel", KERNELS)
def test_causality_perturbation_bit_identical(wf, kernel):
    L, W, Hh, H, D, r = 200, 4, 2, 2, 128, 6
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=5)
    plan = make_plan(wf, L, W, Hh, H, D, kernel)
    base, _ = run_attn(wf, plan, r, q, kc, vc)
    R = W + Hh
    for j in range(W):
        kc2, vc2 = kc.clone(), vc.clone()
        slot = (r + j) % R
        kc2[slot] = rand_bf16((L, H, D), 100 + j)
        vc2[slot] = rand_bf16((L, H, D), 200 + j)
        pert, _ = run_attn(wf, plan, r, q, kc2, vc2)
        assert torch.equal(pert[:j * L].view(torch.int16), base[:j * L].view(torch.int16))
        assert not torch.equal(pert[j * L:], base[j * L:])
    plan.destroy()


@pytest.mark.parametrize("kernel", KERNELS)
def test_repeat_runs_bit_identical(wf, kernel):
    L, W, Hh, H, D, r = 4680 // 4, 5, 2, 4, 128, 2
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=9)
    plan = make_plan(wf, L, W, Hh, H, D, kernel)
    first, lse0 = run_attn(wf, plan, r, q, kc, vc)
    for _ in range(5):
        again, lse1 = run_attn(wf, plan, r, q, kc, vc)
        assert torch.equal(again.view(torch.int16), first.view(torch.int16))
        assert torch.equal(lse1, lse0)
    plan.destroy()


@pytest.mark.parametrize("L,W,Hh,H,D,r", [(300, 3, 2, 7, 128, 4), (200, 3, 1, 5, 64, 3)])
def test_head_blocks_all_rows(wf, L, W, Hh, H, D, r):
    """Every head-block order of the work units gives bit-identical outputs
    (each unit computes the same rows in the same order), and they match the
    oracle on every row."""
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=31 + D)
    plan = wf.Plan(L, W, Hh, H, D)
    outs = {}
    for g in (H, 1, 2, 3, 0):
        plan.set_head_block(g)
        assert plan.head_block(r) == g if g else 1 <= plan.head_block(r) <= H
        o = torch.full_like(q, float("nan"))
        lse = torch.full((H, W * L), float("nan"), dtype=torch.float32, device=q.device)
        wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o, lse)
        torch.cuda.synchronize()
        assert wf.wf_sync_status(plan) == wf.WF_OK
        outs[g] = (o, lse)
    o0, lse0 = outs[H]
    for g, (o, lse) in outs.items():
        assert torch.equal(o.view(torch.int16), o0.view(torch.int16)), "head block %d" % g
        assert torch.equal(lse, lse0), "head block %d" % g
    cache = oracle_cache_from_ring(kc, vc, r, W, Hh)
    T = W * L
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    o_ref, lse_ref = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    o_gpu = outs[2][0].float().cpu().numpy().reshape(T * H, D)
    assert_attention_close(o_gpu, o_ref, "head blocks L=%d H=%d D=%d" % (L, H, D))
    assert np.max(np.abs(outs[2][1].cpu().numpy().T.reshape(-1) - lse_ref)) <= 1e-3
    plan.destroy()


def test_head_blocks_more_units_than_ctas(wf):
    """A round with more work units than SMs, so that CTAs take several units
    and the blocks follow one another through the global counter: every
    head-block order gives the same bits, and no row is left unwritten."""
    L, W, Hh, H, D, r = 1000, 4, 2, 12, 128, 3
    q, kc, vc = place_round(L, W, Hh, H, D, r, seed=77)
    plan = wf.Plan(L, W, Hh, H, D)
    ref = None
    for g in (H, 1, 2, 3, 5, 0):
        plan.set_head_block(g)
        o = torch.full_like(q, float("nan"))
        wf.wf_chunk_causal_attn(plan, r, q, kc, vc, o, None)
        torch.cuda.synchronize()
        assert wf.wf_sync_status(plan) == wf.WF_OK
        assert not torch.isnan(o).any(), "head block %d left rows unwritten" % g
        if ref is None:
            ref = o
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), "head block %d" % g
    # sampled rows of the last chunk (the longest units) against the oracle
    cache = oracle_cache_from_ring(kc, vc, r, W, Hh)
    rows = np.repeat(np.array([(W - 1) * L, (W - 1) * L + 511, W * L - 1]), H)
    heads = np.tile(np.arange(H), 3)
    o_ref, _ = oracle.round_attention(cache, r, W, Hh, wi.bits(q.cpu()), rows, heads)
    got = ref.float().cpu().numpy()[rows, heads]
    assert_attention_close(got, o_ref, "head blocks, sampled rows")
    plan.destroy()


def test_ring_over_rounds_end_to_end(wf):
    # append + attention for rounds 0 .. 2R+1 against the oracle's absolute-id cache
    w = wi.Workload("ring", H=2, D=64, F=1, gh=5, gw=8, n_wave=3, n_hist=2)
    dev = "cuda"
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    cache = oracle.OracleCache(w.L)
    rows = np.repeat(np.arange(w.T), w.H)
    heads = np.tile(np.arange(w.H), w.T)
    for r in range(2 * w.R + 2):
        x = wi.wave_inputs(w, seed=0, salt=r)
        q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
        o = torch.empty_like(q_out)
        wf.wf_qk_norm_rope_append(plan, r, x.q.to(dev), x.k.to(dev), x.v.to(dev), None,
                                  x.gamma_q.to(dev), x.gamma_k.to(dev), q_out, kc, vc)
        wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None)
        torch.cuda.synchronize()
        assert wf.wf_sync_status(plan) == wf.WF_OK
        pos = oracle.positions(r, w.n_wave, w.F, w.gh, w.gw)
        qo, ko, vo = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos,
                                   x.gamma_q.numpy(), x.gamma_k.numpy())
        cache.put_wave(r, ko, vo)
        o_ref, _ = oracle.round_attention(cache, r, w.n_wave, w.n_hist, qo, rows, heads)
        assert_attention_close(o.float().cpu().numpy().reshape(-1, w.D), o_ref, "round %d" % r)
    plan.destroy()


def test_tiny_wave_end_to_end_and_isolated(wf):
    w = wi.WORKLOADS["tiny"]
    dev = "cuda"
    x = wi.wave_inputs(w, seed=0)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    o = torch.empty_like(q_out)
    wf.wf_qk_norm_rope_append(plan, 0, x.q.to(dev), x.k.to(dev), x.v.to(dev), None,
                              x.gamma_q.to(dev), x.gamma_k.to(dev), q_out, kc, vc)
    wf.wf_chunk_causal_attn(plan, 0, q_out, kc, vc, o, None)
    torch.cuda.synchronize()
    rows = np.repeat(np.arange(w.T), w.H)
    heads = np.tile(np.arange(w.H), w.T)
    # isolated: the oracle attends over the GPU's own q_out / K' / V
    cache = oracle_cache_from_ring(kc, vc, 0, w.n_wave, w.n_hist)
    o_iso, _ = oracle.round_attention(cache, 0, w.n_wave, w.n_hist, wi.bits(q_out.cpu()),
                                      rows, heads)
    got = o.float().cpu().numpy().reshape(-1, w.D)
    assert_attention_close(got, o_iso, "tiny isolated")
    # end to end: the oracle's own append feeds its attention
    pos = oracle.positions(0, w.n_wave, w.F, w.gh, w.gw)
    qo, ko, vo = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos,
                               x.gamma_q.numpy(), x.gamma_k.numpy())
    cache2 = oracle.OracleCache(w.L)
    cache2.put_wave(0, ko, vo)
    o_e2e, _ = oracle.round_attention(cache2, 0, w.n_wave, w.n_hist, qo, rows, heads)
    assert_attention_close(got, o_e2e, "tiny end to end")
    plan.destroy()


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name,head_sel", [("wan13b_4step", None), ("wan13b_5step", [0, 5, 11]),
                                           ("wan14b_4step", [0, 1, 22, 39])])
def test_full_size_sampled(wf, name, head_sel, kernel):
    """Full-size round r = n_hist (steady state), the launch the benchmark times;
    checked on rows at chunk and tile boundaries plus random rows."""
    w = wi.WORKLOADS[name]
    dev = "cuda"
    r = w.n_hist
    x = wi.wave_inputs(w, seed=0)
    hk, hv = wi.history_prefill(w, seed=0)
    plan = make_plan(wf, w.L, w.n_wave, w.n_hist, w.H, w.D, kernel).set_rope(w.F, w.gh, w.gw)
    kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    for j in range(w.n_hist):                 # history chunk ids 0 .. n_hist-1
        kc[j % w.R] = hk[j].to(dev)
        vc[j % w.R] = hv[j].to(dev)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q_out)
    lse = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
    wf.wf_qk_norm_rope_append(plan, r, x.q.to(dev), x.k.to(dev), x.v.to(dev), None,
                              x.gamma_q.to(dev), x.gamma_k.to(dev), q_out, kc, vc)
    wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, lse)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    cache = oracle_cache_from_ring(kc, vc, r, w.n_wave, w.n_hist)
    sel = sample_rows(w.L, w.n_wave, 48, seed=1)
    hs = list(range(w.H)) if head_sel is None else head_sel
    rows = np.repeat(sel, len(hs))
    heads = np.tile(hs, len(sel))
    o_ref, lse_ref = oracle.round_attention(cache, r, w.n_wave, w.n_hist,
                                            wi.bits(q_out.cpu()), rows, heads)
    o_all = o.float().cpu().numpy()
    got = o_all[rows, heads]
    assert_attention_close(got, o_ref, name)
    lse_all = lse.cpu().numpy()
    assert np.max(np.abs(lse_all[heads, rows] - lse_ref)) <= 1e-3
    assert np.isfinite(o_all).all()
    plan.destroy()
