"""GPU checks of the FP8 (E4M3) Q.K^T path through the C ABI.

* Quantization is integer work: q8 / q_scale and k8 / k_scale must equal the
  oracle's rule bit for bit (codes and fp32 scales), including ragged last key
  tiles, all-zero groups and chunks that land in wrapped ring slots; slots that
  are not quantized stay untouched.
* Attention: against the oracle's FP8 route (E4M3 q and k dequantized exactly by
  their scales, bf16 v) the kernel must meet the bf16 attention bars, since the
  E4M3 products are exact in fp32 and only the accumulation order, the bf16
  rounding of P and of O differ.  Against the exact bf16 oracle the gap is the
  quantization error itself; its bar (mean abs <= 4e-3, max abs <= 4e-2 on
  unit-normal data) follows from the E4M3 step: half an ulp is 2^-4 relative,
  ~3.6% RMS per element, so a score over D = 128 products moves by ~0.05 and a
  weight by ~5%, which averages over the hundreds of visible keys of these
  shapes to a few 1e-3 on O.
"""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_attention_close, rand_bf16, sample_rows

pytestmark = pytest.mark.gpu

FP8_VS_EXACT_MEAN = 4e-3
FP8_VS_EXACT_MAX = 4e-2


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def _bits(t):
    return wi.bits(t.cpu())


def _quantize_all(wf, plan, q, kc, first, n):
    T, H, D = q.shape
    R, L = kc.shape[0], kc.shape[1]
    nt = (L + 127) // 128
    q8 = torch.empty((T, H, D), dtype=torch.uint8, device=q.device)
    qs = torch.empty((H, T), dtype=torch.float32, device=q.device)
    k8 = torch.full((R, L, H, D), 0xAA, dtype=torch.uint8, device=q.device)
    ks = torch.full((R, nt, H), -1.0, dtype=torch.float32, device=q.device)
    wf.wf_quantize_q_fp8(plan, q, q8, qs)
    wf.wf_quantize_k_fp8(plan, first, n, kc, k8, ks)
    torch.cuda.synchronize()
    return q8, qs, k8, ks


@pytest.mark.parametrize("L,W,Hh,H,D", [(300, 4, 2, 3, 128), (200, 3, 1, 2, 64), (128, 2, 0, 1, 128)])
def test_quantization_bit_exact(wf, L, W, Hh, H, D):
    R = W + Hh
    q = rand_bf16((W * L, H, D), 11)
    q[5] = 0                                              # all-zero rows: scale 1, codes 0
    q[7, 0] = q[7, 0] * 1e-3                              # small row
    kc = rand_bf16((R, L, H, D), 12)
    kc[1 % R, 128:256, 0] = kc[1 % R, 128:256, 0] * 300.0   # one loud tile
    kc[2 % R, :, H - 1] = 0                                 # an all-zero head
    plan = wf.Plan(L, W, Hh, H, D)
    first, n = 3, W                                       # chunks 3.. wrap around the ring
    q8, qs, k8, ks = _quantize_all(wf, plan, q, kc, first, n)
    rq8, rqs = oracle.quantize_rows_fp8(_bits(q))
    assert np.array_equal(q8.cpu().numpy(), rq8)
    assert np.array_equal(qs.cpu().numpy(), rqs)
    k8h, ksh, kb = k8.cpu().numpy(), ks.cpu().numpy(), _bits(kc)
    done = set()
    for g in range(first, first + n):
        slot = g % R
        done.add(slot)
        c8, cs = oracle.quantize_tiles_fp8(kb[slot])
        assert np.array_equal(k8h[slot], c8), "codes of chunk %d" % g
        assert np.array_equal(ksh[slot], cs), "scales of chunk %d" % g
    for slot in set(range(R)) - done:
        assert (k8h[slot] == 0xAA).all() and (ksh[slot] == -1.0).all()
    plan.destroy()


SHAPES = [
    # L, W, Hh, H, round
    (300, 4, 2, 3, 5),      # ragged chunk
    (129, 3, 3, 2, 1),      # one row past a tile, pipeline filling
    (513, 2, 2, 1, 9),      # odd number of query tiles
    (128, 2, 0, 1, 0),      # one tile, no history
    (300, 1, 0, 2, 0),      # a single chunk: plain bidirectional attention
]


@pytest.mark.parametrize("L,W,Hh,H,r", SHAPES)
def test_attention_fp8qk(wf, L, W, Hh, H, r):
    D = 128
    R = W + Hh
    q = rand_bf16((W * L, H, D), L + 1)
    kc = rand_bf16((R, L, H, D), L + 2)
    vc = rand_bf16((R, L, H, D), L + 3)
    plan = wf.Plan(L, W, Hh, H, D)
    q8, qs, k8, ks = _quantize_all(wf, plan, q, kc, 0, R)        # every slot
    o = torch.empty_like(q)
    lse = torch.empty((H, W * L), dtype=torch.float32, device=q.device)
    wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o, lse)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    kb, vb = _bits(kc), _bits(vc)
    cache8 = oracle.OracleCacheFP8(L)
    cache = oracle.OracleCache(L)
    k8h, ksh = k8.cpu().numpy(), ks.cpu().numpy()
    for g in range(r - min(Hh, r), r + W):
        cache8.put(g, k8h[g % R], ksh[g % R], vb[g % R])
        cache.put(g, kb[g % R], vb[g % R])
    T = W * L
    rows = np.repeat(np.arange(T), H)
    heads = np.tile(np.arange(H), T)
    ref8, lse8 = oracle.round_attention_fp8qk(cache8, r, W, Hh, q8.cpu().numpy(),
                                              qs.cpu().numpy(), rows, heads)
    got = o.float().cpu().numpy().reshape(T * H, D)
    assert_attention_close(got, ref8, "fp8qk vs oracle fp8 route L=%d r=%d" % (L, r))
    lse_gpu = lse.cpu().numpy().T.reshape(-1)
    assert np.max(np.abs(lse_gpu - lse8)) <= 1e-3
    ref, _ = oracle.round_attention(cache, r, W, Hh, _bits(q), rows, heads)
    d = np.abs(got - ref)
    assert d.mean() <= FP8_VS_EXACT_MEAN and d.max() <= FP8_VS_EXACT_MAX, \
        "quantization error: mean %.3g max %.3g" % (d.mean(), d.max())
    plan.destroy()


def test_fp8qk_repeat_bit_identical_and_head_dim_64_unsupported(wf):
    L, W, Hh, H, r = 4680 // 4, 5, 2, 4, 2
    D, R = 128, 7
    q = rand_bf16((W * L, H, D), 21)
    kc = rand_bf16((R, L, H, D), 22)
    vc = rand_bf16((R, L, H, D), 23)
    plan = wf.Plan(L, W, Hh, H, D)
    q8, qs, k8, ks = _quantize_all(wf, plan, q, kc, 0, R)
    o0, o1 = torch.empty_like(q), torch.empty_like(q)
    wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o0)
    for _ in range(3):
        wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o1)
        torch.cuda.synchronize()
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    # every head-block order of the units gives the same bits
    for g in (1, 3, H):
        plan.set_head_block(g)
        o1.fill_(float("nan"))
        wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o1)
        torch.cuda.synchronize()
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16)), "head block %d" % g
    plan.destroy()
    p64 = wf.Plan(200, 3, 1, 2, 64)
    with pytest.raises(wf.WFError) as e:
        wf.wf_chunk_causal_attn_fp8qk(p64, 1, q8, qs, k8, ks, vc, o0)
    assert e.value.status == wf.WF_ERR_UNSUPPORTED
    p64.destroy()


def test_full_size_sampled_fp8qk(wf):
    """Wan-1.3B 4-step wave at steady state: append, quantize, FP8 attention;
    sampled rows against the oracle's FP8 route."""
    w = wi.WORKLOADS["wan13b_4step"]
    dev = "cuda"
    r = w.n_hist
    x = wi.wave_inputs(w, seed=0)
    hk, hv = wi.history_prefill(w, seed=0)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    for j in range(w.n_hist):
        kc[j % w.R] = hk[j].to(dev)
        vc[j % w.R] = hv[j].to(dev)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    wf.wf_qk_norm_rope_append(plan, r, x.q.to(dev), x.k.to(dev), x.v.to(dev), None,
                              x.gamma_q.to(dev), x.gamma_k.to(dev), q_out, kc, vc)
    nt = (w.L + 127) // 128
    q8 = torch.empty((w.T, w.H, w.D), dtype=torch.uint8, device=dev)
    qs = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
    k8 = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.uint8, device=dev)
    ks = torch.empty((w.R, nt, w.H), dtype=torch.float32, device=dev)
    wf.wf_quantize_k_fp8(plan, 0, w.n_hist, kc, k8, ks)         # history, appended earlier
    wf.wf_quantize_q_fp8(plan, q_out, q8, qs)
    wf.wf_quantize_k_fp8(plan, r, w.n_wave, kc, k8, ks)         # this round's wave
    o = torch.empty_like(q_out)
    lse = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
    wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o, lse)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    cache8 = oracle.OracleCacheFP8(w.L)
    k8h, ksh, vb = k8.cpu().numpy(), ks.cpu().numpy(), _bits(vc)
    for g in range(r - w.n_hist, r + w.n_wave):
        cache8.put(g, k8h[g % w.R], ksh[g % w.R], vb[g % w.R])
    sel = sample_rows(w.L, w.n_wave, 32, seed=2)
    hs = [0, 5, 11]
    rows = np.repeat(sel, len(hs))
    heads = np.tile(hs, len(sel))
    ref, lse_ref = oracle.round_attention_fp8qk(cache8, r, w.n_wave, w.n_hist, q8.cpu().numpy(),
                                                qs.cpu().numpy(), rows, heads)
    o_all = o.float().cpu().numpy()
    assert_attention_close(o_all[rows, heads], ref, "fp8qk full size")
    assert np.max(np.abs(lse.cpu().numpy()[heads, rows] - lse_ref)) <= 1e-3
    assert np.isfinite(o_all).all()
    plan.destroy()


@pytest.mark.parametrize("L,W,Hh,H,D,r,with_q_out", [(300, 4, 2, 3, 128, 5, True),
                                                     (200, 3, 1, 2, 64, 2, True),
                                                     (4680 // 4, 5, 2, 12, 128, 2, False)])
def test_fused_append_quantization_bit_exact(wf, L, W, Hh, H, D, r, with_q_out):
    """wf_qk_norm_rope_append_fp8q: the ring writes equal the plain append's bit for
    bit, q_out (when given) too, and q8 / q_scale equal the oracle's row rule applied
    to that bf16 q_out (and so the stand-alone wf_quantize_q_fp8 on it)."""
    T, R = W * L, W + Hh
    F, gh, gw = 1, 1, L                      # a row of patches per chunk: positions derived
    x = [rand_bf16((T, H, D), 30 + i) for i in range(3)]
    x[0][3] = 0                              # an all-zero q row: its q' is zero, scale 1
    gq, gk = (t.cuda() for t in wi.gains(H, D, 4))
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    kc0 = torch.full((R, L, H, D), 1.5, dtype=torch.bfloat16, device="cuda")
    vc0 = torch.full_like(kc0, -2.0)
    kc1, vc1 = kc0.clone(), vc0.clone()
    q_ref = torch.empty_like(x[0])
    wf.wf_qk_norm_rope_append(plan, r, x[0], x[1], x[2], None, gq, gk, q_ref, kc0, vc0)
    q_out = torch.full_like(x[0], float("nan")) if with_q_out else None
    q8 = torch.full((T, H, D), 0xAA, dtype=torch.uint8, device="cuda")
    qs = torch.full((H, T), -1.0, dtype=torch.float32, device="cuda")
    wf.wf_qk_norm_rope_append_fp8q(plan, r, x[0], x[1], x[2], None, gq, gk, q_out, q8, qs, kc1, vc1)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    assert torch.equal(kc1.view(torch.int16), kc0.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc0.view(torch.int16))
    if with_q_out:
        assert torch.equal(q_out.view(torch.int16), q_ref.view(torch.int16))
    rq8, rqs = oracle.quantize_rows_fp8(_bits(q_ref))
    assert np.array_equal(q8.cpu().numpy(), rq8)
    assert np.array_equal(qs.cpu().numpy(), rqs)
    assert float(qs[0, 3]) == 1.0            # the zero row
    plan.destroy()
