"""GPU parity of the DiT-block calls (tcgen05 GEMM with fused epilogues, LayerNorm
with modulation) against the fp64 oracle in oracle/block.py, through the C ABI.

Bars (per element, against the oracle's exact value y):
* a GEMM output: |got - y| <= one bf16 quantum of y + 2^-20 * S, where
  S = sum_k |x_k w_k| bounds the fp32 accumulation error of the tensor-core sum
  (2^-24 per addition, over a few dozen additions of partial sums of size S);
* q and k of the fused QKV projection: the same accumulation term carried
  through the RMSNorm (times |gamma| / rms of the head's projection), plus the
  fp32 rotation term 2^-20 * |pair| of the stand-alone append;
* LayerNorm: one bf16 quantum + 2^-18 * (|x_hat (1 + scale)| + |shift|).
Shapes span several tiles, ragged M (rows past M in a tile), N not a multiple
of 256 (a half-empty column tile), K with a ragged last 64-slice, and the full
Wan-1.3B widths (sampled rows).
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.block as ob
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import bf16_quantum, pair_norm

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def _bits(t):
    return wi.bits(t.cpu())


def _f64(t):
    return t.cpu().double().numpy()


def _assert_gemm_close(got_bits, ref_f64, S, what):
    g = wi.from_bits(got_bits).double().numpy()
    r = oracle.bf16_to_f64(oracle.f64_to_bf16(ref_f64))
    tol = bf16_quantum(r) * 1.0000001 + 2.0 ** -20 * S
    d = np.abs(g - ref_f64)
    bad = d > tol
    assert not bad.any(), "%s: %d of %d outside the bar (worst excess %g)" % (
        what, int(bad.sum()), bad.size, float((d - tol).max()))
    return float((got_bits != oracle.f64_to_bf16(ref_f64)).mean())


def _abs_sum(x, w):
    return np.abs(_f64(x)) @ np.abs(_f64(w)).T


def _assert_qk_close(got_bits, ref64, y_head, S_head, gamma, what):
    """q or k [n, H, D]: one bf16 quantum, the rotation's fp32 term and the
    accumulation term 2^-20 * S carried through the norm (x |gamma| / rms)."""
    rms = np.sqrt((y_head ** 2).mean(axis=-1, keepdims=True))
    acc = 2.0 ** -20 * S_head.max(axis=-1, keepdims=True) / rms * \
        np.abs(gamma.numpy().astype(np.float64)).max(axis=-1)[None, :, None]
    g = wi.from_bits(got_bits).double().numpy()
    r_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(ref64))
    tol = bf16_quantum(r_bf) * 1.0000001 + 2.0 ** -20 * pair_norm(ref64) + acc
    d = np.abs(g - ref64)
    assert not (d > tol).any(), "%s: %d values outside the bar (worst excess %g)" % (
        what, int((d > tol).sum()), float((d - tol).max()))


LINEAR_SHAPES = [
    # M, N, K
    (300, 256, 64),        # one column tile, ragged M (rows 300..511 of the tile unused)
    (513, 96, 200),        # N < 256 (a partial column tile), ragged K slice (200 = 3*64 + 8)
    (1000, 768, 1536),     # several tiles both ways, Wan-1.3B width K
    (256, 1280, 136),      # exact M, K ragged again
]


@pytest.mark.parametrize("M,N,K", LINEAR_SHAPES)
@pytest.mark.parametrize("epi", ["store", "gelu_tanh", "gated_residual"])
def test_linear_parity(wf, M, N, K, epi):
    dev = "cuda"
    seed = M + 7 * N + 13 * K
    x = wi.bf16_normal((M, K), seed, wi.STREAM_X)
    w = wi.bf16_weight(N, K, seed)
    bias = wi.f32_vector((N,), 0.5, seed, wi.STREAM_BIAS)
    rpg = 97
    G = (M + rpg - 1) // rpg
    gate = wi.f32_vector((G, N), 1.0, seed, wi.STREAM_MOD)
    resid = wi.bf16_normal((M, N), seed, wi.STREAM_V)
    code = {"store": wf.WF_EPI_STORE, "gelu_tanh": wf.WF_EPI_GELU_TANH,
            "gated_residual": wf.WF_EPI_GATED_RESIDUAL}[epi]
    plan = wf.Plan(32, 1, 0, 1, 64)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    gr = epi == "gated_residual"
    wf.wf_linear(plan, x.to(dev), w.to(dev), y, bias.to(dev), code,
                 gate.to(dev) if gr else None, resid.to(dev) if gr else None, rpg)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref = ob.linear_f64(_bits(x), _bits(w), bias.numpy(), epi, gate.numpy() if gr else None,
                        _bits(resid) if gr else None, rpg)
    S = _abs_sum(x, w)
    if gr:
        S = S * np.abs(gate.numpy().astype(np.float64))[np.arange(M) // rpg]
    _assert_gemm_close(_bits(y), ref, S, "linear %s %dx%dx%d" % (epi, M, N, K))
    plan.destroy()


def test_linear_in_place_residual_and_empty(wf):
    """y may be the residual buffer (the block's residual update); M = 0 is a no-op."""
    dev = "cuda"
    M, N, K = 300, 256, 128
    x = wi.bf16_normal((M, K), 3, wi.STREAM_X)
    w = wi.bf16_weight(N, K, 3)
    gate = wi.f32_vector((1, N), 1.0, 3, wi.STREAM_MOD)
    r0 = wi.bf16_normal((M, N), 3, wi.STREAM_V)
    r = r0.to(dev)
    plan = wf.Plan(32, 1, 0, 1, 64)
    wf.wf_linear(plan, x.to(dev), w.to(dev), r, None, wf.WF_EPI_GATED_RESIDUAL, gate.to(dev), r, M)
    ref = ob.linear_f64(_bits(x), _bits(w), None, "gated_residual", gate.numpy(), _bits(r0), M)
    S = _abs_sum(x, w) * np.abs(gate.numpy().astype(np.float64))
    _assert_gemm_close(_bits(r), ref, S, "in-place gated residual")
    e = torch.empty((0, N), dtype=torch.bfloat16, device=dev)
    wf.wf_linear(plan, torch.empty((0, K), dtype=torch.bfloat16, device=dev), w.to(dev), e)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()


QKV_SHAPES = [
    # F, gh, gw, W, Hh, H, D, hidden, round
    (2, 6, 25, 3, 1, 2, 128, 256, 4),     # L = 300 (ragged tiles), ring wraps at round 4
    (1, 8, 17, 2, 2, 4, 64, 192, 1),      # D = 64: two heads per 128-column half
    (3, 4, 11, 4, 0, 1, 128, 520, 0),     # H*D = 128: N = 384, a half-empty last tile
]


@pytest.mark.parametrize("F,gh,gw,W,Hh,H,D,hidden,r", QKV_SHAPES)
def test_qkv_fused_parity(wf, F, gh, gw, W, Hh, H, D, hidden, r):
    dev = "cuda"
    L = F * gh * gw
    R = W + Hh
    T = W * L
    seed = L + H + D
    x = wi.bf16_normal((T, hidden), seed, wi.STREAM_X)
    w_qkv = wi.bf16_weight(3 * H * D, hidden, seed)
    b = wi.f32_vector((3 * H * D,), 0.3, seed, wi.STREAM_BIAS)
    gq, gk = wi.gains(H, D, seed)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    q_out = torch.full((T, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
    sentinel = -7.0
    kc = torch.full((R, L, H, D), sentinel, dtype=torch.bfloat16, device=dev)
    vc = torch.full((R, L, H, D), sentinel, dtype=torch.bfloat16, device=dev)
    wf.wf_qkv_proj_norm_rope_append(plan, r, x.to(dev), w_qkv.to(dev), b.to(dev), gq.to(dev),
                                    gk.to(dev), q_out, kc, vc)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    pos = oracle.positions(r, W, F, gh, gw)
    rq, rk, rv, q64, k64, v64 = ob.qkv_project_append(_bits(x), _bits(w_qkv), b.numpy(), pos,
                                                      gq.numpy(), gk.numpy(), H, D, want_f64=True)
    S = _abs_sum(x, w_qkv).reshape(T, 3, H, D)
    y = ob.linear_f64(_bits(x), _bits(w_qkv), b.numpy()).reshape(T, 3, H, D)
    kcb, vcb = _bits(kc), _bits(vc)
    got_k = np.empty((T, H, D), np.uint16)
    got_v = np.empty((T, H, D), np.uint16)
    for c in range(W):
        slot = (r + c) % R
        got_k[c * L:(c + 1) * L] = kcb[slot]
        got_v[c * L:(c + 1) * L] = vcb[slot]
    _assert_qk_close(_bits(q_out), q64, y[:, 0], S[:, 0], gq, "q")
    _assert_qk_close(got_k, k64, y[:, 1], S[:, 1], gk, "k")
    _assert_gemm_close(got_v, v64, S[:, 2], "v")
    # slots of the history chunks are not written
    touched = {(r + c) % R for c in range(W)}
    for slot in set(range(R)) - touched:
        assert (kc[slot].float() == sentinel).all() and (vc[slot].float() == sentinel).all()
    plan.destroy()


def test_qkv_equals_projection_then_append(wf):
    """Up to the bf16 rounding of q and k between the two kernels, the fused call
    equals wf_linear (store) followed by wf_qk_norm_rope_append; v agrees bit for
    bit (both paths round the same fp32 accumulator once and the append copies v)."""
    dev = "cuda"
    F, gh, gw, W, Hh, H, D, hidden, r = 2, 5, 13, 3, 2, 2, 128, 256, 3
    L, R, T = F * gh * gw, W + Hh, W * F * gh * gw
    x = wi.bf16_normal((T, hidden), 5, wi.STREAM_X).to(dev)
    w_qkv = wi.bf16_weight(3 * H * D, hidden, 5).to(dev)
    gq, gk = (t.to(dev) for t in wi.gains(H, D, 5))
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    q1 = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    k1 = torch.zeros((R, L, H, D), dtype=torch.bfloat16, device=dev)
    v1 = torch.zeros_like(k1)
    wf.wf_qkv_proj_norm_rope_append(plan, r, x, w_qkv, None, gq, gk, q1, k1, v1)
    y = torch.empty((T, 3 * H * D), dtype=torch.bfloat16, device=dev)
    wf.wf_linear(plan, x, w_qkv, y)
    y3 = y.view(T, 3, H, D)
    q2 = torch.empty_like(q1)
    k2 = torch.zeros_like(k1)
    v2 = torch.zeros_like(k1)
    wf.wf_qk_norm_rope_append(plan, r, y3[:, 0].contiguous(), y3[:, 1].contiguous(),
                              y3[:, 2].contiguous(), None, gq, gk, q2, k2, v2)
    torch.cuda.synchronize()
    assert torch.equal(v1.view(torch.int16), v2.view(torch.int16))
    for a, b in ((q1, q2), (k1, k2)):
        d = (a.float() - b.float()).abs()
        assert float(d.max()) <= 2.0 ** -5 and float(d.mean()) <= 2e-3
    plan.destroy()


@pytest.mark.parametrize("M,C,rpg", [(1000, 1536, 300), (37, 5120, 10), (64, 8, 64), (5, 6144, 2),
                                     (1000, 2048, 7), (3, 1536, 1), (333, 2056, 50),
                                     (4679, 1024, 4680), (23400, 1536, 4680)])
def test_layer_norm_modulate_parity(wf, M, C, rpg):
    dev = "cuda"
    seed = M + C
    x = (wi.bf16_normal((M, C), seed, wi.STREAM_X).float() * 3.0 + 0.5).to(torch.bfloat16)
    G = (M + rpg - 1) // rpg
    shift = wi.f32_vector((G, C), 0.5, seed, wi.STREAM_MOD)
    scale = wi.f32_vector((G, C), 0.5, seed, wi.STREAM_BIAS)
    plan = wf.Plan(32, 1, 0, 1, 64)
    y = torch.full((M, C), float("nan"), dtype=torch.bfloat16, device=dev)
    wf.wf_layer_norm_modulate(plan, x.to(dev), shift.to(dev), scale.to(dev), rpg, y)
    torch.cuda.synchronize()
    ref = ob.layer_norm_modulate_f64(_bits(x), shift.numpy(), scale.numpy(), rpg)
    xh = ob.layer_norm_modulate_f64(_bits(x), np.zeros(C, np.float32), np.zeros(C, np.float32), M)
    grp = np.arange(M) // rpg
    mag = np.abs(xh * (1.0 + scale.numpy()[grp])) + np.abs(shift.numpy()[grp])
    r_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(ref))
    tol = bf16_quantum(r_bf) * 1.0000001 + 2.0 ** -18 * mag
    d = np.abs(_f64(y.float()) - ref)
    assert not (d > tol).any(), "layer norm: %d outside the bar (worst excess %g)" % (
        int((d > tol).sum()), float((d - tol).max()))
    plan.destroy()


def test_full_size_sampled(wf):
    """Wan-1.3B widths at the 4-step wave's T = 23400 rows: the fused QKV projection
    and the second feed-forward GEMM (K = 8960), sampled rows against the oracle."""
    dev = "cuda"
    w = wi.WORKLOADS["wan13b_4step"]
    C, Ff = wi.WAN13B_HIDDEN, wi.WAN13B_FFN
    b = wi.block_inputs(w, C, Ff, seed=0)
    r = w.n_hist
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    x = b.x.to(dev)
    wf.wf_qkv_proj_norm_rope_append(plan, r, x, b.w_qkv.to(dev), b.b_qkv.to(dev),
                                    b.gamma_q.to(dev), b.gamma_k.to(dev), q_out, kc, vc)
    h = wi.bf16_normal((w.T, Ff), 1, wi.STREAM_Q)
    out = torch.empty((w.T, C), dtype=torch.bfloat16, device=dev)
    gate = b.mod[5]
    wf.wf_linear(plan, h.to(dev), b.w_2.to(dev), out, b.b_2.to(dev), wf.WF_EPI_GATED_RESIDUAL,
                 gate.to(dev), x, w.L)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    rows = np.unique(np.concatenate([np.arange(0, w.T, 997), [w.T - 1, w.L - 1, w.L, 2 * w.L]]))
    pos = oracle.positions(r, w.n_wave, w.F, w.gh, w.gw)[rows]
    rq, rk, rv, q64, k64, v64 = ob.qkv_project_append(_bits(b.x[rows]), _bits(b.w_qkv),
                                                      b.b_qkv.numpy(), pos, b.gamma_q.numpy(),
                                                      b.gamma_k.numpy(), w.H, w.D, want_f64=True)
    qb = _bits(q_out)[rows]
    kcb = _bits(kc)
    c_of = rows // w.L
    kb = np.stack([kcb[(r + c) % w.R, n - c * w.L] for n, c in zip(rows, c_of)])
    n = rows.size
    y = ob.linear_f64(_bits(b.x[rows]), _bits(b.w_qkv), b.b_qkv.numpy()).reshape(n, 3, w.H, w.D)
    S = _abs_sum(b.x[rows], b.w_qkv).reshape(n, 3, w.H, w.D)
    _assert_qk_close(qb, q64, y[:, 0], S[:, 0], b.gamma_q, "q full size")
    _assert_qk_close(kb, k64, y[:, 1], S[:, 1], b.gamma_k, "k full size")
    # rows of the sample sit in different chunks: the gate row follows the row's chunk
    ref2 = np.stack([ob.linear_f64(_bits(h[n:n + 1]), _bits(b.w_2), b.b_2.numpy(),
                                   "gated_residual", gate.numpy()[c:c + 1], _bits(b.x[n:n + 1]),
                                   1)[0] for n, c in zip(rows, c_of)])
    S = _abs_sum(h[rows], b.w_2) * np.abs(gate.numpy().astype(np.float64))[c_of]
    _assert_gemm_close(_bits(out)[rows], ref2, S, "ffn2 full size")
    plan.destroy()


def test_block_composition(wf):
    """The seven calls of one DiT block, composed as bench.py's block leg composes
    them (gated residuals in place on the residual stream, ring with history),
    against oracle.block.block_forward.  Bar: the two stored roundings of the
    residual stream (x1 and x2) may each land one bf16 quantum apart from the
    oracle's, and the attention's error (1e-2 max, 1e-3 mean on unit-scale data)
    reaches x2 through W_o (unit gain) times a gate of ~0.1, so
    |got - ref| <= 2 quanta(ref) + 1e-2 per element and mean |got - ref| <= 1e-3."""
    import oracle
    import oracle.block as ob
    dev = "cuda"
    F, gh, gw, W, Hh, H, D, ffn, r = 2, 6, 25, 3, 1, 2, 128, 512, 2
    L, T, C, R = F * gh * gw, W * F * gh * gw, H * D, W + Hh
    s = 21
    x = wi.bf16_normal((T, C), s, wi.STREAM_X)
    wts = dict(w_qkv=wi.bf16_weight(3 * C, C, s, 1), w_o=wi.bf16_weight(C, C, s, 2),
               w_1=wi.bf16_weight(ffn, C, s, 3), w_2=wi.bf16_weight(C, ffn, s, 4),
               b_qkv=wi.f32_vector((3 * C,), 0.02, s, wi.STREAM_BIAS, 1),
               b_o=wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 2),
               b_1=wi.f32_vector((ffn,), 0.02, s, wi.STREAM_BIAS, 3),
               b_2=wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 4))
    wts["gamma_q"], wts["gamma_k"] = wi.gains(H, D, s)
    mod = wi.f32_vector((6, W, C), 0.1, s, wi.STREAM_MOD)
    hk = wi.bf16_normal((Hh, L, H, D), s, 3)
    hv = wi.bf16_normal((Hh, L, H, D), s, 4)
    d = {k: t.to(dev) for k, t in wts.items()}
    md = mod.to(dev)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    kc = torch.zeros((R, L, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    for j in range(Hh):
        kc[(r - Hh + j) % R].copy_(hk[j])
        vc[(r - Hh + j) % R].copy_(hv[j])
    X = x.to(dev)
    h = torch.empty_like(X)
    q_out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q_out)
    f = torch.empty((T, ffn), dtype=torch.bfloat16, device=dev)
    wf.wf_layer_norm_modulate(plan, X, md[0], md[1], L, h)
    wf.wf_qkv_proj_norm_rope_append(plan, r, h, d["w_qkv"], d["b_qkv"], d["gamma_q"],
                                    d["gamma_k"], q_out, kc, vc)
    wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o)
    wf.wf_linear(plan, o.view(T, C), d["w_o"], X, d["b_o"], wf.WF_EPI_GATED_RESIDUAL, md[2], X, L)
    wf.wf_layer_norm_modulate(plan, X, md[3], md[4], L, h)
    wf.wf_linear(plan, h, d["w_1"], f, d["b_1"], wf.WF_EPI_GELU_TANH)
    wf.wf_linear(plan, f, d["w_2"], X, d["b_2"], wf.WF_EPI_GATED_RESIDUAL, md[5], X, L)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    cache = oracle.OracleCache(L)
    for j in range(Hh):
        cache.put(r - Hh + j, _bits(hk[j]), _bits(hv[j]))
    bw = {k: (_bits(t) if t.dtype == torch.bfloat16 else t.numpy()) for k, t in wts.items()}
    x2, inter = ob.block_forward(_bits(x), bw, mod.numpy(), oracle.positions(r, W, F, gh, gw),
                                 cache, r, W, Hh, H, D, L)
    ref = oracle.bf16_to_f64(x2)
    got = _f64(X.float())
    diff = np.abs(got - ref)
    tol = 2.0 * bf16_quantum(ref) + 1e-2
    assert not (diff > tol).any(), "block: %d outside the bar (max %g)" % (
        int((diff > tol).sum()), float(diff.max()))
    assert diff.mean() <= 1e-3, "block: mean abs %g" % diff.mean()
    # the ring holds the wave's K/V where the attention read them
    for c in range(W):
        got_k = _bits(kc[(r + c) % R])
        want_k = inter["k"][c * L:(c + 1) * L]
        assert (got_k != want_k).mean() < 0.05        # bf16 roundings of the fused epilogue
    plan.destroy()


@pytest.mark.parametrize("epi", ["store", "gelu_tanh", "gated_residual", "qkv"])
def test_repeat_runs_bit_identical(wf, epi):
    """Ten launches of each GEMM epilogue (and of the LayerNorm) give the same bits:
    a race in the stage ring or the double-buffered accumulator (a slot reused
    early, an epilogue reading a tile the MMAs are overwriting) would show as
    run-to-run differences.  Shapes of several tiles per cluster."""
    dev = "cuda"
    F, gh, gw, W, Hh, H, D = 2, 10, 26, 4, 1, 4, 128     # T = 2080, N = 1536 for qkv
    L, T, C = F * gh * gw, W * F * gh * gw, 512
    x = wi.bf16_normal((T, C), 31, wi.STREAM_X).to(dev)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    outs = []
    if epi == "qkv":
        w_qkv = wi.bf16_weight(3 * H * D, C, 31).to(dev)
        gq, gk = (t.to(dev) for t in wi.gains(H, D, 31))
        q_out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        kc = torch.zeros((W + Hh, L, H, D), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        for _ in range(10):
            wf.wf_qkv_proj_norm_rope_append(plan, 3, x, w_qkv, None, gq, gk, q_out, kc, vc)
            outs.append(torch.cat([q_out.view(-1), kc.view(-1), vc.view(-1)]).view(torch.int16)
                        .clone())
    else:
        N = 1280
        w = wi.bf16_weight(N, C, 32).to(dev)
        b = wi.f32_vector((N,), 0.5, 32, wi.STREAM_BIAS).to(dev)
        gate = wi.f32_vector((W, N), 1.0, 32, wi.STREAM_MOD).to(dev)
        resid = wi.bf16_normal((T, N), 32, wi.STREAM_V).to(dev)
        y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        code = {"store": wf.WF_EPI_STORE, "gelu_tanh": wf.WF_EPI_GELU_TANH,
                "gated_residual": wf.WF_EPI_GATED_RESIDUAL}[epi]
        gr = epi == "gated_residual"
        for _ in range(10):
            wf.wf_linear(plan, x, w, y, b, code, gate if gr else None, resid if gr else None, L)
            outs.append(y.view(torch.int16).clone())
        mod = wi.f32_vector((2, W, C), 0.3, 33, wi.STREAM_MOD).to(dev)
        h = torch.empty_like(x)
        hs = []
        for _ in range(10):
            wf.wf_layer_norm_modulate(plan, x, mod[0], mod[1], L, h)
            hs.append(h.view(torch.int16).clone())
        assert all(torch.equal(hs[0], t) for t in hs[1:])
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    assert all(torch.equal(outs[0], t) for t in outs[1:])
    plan.destroy()


@pytest.mark.parametrize("M,N,K", [(1, 32, 8), (257, 32, 8), (3, 64, 2056), (511, 256, 72)])
def test_linear_edge_shapes(wf, M, N, K):
    """Degenerate and ragged GEMM shapes: one row, the smallest N and K the call
    accepts, one row past a 256-row tile, a K of 32 slices plus 8, a single column
    tile with M one short of two tiles."""
    dev = "cuda"
    seed = 3 * M + N + K
    x = wi.bf16_normal((M, K), seed, wi.STREAM_X)
    w = wi.bf16_weight(N, K, seed)
    bias = wi.f32_vector((N,), 0.5, seed, wi.STREAM_BIAS)
    gate = wi.f32_vector((1, N), 1.0, seed, wi.STREAM_MOD)
    resid = wi.bf16_normal((M, N), seed, wi.STREAM_V)
    plan = wf.Plan(32, 1, 0, 1, 64)
    for epi, code in (("store", wf.WF_EPI_STORE), ("gelu_tanh", wf.WF_EPI_GELU_TANH),
                      ("gated_residual", wf.WF_EPI_GATED_RESIDUAL)):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        gr = epi == "gated_residual"
        wf.wf_linear(plan, x.to(dev), w.to(dev), y, bias.to(dev), code,
                     gate.to(dev) if gr else None, resid.to(dev) if gr else None, M)
        torch.cuda.synchronize()
        assert wf.wf_sync_status(plan) == wf.WF_OK
        ref = ob.linear_f64(_bits(x), _bits(w), bias.numpy(), epi, gate.numpy() if gr else None,
                            _bits(resid) if gr else None, M)
        S = _abs_sum(x, w) * (np.abs(gate.numpy().astype(np.float64)) if gr else 1.0)
        _assert_gemm_close(_bits(y), ref, S, "linear %s %dx%dx%d" % (epi, M, N, K))
    plan.destroy()


def test_qkv_first_round_with_history_slots(wf):
    """Round 0 of a ring with history slots (no history visible yet): the fused
    projection writes the wave's chunks to slots 0..W-1 with t = c*F + f and
    leaves the history slots alone."""
    dev = "cuda"
    F, gh, gw, W, Hh, H, D, C = 1, 4, 9, 2, 3, 1, 128, 128
    L, T, R = F * gh * gw, W * F * gh * gw, W + Hh
    x = wi.bf16_normal((T, C), 41, wi.STREAM_X)
    w_qkv = wi.bf16_weight(3 * H * D, C, 41)
    gq, gk = wi.gains(H, D, 41)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    q_out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    kc = torch.full((R, L, H, D), -5.0, dtype=torch.bfloat16, device=dev)
    vc = torch.full_like(kc, -5.0)
    wf.wf_qkv_proj_norm_rope_append(plan, 0, x.to(dev), w_qkv.to(dev), None, gq.to(dev),
                                    gk.to(dev), q_out, kc, vc)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    pos = oracle.positions(0, W, F, gh, gw)
    _, _, _, q64, k64, v64 = ob.qkv_project_append(_bits(x), _bits(w_qkv), None, pos, gq.numpy(),
                                                   gk.numpy(), H, D, want_f64=True)
    y = ob.linear_f64(_bits(x), _bits(w_qkv)).reshape(T, 3, H, D)
    S = _abs_sum(x, w_qkv).reshape(T, 3, H, D)
    got_k = np.concatenate([_bits(kc[c]) for c in range(W)])
    _assert_qk_close(_bits(q_out), q64, y[:, 0], S[:, 0], gq, "q round 0")
    _assert_qk_close(got_k, k64, y[:, 1], S[:, 1], gk, "k round 0")
    for slot in range(W, R):
        assert (kc[slot].float() == -5.0).all() and (vc[slot].float() == -5.0).all()
    plan.destroy()


def test_layer_norm_single_row_and_group(wf):
    """One row of 64 channels around a common offset, one modulation group."""
    dev = "cuda"
    x = (wi.bf16_normal((1, 64), 5, wi.STREAM_X).float() * 0.5 + 3.0).to(torch.bfloat16)
    shift = wi.f32_vector((1, 64), 0.5, 5, wi.STREAM_MOD)
    scale = wi.f32_vector((1, 64), 0.5, 5, wi.STREAM_BIAS)
    plan = wf.Plan(32, 1, 0, 1, 64)
    y = torch.empty((1, 64), dtype=torch.bfloat16, device=dev)
    wf.wf_layer_norm_modulate(plan, x.to(dev), shift.to(dev), scale.to(dev), 1, y)
    torch.cuda.synchronize()
    ref = ob.layer_norm_modulate_f64(_bits(x), shift.numpy(), scale.numpy(), 1)
    xh = ob.layer_norm_modulate_f64(_bits(x), np.zeros(64, np.float32), np.zeros(64, np.float32), 1)
    mag = np.abs(xh * (1.0 + scale.numpy())) + np.abs(shift.numpy())
    r_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(ref))
    tol = bf16_quantum(r_bf) * 1.0000001 + 2.0 ** -18 * mag   # the bar of the main LN test
    assert (np.abs(_f64(y.float()) - ref) <= tol).all()
    plan.destroy()
