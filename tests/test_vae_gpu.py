"""GPU parity of the streaming VAE-decode stage (causal 3x3x3 convolution as a
tcgen05 implicit GEMM, RMSNorm + SiLU) against the fp64 oracle in oracle/vae.py,
through the C ABI.

Bars (per element, against the oracle's exact value y):
* a convolution output: |got - y| <= one bf16 quantum of y + 2^-20 * S, where
  S = sum over taps and channels of |w x| (plus |bias|) bounds the fp32
  accumulation error of the tensor-core sum, as for the linear layers;
* RMSNorm + SiLU: one bf16 quantum + 2^-18 * |y| (fp32 norm and exponential);
* the residual block composed of the four calls, streamed over two chunks:
  two bf16 quanta + 1e-2 per element and mean <= 1e-3 (the stored intermediate
  conv1 output may round one quantum apart and carries that through the second
  norm and convolution).
Shapes cover frames smaller than a 16 x 16 pixel tile, rows and columns past the
frame in a tile, input channels below and not a multiple of the 64-channel slice,
output channels filling 192- and 256-wide tiles partly, the start of a video
(no history) and a chunk streamed after another; the full 120 x 208 x 384 stage
is checked on sampled pixels.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.vae as ov
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import bf16_quantum

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def _bits(t):
    return wi.bits(t.contiguous().cpu())


def _abs_bits(b):
    return None if b is None else (np.asarray(b, np.uint16) & np.uint16(0x7FFF))


def conv_weight(Cout, Cin, seed, salt=0):
    """Random-init conv weight [Cout, 3, 3, 3, Cin]: N(0, 1/(27 Cin)) in bf16."""
    return wi.bf16_weight(Cout, 27 * Cin, seed, salt).reshape(Cout, 3, 3, 3, Cin).contiguous()


def assert_conv_close(got, ref64, S, what):
    g = got.cpu().double().numpy()
    r = oracle.bf16_to_f64(oracle.f64_to_bf16(ref64))
    tol = bf16_quantum(r) * 1.0000001 + 2.0 ** -20 * S
    d = np.abs(g - ref64)
    bad = d > tol
    assert not bad.any(), "%s: %d of %d outside the bar (worst excess %g)" % (
        what, int(bad.sum()), bad.size, float((d - tol).max()))


def _oracle_conv(x, hist, w, bias, resid):
    xb, hb, wb = _bits(x), None if hist is None else _bits(hist), _bits(w)
    rb = None if resid is None else _bits(resid)
    b = None if bias is None else bias.cpu().numpy()
    ref = ov.causal_conv3d_f64(xb, hb, wb, b, rb)
    S = ov.causal_conv3d_f64(_abs_bits(xb), _abs_bits(hb), _abs_bits(wb),
                             None if b is None else np.abs(b))
    return ref, S


CONV_SHAPES = [
    # T, H, W, Cin, Cout, history, residual
    (3, 20, 37, 64, 64, True, False),      # ragged rows and columns of the 16 x 16 tiles
    (2, 8, 16, 96, 96, False, True),       # Cin past one 64-slice, half-empty 256 tile
    (4, 17, 23, 24, 192, True, True),      # Cin below one slice, one full 192 tile
    (1, 5, 3, 8, 32, False, False),        # a frame smaller than a tile
    (2, 12, 40, 128, 384, True, False),    # two 192 tiles
]


@pytest.mark.parametrize("T,H,W,Cin,Cout,hist,res", CONV_SHAPES)
def test_conv_all_outputs(wf, T, H, W, Cin, Cout, hist, res):
    s = T + H + W + Cin + Cout
    x = wi.bf16_normal((T, H, W, Cin), s, wi.STREAM_X).cuda()
    xh = wi.bf16_normal((2, H, W, Cin), s, wi.STREAM_CACHE).cuda() if hist else None
    w = conv_weight(Cout, Cin, s).cuda()
    b = wi.f32_vector((Cout,), 0.02, s, wi.STREAM_BIAS).cuda()
    r = wi.bf16_normal((T, H, W, Cout), s, wi.STREAM_MOD).cuda() if res else None
    y = torch.full((T, H, W, Cout), float("nan"), dtype=torch.bfloat16, device="cuda")
    plan = wf.Plan(64, 1, 0, 1, 128)
    wf.wf_causal_conv3d(plan, x, xh, w, b, r, y)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref, S = _oracle_conv(x, xh, w, b, r)
    assert_conv_close(y, ref, S, "conv T=%d H=%d W=%d Cin=%d Cout=%d" % (T, H, W, Cin, Cout))
    plan.destroy()


def test_conv_streamed_chunks_equal_whole_video(wf):
    """Two chunks, the second reading the first chunk's last two frames as its
    history (a view into the first chunk's buffer, no copy), against the oracle's
    convolution of the whole sequence; the residual written in place (y = resid)."""
    T1, T2, H, W, C = 3, 4, 18, 33, 64
    s = 7
    x = wi.bf16_normal((T1 + T2, H, W, C), s, wi.STREAM_X).cuda()
    w = conv_weight(C, C, s).cuda()
    b = wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS).cuda()
    r = wi.bf16_normal((T1 + T2, H, W, C), s, wi.STREAM_MOD).cuda()
    plan = wf.Plan(64, 1, 0, 1, 128)
    x1, x2 = x[:T1].contiguous(), x[T1:].contiguous()
    y = r.clone()
    y1, y2 = y[:T1], y[T1:]                     # contiguous views of the output
    wf.wf_causal_conv3d(plan, x1, None, w, b, y1, y1)
    wf.wf_causal_conv3d(plan, x2, x1[T1 - 2:], w, b, y2, y2)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref, S = _oracle_conv(x, None, w, b, r)
    assert_conv_close(y, ref, S, "streamed conv")
    plan.destroy()


def test_conv_repeat_runs_bit_identical(wf):
    T, H, W, Cin, Cout = 3, 40, 52, 128, 192
    x = wi.bf16_normal((T, H, W, Cin), 3, wi.STREAM_X).cuda()
    xh = wi.bf16_normal((2, H, W, Cin), 3, wi.STREAM_CACHE).cuda()
    w = conv_weight(Cout, Cin, 3).cuda()
    plan = wf.Plan(64, 1, 0, 1, 128)
    first = torch.empty((T, H, W, Cout), dtype=torch.bfloat16, device="cuda")
    wf.wf_causal_conv3d(plan, x, xh, w, None, None, first)
    for _ in range(5):
        again = torch.empty_like(first)
        wf.wf_causal_conv3d(plan, x, xh, w, None, None, again)
        torch.cuda.synchronize()
        assert torch.equal(again.view(torch.int16), first.view(torch.int16))
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()


def test_conv_full_stage_sampled(wf):
    """The benchmark's stage: one chunk of 12 frames at 120 x 208 with 384 channels
    in and out, history present; checked on pixels at tile and frame edges plus
    random pixels, every output channel."""
    T, H, W, C = 12, 120, 208, 384
    x = wi.bf16_normal((T, H, W, C), 0, wi.STREAM_X).cuda()
    xh = wi.bf16_normal((2, H, W, C), 0, wi.STREAM_CACHE).cuda()
    w = conv_weight(C, C, 0).cuda()
    b = wi.f32_vector((C,), 0.02, 0, wi.STREAM_BIAS).cuda()
    y = torch.empty((T, H, W, C), dtype=torch.bfloat16, device="cuda")
    plan = wf.Plan(64, 1, 0, 1, 128)
    wf.wf_causal_conv3d(plan, x, xh, w, b, None, y)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    rng = np.random.default_rng(0)
    edge = [(t, i, j) for t in (0, 1, 2, T - 1) for i in (0, 7, 8, 15, 16, H - 1)
            for j in (0, 15, 16, W - 1)]
    rnd = [tuple(int(v) for v in (rng.integers(T), rng.integers(H), rng.integers(W)))
           for _ in range(24)]
    px = np.array(edge + rnd, np.int64)
    ref, S = ov.causal_conv3d_at(_bits(x), _bits(xh), _bits(w), px, b.cpu().numpy())
    # S from |x| and |w| (the helper's second output already is sum |w x| + |b|)
    got = y[px[:, 0], px[:, 1], px[:, 2]]
    assert_conv_close(got, ref, S, "full stage")
    assert torch.isfinite(y.float()).all()
    plan.destroy()


@pytest.mark.parametrize("M,C", [(1000, 384), (333, 96), (50, 512), (7, 8)])
def test_rms_norm_silu(wf, M, C):
    x = wi.bf16_normal((M, C), M + C, wi.STREAM_X).cuda() * 3
    g = (1 + 0.1 * wi.f32_vector((C,), 1.0, M, wi.STREAM_GAMMA)).cuda()
    y = torch.empty_like(x)
    plan = wf.Plan(64, 1, 0, 1, 128)
    wf.wf_rms_norm_silu(plan, x, g, y)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref = ov.rms_norm_silu_f64(_bits(x), g.cpu().numpy())
    got = y.cpu().double().numpy()
    r = oracle.bf16_to_f64(oracle.f64_to_bf16(ref))
    tol = bf16_quantum(r) * 1.0000001 + 2.0 ** -18 * np.abs(ref) + 1e-30
    d = np.abs(got - ref)
    assert not (d > tol).any(), "rms_norm_silu M=%d C=%d: worst excess %g" % (
        M, C, float((d - tol).max()))
    plan.destroy()


def test_res_block_streamed_against_oracle(wf):
    """The decode stage's residual block (norm + SiLU, conv, norm + SiLU, conv +
    residual) over two chunks, the convolutions' histories taken from the first
    chunk's buffers, against oracle.vae.res_block."""
    T1, T2, H, W, C = 3, 2, 17, 30, 96
    s = 11
    x = wi.bf16_normal((T1 + T2, H, W, C), s, wi.STREAM_X)
    wts = dict(gamma1=(1 + 0.1 * wi.f32_vector((C,), 1.0, s, wi.STREAM_GAMMA, 1)),
               gamma2=(1 + 0.1 * wi.f32_vector((C,), 1.0, s, wi.STREAM_GAMMA, 2)),
               w1=conv_weight(C, C, s, 1), w2=conv_weight(C, C, s, 2),
               b1=wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 1),
               b2=wi.f32_vector((C,), 0.02, s, wi.STREAM_BIAS, 2))
    d = {k: v.cuda() for k, v in wts.items()}
    plan = wf.Plan(64, 1, 0, 1, 128)
    outs, hist = [], None
    for xs in (x[:T1], x[T1:]):
        xc = xs.contiguous().cuda()
        h1 = torch.empty_like(xc)
        wf.wf_rms_norm_silu(plan, xc, d["gamma1"], h1)
        c1 = torch.empty_like(xc)
        wf.wf_causal_conv3d(plan, h1, None if hist is None else hist[0], d["w1"], d["b1"], None, c1)
        h2 = torch.empty_like(xc)
        wf.wf_rms_norm_silu(plan, c1, d["gamma2"], h2)
        out = torch.empty_like(xc)
        wf.wf_causal_conv3d(plan, h2, None if hist is None else hist[1], d["w2"], d["b2"], xc, out)
        hist = (h1[-2:], h2[-2:])                # views: the next chunk's histories
        outs.append(out)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    got = torch.cat(outs).cpu().double().numpy()
    bw = {k: (_bits(v) if v.dtype == torch.bfloat16 else v.numpy()) for k, v in wts.items()}
    ref, _, _ = ov.res_block(_bits(x), bw)
    r = oracle.bf16_to_f64(ref)
    diff = np.abs(got - r)
    tol = 2.0 * bf16_quantum(r) + 1e-2
    assert not (diff > tol).any(), "res block: %d outside the bar (max %g)" % (
        int((diff > tol).sum()), float(diff.max()))
    assert diff.mean() <= 1e-3, "res block: mean abs %g" % diff.mean()
    plan.destroy()
