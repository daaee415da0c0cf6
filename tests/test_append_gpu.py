"""GPU parity of wf_qk_norm_rope_append against the fp64 oracle.

Bar: q_out and K' equal the oracle's round-to-nearest-even bf16 or differ by
one bf16 ulp, plus the fp32 rounding error of the GPU's rotation (2^-20 times
the pair's length, which matters only where the rotation nearly cancels); V
and the ring slot of every chunk are bit-exact; slots outside the wave are
untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_within_one_ulp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


SENTINEL = 0x7FBF   # a NaN pattern the append never writes


def run_append(wf, w, round_, seed=0, explicit_pos=False):
    x = wi.wave_inputs(w, seed=seed)
    dev = "cuda"
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    pos_np = oracle.positions(round_, w.n_wave, w.F, w.gh, w.gw)
    pos = torch.from_numpy(pos_np).to(dev) if explicit_pos else None
    q_out = torch.empty_like(q)
    kc = torch.full((w.R, w.L, w.H, w.D), SENTINEL, dtype=torch.int16,
                    device=dev).view(torch.bfloat16)
    vc = kc.clone()
    wf.wf_qk_norm_rope_append(plan, round_, q, k, v, pos, gq, gk, q_out, kc, vc)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    ref = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos_np, x.gamma_q.numpy(),
                        x.gamma_k.numpy(), want_f64=True)
    out = (wi.bits(q_out.cpu()), wi.bits(kc.cpu()), wi.bits(vc.cpu()))
    plan.destroy()
    return x, ref, out


def check_append(w, round_, ref, out):
    qo_ref, ko_ref, vo_ref, q64, k64 = ref
    qo, kc, vc = out
    frac_q = assert_within_one_ulp(qo, qo_ref, "q_out", q64)
    written = set()
    for c in range(w.n_wave):
        slot = (round_ + c) % w.R
        written.add(slot)
        sl = slice(c * w.L, (c + 1) * w.L)
        assert_within_one_ulp(kc[slot], ko_ref[sl], "K' chunk %d" % c, k64[sl])
        assert np.array_equal(vc[slot], vo_ref[sl]), "V chunk %d not bit-exact" % c
    for s in range(w.R):
        if s not in written:
            assert np.all(kc[s] == SENTINEL) and np.all(vc[s] == SENTINEL), "slot %d touched" % s
    return frac_q


@pytest.mark.parametrize("round_", [0, 1, 4])
def test_append_tiny(wf, round_):
    w = wi.WORKLOADS["tiny"]
    x, ref, out = run_append(wf, w, round_)
    frac = check_append(w, round_, ref, out)
    assert frac < 0.02      # nearly all values are the correctly rounded ones


def test_append_explicit_positions_equal_derived(wf):
    w = wi.Workload("ragged", H=3, D=128, F=2, gh=5, gw=7, n_wave=4, n_hist=2)
    _, ref, out_d = run_append(wf, w, 6)
    _, _, out_e = run_append(wf, w, 6, explicit_pos=True)
    for a, b in zip(out_d, out_e):
        assert np.array_equal(a, b)
    check_append(w, 6, ref, out_d)


def test_append_ragged_d64(wf):
    w = wi.Workload("ragged64", H=5, D=64, F=1, gh=9, gw=11, n_wave=3, n_hist=1)
    _, ref, out = run_append(wf, w, 2, seed=3)
    check_append(w, 2, ref, out)


def test_append_full_size_wan13b(wf):
    # 12 heads x 128, 5 chunks x 4680 tokens (3 x 30 x 52), every element checked
    w = wi.WORKLOADS["wan13b_4step"]
    _, ref, out = run_append(wf, w, 2)
    check_append(w, 2, ref, out)


def test_append_alternative_tiny_positions(wf):
    """The tiny wave's description ("t = 0..2, 4x4 grid" with 32-token chunks) also
    reads as t = chunk index shared by both frames of a chunk; the explicit
    pos_thw input carries that reading through the same kernel."""
    w = wi.WORKLOADS["tiny"]
    x = wi.wave_inputs(w, seed=5)
    dev = "cuda"
    n = np.arange(w.T)
    c, rem = n // w.L, n % w.L
    pos_np = np.stack([c, (rem % 16) // 4, rem % 4], axis=1).astype(np.int32)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D)      # no geometry: explicit only
    q_out = torch.empty_like(x.q, device=dev)
    kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    wf.wf_qk_norm_rope_append(plan, 0, x.q.to(dev), x.k.to(dev), x.v.to(dev),
                              torch.from_numpy(pos_np).to(dev), x.gamma_q.to(dev),
                              x.gamma_k.to(dev), q_out, kc, vc)
    torch.cuda.synchronize()
    ref = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos_np, x.gamma_q.numpy(),
                        x.gamma_k.numpy(), want_f64=True)
    check_append(w, 0, ref, (wi.bits(q_out.cpu()), wi.bits(kc.cpu()), wi.bits(vc.cpu())))
    plan.destroy()


def test_append_in_place_q(wf):
    """q_out may alias q (wf.h): the in-place call writes the same bits as the call
    with a separate q_out, on a ragged wave with several blocks per token range."""
    w = wi.Workload("inplace", 3, 128, 2, 6, 25, 3, 1)        # L = 300
    x = wi.wave_inputs(w, seed=4)
    dev = "cuda"
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    kc1 = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    vc1, kc2, vc2 = kc1.clone(), kc1.clone(), kc1.clone()
    q_out = torch.empty_like(q)
    wf.wf_qk_norm_rope_append(plan, 2, q, k, v, None, gq, gk, q_out, kc1, vc1)
    q_inplace = q.clone()
    wf.wf_qk_norm_rope_append(plan, 2, q_inplace, k, v, None, gq, gk, q_inplace, kc2, vc2)
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    assert torch.equal(q_inplace.view(torch.int16), q_out.view(torch.int16))
    assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))
    plan.destroy()
