"""HostRoundPipeline (rounds streamed from pinned host memory) gives exactly the
results of the direct calls, round after round, ring included."""
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


def test_pipeline_matches_direct_calls(wf):
    from chunk_causal_dit_b200.pipeline import HostRoundPipeline
    w = wi.Workload("pipe", H=3, D=128, F=2, gh=10, gw=15, n_wave=4, n_hist=2)
    dev = torch.device("cuda", 0)
    rounds = range(0, 7)
    xs = [wi.wave_inputs(w, seed=0, salt=r) for r in rounds]
    gq, gk = xs[0].gamma_q.to(dev), xs[0].gamma_k.to(dev)

    def fresh():
        plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
        kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
        return plan, kc, torch.zeros_like(kc)

    plan, kc, vc = fresh()
    direct = []
    for r, x in zip(rounds, xs):
        q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
        o = torch.empty_like(q_out)
        wf.wf_qk_norm_rope_append(plan, r, x.q.to(dev), x.k.to(dev), x.v.to(dev), None, gq, gk,
                                  q_out, kc, vc)
        wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None)
        direct.append(o.cpu())
    torch.cuda.synchronize()

    plan2, kc2, vc2 = fresh()
    pipe = HostRoundPipeline(plan2, kc2, vc2, gq, gk, device=dev)
    host_o = [torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16).pin_memory() for _ in rounds]
    pipe.run([(r, x.q.pin_memory(), x.k.pin_memory(), x.v.pin_memory(), ho)
              for r, x, ho in zip(rounds, xs, host_o)])
    pipe.synchronize()
    assert wf.wf_sync_status(plan2) == wf.WF_OK
    for a, b in zip(direct, host_o):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    plan.destroy()
    plan2.destroy()


def test_pipeline_fp8qk_matches_direct_calls(wf):
    """The FP8 Q.K^T variant through the pipeline: append, quantize q and the
    wave's key chunks, E4M3 attention, round after round, E4M3 ring included."""
    from chunk_causal_dit_b200.pipeline import HostRoundPipeline
    w = wi.Workload("pipe8", H=2, D=128, F=2, gh=10, gw=13, n_wave=3, n_hist=2)
    dev = torch.device("cuda", 0)
    rounds = range(0, 6)
    xs = [wi.wave_inputs(w, seed=1, salt=r) for r in rounds]
    gq, gk = xs[0].gamma_q.to(dev), xs[0].gamma_k.to(dev)
    nt = (w.L + 127) // 128

    def fresh():
        plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
        kc = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
        k8 = torch.zeros((w.R, w.L, w.H, w.D), dtype=torch.uint8, device=dev)
        ks = torch.ones((w.R, nt, w.H), dtype=torch.float32, device=dev)
        return plan, kc, torch.zeros_like(kc), k8, ks

    plan, kc, vc, k8, ks = fresh()
    q8 = torch.empty((w.T, w.H, w.D), dtype=torch.uint8, device=dev)
    qs = torch.empty((w.H, w.T), dtype=torch.float32, device=dev)
    direct = []
    for r, x in zip(rounds, xs):
        q_out = torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16, device=dev)
        o = torch.empty_like(q_out)
        wf.wf_qk_norm_rope_append(plan, r, x.q.to(dev), x.k.to(dev), x.v.to(dev), None, gq, gk,
                                  q_out, kc, vc)
        wf.wf_quantize_q_fp8(plan, q_out, q8, qs)
        wf.wf_quantize_k_fp8(plan, r, w.n_wave, kc, k8, ks)
        wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o)
        direct.append(o.cpu())
    torch.cuda.synchronize()

    plan2, kc2, vc2, k82, ks2 = fresh()
    pipe = HostRoundPipeline(plan2, kc2, vc2, gq, gk, device=dev, fp8=(k82, ks2))
    host_o = [torch.empty((w.T, w.H, w.D), dtype=torch.bfloat16).pin_memory() for _ in rounds]
    pipe.run([(r, x.q.pin_memory(), x.k.pin_memory(), x.v.pin_memory(), ho)
              for r, x, ho in zip(rounds, xs, host_o)])
    pipe.synchronize()
    assert wf.wf_sync_status(plan2) == wf.WF_OK
    for a, b in zip(direct, host_o):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(k8, k82) and torch.equal(ks, ks2)
    plan.destroy()
    plan2.destroy()
