"""The multi-layer round loop at the Wan-1.3B shape (the 30-layer workload as
bench.py runs it: one ring per layer, a pool of two q/k/v sets across layers,
the ring advancing one chunk per round), spot-checked on one (layer, round)
against the oracle, which rebuilds that layer's cache from absolute chunk ids."""
import numpy as np
import pytest
import torch

import oracle
from chunk_causal_dit_b200 import build as wf_build
from chunk_causal_dit_b200 import inputs as wi
from tests.wfcase import assert_attention_close, sample_rows

pytestmark = pytest.mark.gpu


def test_round_loop_spot_check():
    wf_build.build()
    from chunk_causal_dit_b200 import wf
    w = wi.WORKLOADS["wan13b_round"]
    dev = "cuda"
    rounds, layer_chk = 3, 17
    plan = wf.Plan(w.L, w.n_wave, w.n_hist, w.H, w.D).set_rope(w.F, w.gh, w.gw)
    sets = [wi.wave_inputs(w, seed=0, salt=s) for s in range(2)]
    qs = [(x.q.to(dev), x.k.to(dev), x.v.to(dev)) for x in sets]
    gq, gk = sets[0].gamma_q.to(dev), sets[0].gamma_k.to(dev)
    hk, hv = wi.history_prefill(w, seed=0)
    caches = []
    for _ in range(w.layers):
        kc = torch.empty((w.R, w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        for j in range(w.n_hist):
            kc[j % w.R].copy_(hk[j])
            vc[j % w.R].copy_(hv[j])
        caches.append((kc, vc))
    q_out = torch.empty_like(qs[0][0])
    o = torch.empty_like(q_out)
    r0 = w.n_hist
    o_chk = None
    for i in range(rounds):
        r = r0 + i
        for layer, (kc, vc) in enumerate(caches):
            q, k, v = qs[layer % 2]
            wf.wf_qk_norm_rope_append(plan, r, q, k, v, None, gq, gk, q_out, kc, vc)
            wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, None)
            if i == rounds - 1 and layer == layer_chk:
                o_chk = o.clone()
    torch.cuda.synchronize()
    assert wf.wf_sync_status(plan) == wf.WF_OK
    plan.destroy()
    # the oracle's view of layer layer_chk: history chunks, then each round's wave
    x = sets[layer_chk % 2]
    cache = oracle.OracleCache(w.L)
    for j in range(w.n_hist):
        cache.put(r0 - w.n_hist + j, wi.bits(hk[j]), wi.bits(hv[j]))
    qo = None
    for i in range(rounds):
        r = r0 + i
        pos = oracle.positions(r, w.n_wave, w.F, w.gh, w.gw)
        qo, ko, vo = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos,
                                   x.gamma_q.numpy(), x.gamma_k.numpy())
        cache.put_wave(r, ko, vo)
    rows_sel = sample_rows(w.L, w.n_wave, 24, seed=7)
    hs = [0, 7, 11]
    rows = np.repeat(rows_sel, len(hs))
    heads = np.tile(hs, len(rows_sel))
    ref, _ = oracle.round_attention(cache, r0 + rounds - 1, w.n_wave, w.n_hist, qo, rows, heads)
    got = o_chk.float().cpu().numpy()[rows, heads]
    assert_attention_close(got, ref, "layer %d round %d" % (layer_chk, r0 + rounds - 1))
