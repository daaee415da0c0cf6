"""Runs every kernel family of libwf on ragged seeded shapes and returns the
outputs (used by tests/test_check_build_gpu.py with the normal library in
process and with the bounds-checked debug build, WF_LIB_VARIANT=check, in a
subprocess: ``python tests/check_build_driver.py OUT.npz``)."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run_all(wf):
    from chunk_causal_dit_b200 import inputs as wi
    dev = "cuda"
    out, statuses = {}, {}
    F, gh, gw, W, Hh, H, D, r = 2, 6, 25, 3, 2, 2, 128, 4       # L = 300, ring wraps
    L, T, R = F * gh * gw, W * F * gh * gw, W + Hh
    x = wi.wave_inputs(wi.Workload("check", H, D, F, gh, gw, W, Hh), seed=5)
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    gq, gk = x.gamma_q.to(dev), x.gamma_k.to(dev)
    kc = wi.bf16_normal((R, L, H, D), 6, 3).to(dev)
    vc = wi.bf16_normal((R, L, H, D), 6, 4).to(dev)
    plan = wf.Plan(L, W, Hh, H, D).set_rope(F, gh, gw)
    q_out = torch.empty_like(q)
    wf.wf_qk_norm_rope_append(plan, r, q, k, v, None, gq, gk, q_out, kc, vc)
    statuses["append"] = wf.wf_sync_status(plan)
    for name, kind in (("attn_single", wf.WF_ATTN_SINGLE), ("attn_pair", wf.WF_ATTN_PAIR)):
        plan.set_attn_kernel(kind)
        o = torch.empty_like(q)
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        wf.wf_chunk_causal_attn(plan, r, q_out, kc, vc, o, lse)
        statuses[name] = wf.wf_sync_status(plan)
        out[name] = o.view(torch.int16).cpu().numpy()
        out[name + "_lse"] = lse.cpu().numpy()
    plan.set_attn_kernel(wf.WF_ATTN_AUTO)
    nt = (L + 127) // 128
    q8 = torch.empty((T, H, D), dtype=torch.uint8, device=dev)
    qs = torch.empty((H, T), dtype=torch.float32, device=dev)
    k8 = torch.empty((R, L, H, D), dtype=torch.uint8, device=dev)
    ks = torch.empty((R, nt, H), dtype=torch.float32, device=dev)
    wf.wf_quantize_q_fp8(plan, q_out, q8, qs)
    wf.wf_quantize_k_fp8(plan, r - Hh, R, kc, k8, ks)
    o8 = torch.empty_like(q)
    wf.wf_chunk_causal_attn_fp8qk(plan, r, q8, qs, k8, ks, vc, o8)
    statuses["fp8"] = wf.wf_sync_status(plan)
    out.update(q_out=q_out.view(torch.int16).cpu().numpy(), ring_k=kc.view(torch.int16).cpu().numpy(),
               ring_v=vc.view(torch.int16).cpu().numpy(), q8=q8.cpu().numpy(), qs=qs.cpu().numpy(),
               k8=k8.cpu().numpy(), ks=ks.cpu().numpy(), o8=o8.view(torch.int16).cpu().numpy())
    # the block's calls: GEMM epilogues (N not a multiple of 256, ragged K), QKV, LayerNorm
    C, N, K = H * D, 352, 200
    xb = wi.bf16_normal((T, K), 7, wi.STREAM_X).to(dev)
    wb = wi.bf16_weight(N, K, 7).to(dev)
    bias = wi.f32_vector((N,), 0.5, 7, wi.STREAM_BIAS).to(dev)
    gate = wi.f32_vector((W, N), 1.0, 7, wi.STREAM_MOD).to(dev)
    resid = wi.bf16_normal((T, N), 7, wi.STREAM_V).to(dev)
    for name, code in (("store", wf.WF_EPI_STORE), ("gelu", wf.WF_EPI_GELU_TANH),
                       ("gated", wf.WF_EPI_GATED_RESIDUAL)):
        y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        gr = code == wf.WF_EPI_GATED_RESIDUAL
        wf.wf_linear(plan, xb, wb, y, bias, code, gate if gr else None, resid if gr else None, L)
        statuses["linear_" + name] = wf.wf_sync_status(plan)
        out["linear_" + name] = y.view(torch.int16).cpu().numpy()
    xc = wi.bf16_normal((T, C), 8, wi.STREAM_X).to(dev)
    wq = wi.bf16_weight(3 * C, C, 8).to(dev)
    bq = wi.f32_vector((3 * C,), 0.3, 8, wi.STREAM_BIAS).to(dev)
    q2 = torch.empty_like(q)
    kc2 = torch.zeros_like(kc)
    vc2 = torch.zeros_like(vc)
    wf.wf_qkv_proj_norm_rope_append(plan, r, xc, wq, bq, gq, gk, q2, kc2, vc2)
    statuses["qkv"] = wf.wf_sync_status(plan)
    out.update(qkv_q=q2.view(torch.int16).cpu().numpy(), qkv_k=kc2.view(torch.int16).cpu().numpy(),
               qkv_v=vc2.view(torch.int16).cpu().numpy())
    mod = wi.f32_vector((2, W, C), 0.5, 9, wi.STREAM_MOD).to(dev)
    h = torch.empty_like(xc)
    wf.wf_layer_norm_modulate(plan, xc, mod[0], mod[1], L, h)
    statuses["layer_norm"] = wf.wf_sync_status(plan)
    out["layer_norm"] = h.view(torch.int16).cpu().numpy()
    # the fused-Q8 append, and the VAE stage's convolution (ragged frame, Cin not a
    # multiple of 64, a partial output tile, history + residual) and RMSNorm + SiLU
    q8b = torch.empty((T, H, D), dtype=torch.uint8, device=dev)
    qsb = torch.empty((H, T), dtype=torch.float32, device=dev)
    kc3, vc3 = kc.clone(), vc.clone()
    wf.wf_qk_norm_rope_append_fp8q(plan, r, q, k, v, None, gq, gk, None, q8b, qsb, kc3, vc3)
    statuses["append_q8"] = wf.wf_sync_status(plan)
    out.update(append_q8=q8b.cpu().numpy(), append_qs=qsb.cpu().numpy())
    Tv, Hv, Wv, Ci, Co = 3, 19, 21, 96, 160
    xv = wi.bf16_normal((Tv, Hv, Wv, Ci), 10, wi.STREAM_X).to(dev)
    hv = wi.bf16_normal((2, Hv, Wv, Ci), 10, wi.STREAM_CACHE).to(dev)
    wv = wi.bf16_weight(Co, 27 * Ci, 10).reshape(Co, 3, 3, 3, Ci).contiguous().to(dev)
    bv = wi.f32_vector((Co,), 0.1, 10, wi.STREAM_BIAS).to(dev)
    rv = wi.bf16_normal((Tv, Hv, Wv, Co), 10, wi.STREAM_MOD).to(dev)
    yv = torch.empty((Tv, Hv, Wv, Co), dtype=torch.bfloat16, device=dev)
    wf.wf_causal_conv3d(plan, xv, hv, wv, bv, rv, yv)
    statuses["conv"] = wf.wf_sync_status(plan)
    out["conv"] = yv.view(torch.int16).cpu().numpy()
    gv = (1 + wi.f32_vector((Ci,), 0.1, 10, wi.STREAM_GAMMA)).to(dev)
    nv = torch.empty_like(xv)
    wf.wf_rms_norm_silu(plan, xv, gv, nv)
    statuses["rms_norm_silu"] = wf.wf_sync_status(plan)
    out["rms_norm_silu"] = nv.view(torch.int16).cpu().numpy()
    plan.destroy()
    return out, statuses


if __name__ == "__main__":
    from chunk_causal_dit_b200 import wf
    assert os.path.basename(wf.LIB_PATH) == ("libwf_check.so"
                                             if os.environ.get("WF_LIB_VARIANT") == "check"
                                             else "libwf.so")
    outs, st = run_all(wf)
    np.savez(sys.argv[1], **outs, **{"status_" + k: np.int64(v) for k, v in st.items()})
