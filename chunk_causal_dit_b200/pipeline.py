"""Streaming wave rounds from host memory through the C ABI.

A caller that keeps a layer's q/k/v on the host (pinned) and wants O back on
the host can run round after round with the copies of one round hidden under
the kernels of its neighbours.  This module only orders copies and launches
on CUDA streams (plumbing); every arithmetic step runs in libwf's kernels via
the binding in ``chunk_causal_dit_b200.wf``.

Per round i (staging slot s = i % 2):
  copy-in stream : q, k, v host -> device slot s   (after round i-2 released s)
  compute stream : wf_qk_norm_rope_append, wf_chunk_causal_attn (after copy-in);
                   with the FP8 Q.K^T variant: the append with fused Q quantization
                   (wf_qk_norm_rope_append_fp8q), wf_quantize_k_fp8 of the wave's chunks,
                   wf_chunk_causal_attn_fp8qk
  copy-out stream: O device slot s -> host         (after the attention)
"""
from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import torch

from . import wf


class HostRoundPipeline:
    """Runs consecutive rounds of one layer whose inputs/outputs live in pinned host memory.

    plan, k_cache, v_cache, gamma_q, gamma_k: as for the direct calls (device
    tensors).  pos_thw: optional device tensor [T, 3] (None = derived positions).
    fp8: optional (k8_cache, k_scale) device tensors; when given, every round runs
    the FP8 Q.K^T variant and keeps the E4M3 key ring up to date.
    """

    def __init__(self, plan: "wf.Plan", k_cache, v_cache, gamma_q, gamma_k,
                 pos_thw=None, device: Optional[torch.device] = None, fp8=None):
        self.plan = plan
        self.fp8 = fp8
        self.kc, self.vc = k_cache, v_cache
        self.gq, self.gk = gamma_q, gamma_k
        self.pos = pos_thw
        self.dev = device or k_cache.device
        shape = (plan.T, plan.H, plan.D)
        bf = torch.bfloat16
        self.q = [torch.empty(shape, dtype=bf, device=self.dev) for _ in range(2)]
        self.k = [torch.empty(shape, dtype=bf, device=self.dev) for _ in range(2)]
        self.v = [torch.empty(shape, dtype=bf, device=self.dev) for _ in range(2)]
        self.q_out = torch.empty(shape, dtype=bf, device=self.dev)
        self.o = [torch.empty(shape, dtype=bf, device=self.dev) for _ in range(2)]
        if fp8 is not None:
            self.q8 = torch.empty(shape, dtype=torch.uint8, device=self.dev)
            self.q_scale = torch.empty((plan.H, plan.T), dtype=torch.float32, device=self.dev)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.in_ready, self.in_free, self.o_ready, self.o_free = ev(), ev(), ev(), ev()
        for s in range(2):       # every slot starts free
            self.in_free[s].record(self.s_comp)
            self.o_free[s].record(self.s_out)

    def _copy_in(self, slot: int, hq, hk, hv):
        with torch.cuda.stream(self.s_in):
            self.s_in.wait_event(self.in_free[slot])
            self.q[slot].copy_(hq, non_blocking=True)
            self.k[slot].copy_(hk, non_blocking=True)
            self.v[slot].copy_(hv, non_blocking=True)
            self.in_ready[slot].record(self.s_in)

    def run(self, rounds: Sequence[Tuple[int, torch.Tensor, torch.Tensor, torch.Tensor,
                                         torch.Tensor]],
            start_event: Optional[torch.cuda.Event] = None,
            end_event: Optional[torch.cuda.Event] = None) -> None:
        """rounds: (round index, host q, host k, host v, host O) per round, in order.

        Host tensors must be pinned for the copies to overlap.  If given,
        start_event is recorded before the first copy and end_event after the
        last copy back, both on streams that bracket all the work.
        """
        rounds = list(rounds)
        if not rounds:
            return
        if start_event is not None:
            start_event.record(self.s_comp)
            self.s_in.wait_stream(self.s_comp)
            self.s_out.wait_stream(self.s_comp)
        self._copy_in(0, *rounds[0][1:4])
        for i, (r, _, _, _, ho) in enumerate(rounds):
            slot = i % 2
            if i + 1 < len(rounds):
                self._copy_in((i + 1) % 2, *rounds[i + 1][1:4])
            c = self.s_comp
            c.wait_event(self.in_ready[slot])
            c.wait_event(self.o_free[slot])
            if self.fp8 is None:
                wf.wf_qk_norm_rope_append(self.plan, r, self.q[slot], self.k[slot], self.v[slot],
                                          self.pos, self.gq, self.gk, self.q_out, self.kc,
                                          self.vc, c)
                self.in_free[slot].record(c)
                wf.wf_chunk_causal_attn(self.plan, r, self.q_out, self.kc, self.vc,
                                        self.o[slot], None, c)
            else:
                # the append writes q's E4M3 codes itself (no bf16 q_out round trip)
                k8, ks = self.fp8
                wf.wf_qk_norm_rope_append_fp8q(self.plan, r, self.q[slot], self.k[slot],
                                               self.v[slot], self.pos, self.gq, self.gk, None,
                                               self.q8, self.q_scale, self.kc, self.vc, c)
                self.in_free[slot].record(c)
                wf.wf_quantize_k_fp8(self.plan, r, self.plan.W, self.kc, k8, ks, c)
                wf.wf_chunk_causal_attn_fp8qk(self.plan, r, self.q8, self.q_scale, k8, ks,
                                              self.vc, self.o[slot], None, c)
            self.o_ready[slot].record(c)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.o_ready[slot])
                ho.copy_(self.o[slot], non_blocking=True)
                self.o_free[slot].record(self.s_out)
        if end_event is not None:
            self.s_comp.wait_stream(self.s_out)
            self.s_comp.wait_stream(self.s_in)
            end_event.record(self.s_comp)

    def synchronize(self) -> None:
        for s in (self.s_in, self.s_comp, self.s_out):
            s.synchronize()
