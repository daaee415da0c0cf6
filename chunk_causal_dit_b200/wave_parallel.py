"""Wave Parallelism: one wave round split over ranks by wave chunk.

"Wave Forcing" (abstract) runs the chunks of a wave on separate GPUs (Wave
Parallelism) and delivers each layer's K/V early and one way: from the GPU of a
chunk to the GPUs of later chunks, overlapped with the computation.  Query
chunk c attends to the history and to chunks 0..c, so nothing flows backwards.

Decomposition.  Rank k owns the contiguous wave chunks [c0, c1) (``partition``
balances the attention work, which grows with the number of chunks a query
chunk reads).  It keeps a K/V ring of its own, R_k = Hh + c1 slots, and a plan of
its own, Plan(L, c1 - c0, Hh + c0, H, D), called with round r + c0:

* The plan's wave is the rank's chunks, absolute ids r + c0 .. r + c1 - 1. The
  append writes them to slots g mod R_k, with the RoPE time of their own
  absolute chunk.
* The plan's history is Hh + c0 chunks, of which min(Hh + c0, r + c0) are
  visible. These are the global history r - Hh .. r - 1 plus the earlier wave
  chunks r .. r + c0 - 1, which other ranks own.
* The ring holds the last R_k chunk ids, so a slot is reused only after its
  chunk has left every window the rank reads.  This is the single-GPU ring,
  distributed.

Per layer, each rank:
1. appends its chunks' K/V;
2. sends them to every later rank (one message per chunk for K and one for V)
   and receives the chunks of every earlier rank into its own slots;
3. runs the chunk-causal attention of its own query chunks.

History chunks are wave chunk 0 of earlier rounds, the refresh chunk of the
rank that owns chunk 0. They arrived then and stay in the ring.  The sends are
posted right after the append, before the sender's attention.  The first rank
receives nothing, so its attention overlaps its sends.  A receiver's attention
waits for its whole exchange, its own sends included: point-to-point
operations posted together complete together.

This module computes nothing.  The append and the attention are libwf kernels
(``LibwfKernels``). For the CPU tests of the exchange they are whatever
``kernels`` object the caller passes.  The exchange is torch.distributed
point-to-point (NCCL between GPUs).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def partition(W: int, n_hist: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous chunk ranges [c0, c1) for ranks 0..world-1, every rank at least one
    chunk, minimising the largest per-rank attention work (query chunk c reads
    n_hist + c + 1 chunks, so its work is proportional to that count).  Ties go
    to the split with the most chunks on the earliest ranks."""
    if not 1 <= world <= W:
        raise ValueError("world size %d must be between 1 and the %d wave chunks" % (world, W))
    work = [n_hist + c + 1 for c in range(W)]
    pre = [0]
    for x in work:
        pre.append(pre[-1] + x)
    INF = float("inf")
    # best[k][j]: smallest max-work splitting chunks [0, j) over k ranks
    best = [[INF] * (W + 1) for _ in range(world + 1)]
    cut = [[0] * (W + 1) for _ in range(world + 1)]
    best[0][0] = 0
    for k in range(1, world + 1):
        for j in range(k, W + 1):
            for i in range(j - 1, k - 2, -1):          # last rank takes [i, j)
                v = max(best[k - 1][i], pre[j] - pre[i])
                if v < best[k][j]:
                    best[k][j], cut[k][j] = v, i
    ranges = []
    j = W
    for k in range(world, 0, -1):
        i = cut[k][j]
        ranges.append((i, j))
        j = i
    return ranges[::-1]


class LibwfKernels:
    """The two hot-path calls of a rank, on the current CUDA stream (the stream
    torch.distributed orders its point-to-point operations against)."""

    def __init__(self, gamma_q, gamma_k):
        from . import wf
        self.wf = wf
        self.gq, self.gk = gamma_q, gamma_k

    def append(self, plan, round_: int, q, k, v, q_out, k_cache, v_cache) -> None:
        self.wf.wf_qk_norm_rope_append(plan, round_, q, k, v, None, self.gq, self.gk, q_out,
                                       k_cache, v_cache)

    def attention(self, plan, round_: int, q_out, k_cache, v_cache, o) -> None:
        self.wf.wf_chunk_causal_attn(plan, round_, q_out, k_cache, v_cache, o, None)

    # the DiT block's calls (run_block)
    def layer_norm(self, plan, x, shift, scale, rows_per_group, y) -> None:
        self.wf.wf_layer_norm_modulate(plan, x, shift, scale, rows_per_group, y)

    def qkv(self, plan, round_: int, h, w_qkv, b_qkv, q_out, k_cache, v_cache) -> None:
        self.wf.wf_qkv_proj_norm_rope_append(plan, round_, h, w_qkv, b_qkv, self.gq, self.gk,
                                             q_out, k_cache, v_cache)

    def linear(self, plan, x, w, y, bias, epilogue, gate, resid, rows_per_group) -> None:
        self.wf.wf_linear(plan, x, w, y, bias, epilogue, gate, resid, rows_per_group)


def libwf_plan(L: int, n_wave: int, n_hist: int, H: int, D: int, rope: Tuple[int, int, int]):
    from . import wf
    return wf.Plan(L, n_wave, n_hist, H, D).set_rope(*rope)


class WaveParallelRound:
    """One rank's share of a wave round (see the module docstring).

    L, W, n_hist, H, D: the whole wave's shape; rope = (F, grid_h, grid_w).
    group: a torch.distributed process group (None: the default group if one is
    initialised, else a single rank).  kernels: an object with ``append`` and
    ``attention`` as ``LibwfKernels``; plan_factory(L, n, hist, H, D, rope) builds
    the rank's plan (default: libwf's).  world and rank, when given, fix the
    decomposition without a process group (``exchange`` is then unavailable;
    ``incoming`` / ``outgoing`` still describe it).
    """

    def __init__(self, L: int, W: int, n_hist: int, H: int, D: int,
                 rope: Tuple[int, int, int], kernels, group=None,
                 plan_factory: Optional[Callable] = None, world: Optional[int] = None,
                 rank: Optional[int] = None):
        self.emulated = world is not None
        if self.emulated:
            if rank is None or not 0 <= rank < world:
                raise ValueError("rank %r out of range for world %r" % (rank, world))
            self.group, self.world, self.rank = None, world, rank
        elif dist.is_available() and dist.is_initialized():
            self.group = group
            self.world = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        else:
            self.group, self.world, self.rank = None, 1, 0
        self.L, self.W, self.n_hist, self.H, self.D = L, W, n_hist, H, D
        self.ranges = partition(W, n_hist, self.world)
        self.c0, self.c1 = self.ranges[self.rank]
        self.n = self.c1 - self.c0
        self.R = n_hist + self.c1                 # this rank's ring slots
        self.kernels = kernels
        self.plan = (plan_factory or libwf_plan)(L, self.n, n_hist + self.c0, H, D, rope)
        self._pending = []                        # sends not yet waited for (see exchange)

    # ---- layout of the rank's tensors ----
    @property
    def rows(self) -> int:
        """Wave tokens this rank owns (q, k, v, q_out and o are [rows, H, D])."""
        return self.n * self.L

    def ring_shape(self) -> Tuple[int, int, int, int]:
        return (self.R, self.L, self.H, self.D)

    def slot(self, chunk_id: int) -> int:
        return chunk_id % self.R

    def _peer(self, k: int) -> int:
        """Global rank of group rank k."""
        return k if self.group is None else dist.get_global_rank(self.group, k)

    # ---- the exchange ----
    def outgoing(self, round_: int) -> List[Tuple[int, int]]:
        """(destination rank, absolute chunk id) of every chunk this rank sends in
        round `round_`: its own chunks, to every later rank, in chunk order."""
        return [(k, round_ + c) for k in range(self.rank + 1, self.world)
                for c in range(self.c0, self.c1)]

    def incoming(self, round_: int) -> List[Tuple[int, int]]:
        """(source rank, absolute chunk id) of every chunk this rank receives in
        round `round_`: the chunks of every earlier rank, in chunk order."""
        return [(k, round_ + c) for k in range(self.rank)
                for c in range(self.ranges[k][0], self.ranges[k][1])]

    def exchange_ops(self, round_: int, k_cache, v_cache) -> List["dist.P2POp"]:
        """Point-to-point operations of round `round_` (``outgoing`` as sends,
        ``incoming`` as receives into this rank's slots), K before V per chunk;
        both ends of a pair enumerate the same chunks in the same order."""
        ops = []
        for k, g in self.outgoing(round_):
            s = self.slot(g)
            ops.append(dist.P2POp(dist.isend, k_cache[s], self._peer(k), self.group))
            ops.append(dist.P2POp(dist.isend, v_cache[s], self._peer(k), self.group))
        for k, g in self.incoming(round_):
            s = self.slot(g)
            ops.append(dist.P2POp(dist.irecv, k_cache[s], self._peer(k), self.group))
            ops.append(dist.P2POp(dist.irecv, v_cache[s], self._peer(k), self.group))
        return ops

    def exchange(self, round_: int, k_cache, v_cache) -> None:
        """Post this round's sends and receives as one batch.  A rank that receives
        nothing (the first rank) does not wait for its sends: its attention only
        reads the slots being sent, so the delivery overlaps it; the sends are
        waited for before the rank next writes its ring (``settle``).  A rank that
        receives waits for the whole batch (sends and receives posted together
        complete together; posting them as two batches would serialise the ranks)."""
        if self.world == 1:
            return
        if self.emulated:
            raise RuntimeError("an emulated rank has no process group to exchange over")
        self.settle()
        ops = self.exchange_ops(round_, k_cache, v_cache)
        if not ops:
            return
        works = dist.batch_isend_irecv(ops)
        if self.incoming(round_):
            for work in works:
                work.wait()
        else:
            self._pending = list(works)

    def settle(self) -> None:
        """Wait for sends still in flight (before the ring is written again)."""
        for work in self._pending:
            work.wait()
        self._pending = []

    def run_layer(self, round_: int, q, k, v, q_out, k_cache, v_cache, o) -> None:
        """One layer of round `round_` for this rank's chunks: append, exchange,
        attention.  q, k, v, q_out, o: [rows, H, D]; k_cache, v_cache: ring_shape()."""
        r = round_ + self.c0
        self.settle()
        self.kernels.append(self.plan, r, q, k, v, q_out, k_cache, v_cache)
        self.exchange(round_, k_cache, v_cache)
        self.kernels.attention(self.plan, r, q_out, k_cache, v_cache, o)

    def run_block(self, round_: int, x, w, mod, buf) -> None:
        """One DiT block of round `round_` for this rank's chunks (the whole block
        runs on the rank's rows; the only exchange is the K/V delivery between the
        QKV projection and the attention):

        * x [rows, C]: the rank's residual stream, updated in place;
        * w: dict of the block's weights (w_qkv, b_qkv, w_o, b_o, w_1, b_1, w_2,
          b_2), as ``wf_linear`` / ``wf_qkv_proj_norm_rope_append`` take them;
        * mod [6, W, C]: the whole wave's modulation rows (shift, scale and gate
          of the attention half, then of the feed-forward half); the rank uses
          rows c0..c1-1;
        * buf: dict of work buffers h [rows, C], q_out and o [rows, H, D], f
          [rows, F], and the ring k_cache, v_cache (ring_shape()).
        The kernels object needs ``layer_norm``, ``qkv``, ``attention`` and
        ``linear`` (as ``LibwfKernels``)."""
        m = self.mod_rows(mod)
        self.norm_and_qkv(round_, x, w, m, buf)
        self.exchange(round_, buf["k_cache"], buf["v_cache"])
        self.attention_and_rest(round_, x, w, m, buf)

    def mod_rows(self, mod):
        """This rank's six modulation row blocks of a wave's table [6, W, C]."""
        return [mod[i, self.c0:self.c1] for i in range(6)]

    def norm_and_qkv(self, round_: int, x, w, m, buf) -> None:
        """The block before the delivery: LayerNorm + modulation and the QKV
        projection, whose epilogue appends this rank's K/V to its ring."""
        k, plan = self.kernels, self.plan
        self.settle()
        k.layer_norm(plan, x, m[0], m[1], self.L, buf["h"])
        k.qkv(plan, round_ + self.c0, buf["h"], w["w_qkv"], w["b_qkv"], buf["q_out"],
              buf["k_cache"], buf["v_cache"])

    def attention_and_rest(self, round_: int, x, w, m, buf) -> None:
        """The block after the delivery: attention, output projection, norm and
        feed-forward layers (m: the rank's six modulation row blocks)."""
        from .wf import WF_EPI_GATED_RESIDUAL, WF_EPI_GELU_TANH
        k, plan, L = self.kernels, self.plan, self.L
        r = round_ + self.c0
        k.attention(plan, r, buf["q_out"], buf["k_cache"], buf["v_cache"], buf["o"])
        o2 = buf["o"].view(self.rows, self.H * self.D)
        k.linear(plan, o2, w["w_o"], x, w["b_o"], WF_EPI_GATED_RESIDUAL, m[2], x, L)
        k.layer_norm(plan, x, m[3], m[4], L, buf["h"])
        k.linear(plan, buf["h"], w["w_1"], buf["f"], w["b_1"], WF_EPI_GELU_TANH, None, None, 1)
        k.linear(plan, buf["f"], w["w_2"], x, w["b_2"], WF_EPI_GATED_RESIDUAL, m[5], x, L)

    def prefill_history(self, round_: int, history: Sequence[Tuple[int, torch.Tensor, torch.Tensor]],
                        k_cache, v_cache) -> None:
        """Place clean history chunks (absolute id, K, V) into the ring before round
        `round_` (ids round_ - n_hist .. round_ - 1 are the ones read)."""
        for g, kk, vv in history:
            k_cache[self.slot(g)].copy_(kk)
            v_cache[self.slot(g)].copy_(vv)

    def destroy(self) -> None:
        self.settle()
        if hasattr(self.plan, "destroy"):
            self.plan.destroy()
