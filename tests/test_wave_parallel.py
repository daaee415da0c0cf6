"""Wave Parallelism host logic on CPU: the chunk partition, and the one-way K/V
exchange between gloo ranks over consecutive rounds.

The exchange tests run each rank's kernels with the oracle (CPU stand-ins
defined here, test-only), so every difference from the expected output is a
difference in what the rank's ring holds: which chunks it received, into
which slots, in which round.  The expectation is the oracle's own round (the
append and attention, or the whole DiT block of oracle/block.py), computed in
one process from absolute chunk ids with no ring at all.
"""
import itertools
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _work(W, Hh):
    return [Hh + c + 1 for c in range(W)]


def test_partition_is_contiguous_and_optimal():
    from chunk_causal_dit_b200.wave_parallel import partition
    for W in range(1, 8):
        for Hh in range(0, 4):
            w = _work(W, Hh)
            for world in range(1, W + 1):
                ranges = partition(W, Hh, world)
                assert ranges[0][0] == 0 and ranges[-1][1] == W and len(ranges) == world
                assert all(a < b for a, b in ranges)
                assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
                got = max(sum(w[a:b]) for a, b in ranges)
                best = min(max(sum(w[a:b]) for a, b in zip((0,) + cuts, cuts + (W,)))
                           for cuts in itertools.combinations(range(1, W), world - 1))
                assert got == best
    assert partition(5, 2, 5) == [(c, c + 1) for c in range(5)]
    assert partition(5, 2, 1) == [(0, 5)]
    with pytest.raises(ValueError):
        partition(3, 1, 4)


def test_exchange_lists_pair_up():
    """What rank j sends to rank k in a round is what rank k receives from j, in
    the same order; every earlier chunk reaches every later rank exactly once."""
    from chunk_causal_dit_b200.wave_parallel import WaveParallelRound
    W, Hh = 6, 2
    for world in (2, 3, 6):
        rs = [WaveParallelRound(16, W, Hh, 1, 64, (1, 4, 4), None, world=world, rank=k,
                                plan_factory=lambda *a: None) for k in range(world)]
        for r in (Hh, Hh + 5):
            for j, k in itertools.product(range(world), repeat=2):
                sent = [g for d, g in rs[j].outgoing(r) if d == k]
                got = [g for s, g in rs[k].incoming(r) if s == j]
                assert sent == got
            for k in range(world):
                need = {r + c for c in range(rs[k].c0)}
                assert sorted(g for _, g in rs[k].incoming(r)) == sorted(need)


# ---- the gloo exchange with oracle kernels -------------------------------------------

SHAPE = dict(F=2, gh=2, gw=4, H=2, D=64)     # L = 16


class OracleKernels:
    """Test-only CPU stand-ins for the append and the attention (the oracle), with
    the ring arithmetic of the GPU kernels: chunk g of a plan's wave goes to slot
    g mod R; the attention reads the visible chunk ids from their slots."""

    def __init__(self, gq, gk):
        import oracle
        from chunk_causal_dit_b200 import inputs as wi
        self.o, self.wi = oracle, wi
        self.gq, self.gk = gq.numpy(), gk.numpy()

    def append(self, plan, r, q, k, v, q_out, kc, vc):
        wi, o = self.wi, self.o
        pos = o.positions(r, plan.W, SHAPE["F"], SHAPE["gh"], SHAPE["gw"])
        qo, ko, vo = o.append(wi.bits(q), wi.bits(k), wi.bits(v), pos, self.gq, self.gk)
        q_out.copy_(wi.from_bits(qo))
        L = plan.L
        for c in range(plan.W):
            s = (r + c) % plan.R
            kc[s].copy_(wi.from_bits(ko[c * L:(c + 1) * L]))
            vc[s].copy_(wi.from_bits(vo[c * L:(c + 1) * L]))

    def attention(self, plan, r, q_out, kc, vc, o_out):
        wi, o = self.wi, self.o
        hv = min(plan.Hh, r)
        cache = o.OracleCache(plan.L)
        for b in range(hv + plan.W):
            g = r - hv + b
            cache.put(g, wi.bits(kc[g % plan.R]), wi.bits(vc[g % plan.R]))
        T = plan.W * plan.L
        rows = np.repeat(np.arange(T), plan.H)
        heads = np.tile(np.arange(plan.H), T)
        ref, _ = o.round_attention(cache, r, plan.W, plan.Hh, wi.bits(q_out), rows, heads)
        o_out.copy_(wi.from_bits(o.f64_to_bf16(ref)).view(o_out.shape))


class OracleBlockKernels(OracleKernels):
    """The block's calls on the oracle (test-only, CPU), with the GPU calls'
    conventions: the QKV projection writes q_out and the ring slots g mod R of the
    plan's chunks; linear layers may write their output over their residual."""

    def __init__(self, gq, gk):
        super().__init__(gq, gk)
        import oracle.block as ob
        from chunk_causal_dit_b200 import wf
        self.ob = ob
        self.epi = {wf.WF_EPI_STORE: "store", wf.WF_EPI_GELU_TANH: "gelu_tanh",
                    wf.WF_EPI_GATED_RESIDUAL: "gated_residual"}

    def layer_norm(self, plan, x, shift, scale, rpg, y):
        wi = self.wi
        y.copy_(wi.from_bits(self.ob.layer_norm_modulate(wi.bits(x), shift.numpy(),
                                                          scale.numpy(), rpg)))

    def qkv(self, plan, r, h, w_qkv, b_qkv, q_out, kc, vc):
        wi = self.wi
        pos = self.o.positions(r, plan.W, SHAPE["F"], SHAPE["gh"], SHAPE["gw"])
        q, k, v = self.ob.qkv_project_append(wi.bits(h), wi.bits(w_qkv), b_qkv.numpy(), pos,
                                             self.gq, self.gk, plan.H, plan.D)
        q_out.copy_(wi.from_bits(q))
        L = plan.L
        for c in range(plan.W):
            s = (r + c) % plan.R
            kc[s].copy_(wi.from_bits(k[c * L:(c + 1) * L]))
            vc[s].copy_(wi.from_bits(v[c * L:(c + 1) * L]))

    def linear(self, plan, x, w, y, bias, epilogue, gate, resid, rpg):
        wi = self.wi
        out = self.ob.linear(wi.bits(x), wi.bits(w), None if bias is None else bias.numpy(),
                             self.epi[epilogue], None if gate is None else gate.numpy(),
                             None if resid is None else wi.bits(resid), rpg)
        y.copy_(wi.from_bits(out))


BLOCK = dict(C=SHAPE["H"] * SHAPE["D"], FF=192)


def _block_weights(seed=9):
    from chunk_causal_dit_b200 import inputs as wi
    C, FF, HD = BLOCK["C"], BLOCK["FF"], SHAPE["H"] * SHAPE["D"]
    return {"w_qkv": wi.bf16_weight(3 * HD, C, seed, 1), "w_o": wi.bf16_weight(C, HD, seed, 2),
            "w_1": wi.bf16_weight(FF, C, seed, 3), "w_2": wi.bf16_weight(C, FF, seed, 4),
            "b_qkv": wi.f32_vector((3 * HD,), 0.02, seed, wi.STREAM_BIAS, 1),
            "b_o": wi.f32_vector((C,), 0.02, seed, wi.STREAM_BIAS, 2),
            "b_1": wi.f32_vector((FF,), 0.02, seed, wi.STREAM_BIAS, 3),
            "b_2": wi.f32_vector((C,), 0.02, seed, wi.STREAM_BIAS, 4)}


def _plan_factory(L, n, hist, H, D, rope):
    return SimpleNamespace(L=L, W=n, Hh=hist, H=H, D=D, R=hist + n)


def _inputs(W, Hh, rounds, seed=3):
    """Whole-wave q, k, v for each round and the clean history before the first."""
    from chunk_causal_dit_b200 import inputs as wi
    L, H, D = SHAPE["F"] * SHAPE["gh"] * SHAPE["gw"], SHAPE["H"], SHAPE["D"]
    xs = []
    for i in range(rounds):
        xs.append(tuple(wi.bf16_normal((W * L, H, D), seed + i, s) for s in range(3)))
    hk = wi.bf16_normal((Hh, L, H, D), seed, 3)
    hv = wi.bf16_normal((Hh, L, H, D), seed, 4)
    gq, gk = wi.gains(H, D, seed)
    return L, xs, hk, hv, gq, gk


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, W, Hh, r0, rounds, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from chunk_causal_dit_b200 import inputs as wi
    from chunk_causal_dit_b200.wave_parallel import WaveParallelRound
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L, xs, hk, hv, gq, gk = _inputs(W, Hh, rounds)
        H, D = SHAPE["H"], SHAPE["D"]
        wp = WaveParallelRound(L, W, Hh, H, D, (SHAPE["F"], SHAPE["gh"], SHAPE["gw"]),
                               OracleKernels(gq, gk), plan_factory=_plan_factory)
        kc = torch.zeros(wp.ring_shape(), dtype=torch.bfloat16)
        vc = torch.zeros_like(kc)
        wp.prefill_history(r0, [(r0 - Hh + j, hk[j], hv[j]) for j in range(Hh)], kc, vc)
        res = []
        rows = slice(wp.c0 * L, wp.c1 * L)
        for i in range(rounds):
            q, k, v = (t[rows].contiguous() for t in xs[i])
            q_out = torch.empty_like(q)
            o = torch.empty_like(q)
            wp.run_layer(r0 + i, q, k, v, q_out, kc, vc, o)
            res.append(wi.bits(o))
        wp.destroy()                             # waits for sends still in flight
        out[rank] = (wp.c0, wp.c1, res)
    finally:
        dist.destroy_process_group()


def _expected(W, Hh, r0, rounds):
    """The oracle's rounds from absolute chunk ids (no ring, no ranks)."""
    import oracle
    from chunk_causal_dit_b200 import inputs as wi
    L, xs, hk, hv, gq, gk = _inputs(W, Hh, rounds)
    H = SHAPE["H"]
    cache = oracle.OracleCache(L)
    for j in range(Hh):
        cache.put(r0 - Hh + j, wi.bits(hk[j]), wi.bits(hv[j]))
    outs = []
    for i in range(rounds):
        r = r0 + i
        q, k, v = xs[i]
        pos = oracle.positions(r, W, SHAPE["F"], SHAPE["gh"], SHAPE["gw"])
        qo, ko, vo = oracle.append(wi.bits(q), wi.bits(k), wi.bits(v), pos, gq.numpy(),
                                   gk.numpy())
        cache.put_wave(r, ko, vo)
        T = W * L
        rows = np.repeat(np.arange(T), H)
        heads = np.tile(np.arange(H), T)
        ref, _ = oracle.round_attention(cache, r, W, Hh, qo, rows, heads)
        outs.append(oracle.f64_to_bf16(ref).reshape(T, H, -1))
    return L, outs


@pytest.mark.parametrize("world,W,Hh", [(2, 3, 1), (3, 4, 2)])
def test_exchange_over_gloo_matches_single_wave(world, W, Hh):
    r0, rounds = Hh, 3          # the third round reads history that arrived as chunk 0
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, W, Hh, r0, rounds, out), nprocs=world,
                       join=True, start_method="spawn")
    L, expected = _expected(W, Hh, r0, rounds)
    covered = []
    for rank in range(world):
        c0, c1, res = out[rank]
        covered.extend(range(c0, c1))
        for i in range(rounds):
            want = expected[i][c0 * L:c1 * L]
            assert np.array_equal(res[i], want), "rank %d round %d" % (rank, i)
    assert covered == list(range(W))


def _rank_block_main(rank, world, port, W, Hh, r0, rounds, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from chunk_causal_dit_b200 import inputs as wi
    from chunk_causal_dit_b200.wave_parallel import WaveParallelRound
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L, xs, hk, hv, gq, gk = _inputs(W, Hh, rounds)
        H, D, C, FF = SHAPE["H"], SHAPE["D"], BLOCK["C"], BLOCK["FF"]
        w = _block_weights()
        mod = wi.f32_vector((6, W, C), 0.1, 9, wi.STREAM_MOD)
        wp = WaveParallelRound(L, W, Hh, H, D, (SHAPE["F"], SHAPE["gh"], SHAPE["gw"]),
                               OracleBlockKernels(gq, gk), plan_factory=_plan_factory)
        buf = {"h": torch.empty((wp.rows, C), dtype=torch.bfloat16),
               "q_out": torch.empty((wp.rows, H, D), dtype=torch.bfloat16),
               "o": torch.empty((wp.rows, H, D), dtype=torch.bfloat16),
               "f": torch.empty((wp.rows, FF), dtype=torch.bfloat16),
               "k_cache": torch.zeros(wp.ring_shape(), dtype=torch.bfloat16),
               "v_cache": torch.zeros(wp.ring_shape(), dtype=torch.bfloat16)}
        wp.prefill_history(r0, [(r0 - Hh + j, hk[j], hv[j]) for j in range(Hh)],
                           buf["k_cache"], buf["v_cache"])
        res = []
        for i in range(rounds):
            x = _block_x(W, L, i)[wp.c0 * L:wp.c1 * L].clone()
            wp.run_block(r0 + i, x, w, mod, buf)
            res.append(wi.bits(x))
        wp.destroy()
        out[rank] = (wp.c0, wp.c1, res)
    finally:
        dist.destroy_process_group()


def _block_x(W, L, i):
    from chunk_causal_dit_b200 import inputs as wi
    return wi.bf16_normal((W * L, BLOCK["C"]), 40 + i, wi.STREAM_X)


@pytest.mark.parametrize("world,W,Hh", [(2, 3, 1), (3, 4, 2)])
def test_block_exchange_over_gloo_matches_the_oracle_block(world, W, Hh):
    """run_block on gloo ranks (the exchange posted between the QKV projection and
    the attention) against oracle.block.block_forward of the whole wave, over two
    rounds (the second reads history delivered in the first)."""
    import oracle
    import oracle.block as ob
    from chunk_causal_dit_b200 import inputs as wi
    r0, rounds = Hh, 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_block_main, args=(world, port, W, Hh, r0, rounds, out),
                       nprocs=world, join=True, start_method="spawn")
    L, xs, hk, hv, gq, gk = _inputs(W, Hh, rounds)
    H, D, C = SHAPE["H"], SHAPE["D"], BLOCK["C"]
    w = _block_weights()
    wts = {k: (wi.bits(t) if t.dtype == torch.bfloat16 else t.numpy()) for k, t in w.items()}
    wts["gamma_q"], wts["gamma_k"] = gq.numpy(), gk.numpy()
    mod = wi.f32_vector((6, W, C), 0.1, 9, wi.STREAM_MOD).numpy()
    cache = oracle.OracleCache(L)
    for j in range(Hh):
        cache.put(r0 - Hh + j, wi.bits(hk[j]), wi.bits(hv[j]))
    for i in range(rounds):
        r = r0 + i
        pos = oracle.positions(r, W, SHAPE["F"], SHAPE["gh"], SHAPE["gw"])
        want, _ = ob.block_forward(wi.bits(_block_x(W, L, i)), wts, mod, pos, cache, r, W, Hh,
                                   H, D, L)
        for rank in range(world):
            c0, c1, res = out[rank]
            assert np.array_equal(res[i], want[c0 * L:c1 * L]), "rank %d round %d" % (rank, r)
