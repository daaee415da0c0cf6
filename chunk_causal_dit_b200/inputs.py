"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and lays out shapes; it holds none of the
method's arithmetic (no norm, no rotation, no softmax, no positions).  Both
sides receive the same bf16 bit patterns.

Recipe: every tensor is drawn from a CPU ``torch.Generator`` seeded with
``seed * 16 + stream`` (streams: q=0, k=1, v=2, cache pre-fill=3, gains=4),
as float32 N(0, 1) and rounded to bf16 by torch (round-to-nearest-even).
Gains are ``1 + 0.1 * N(0, 1)`` in float32.  Unit-scale N(0,1) activations
stand in for the projections of a trained Wan-style DiT layer (no weights
are available); the shapes follow the workloads named below.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

STREAM_Q, STREAM_K, STREAM_V, STREAM_CACHE, STREAM_GAMMA = 0, 1, 2, 3, 4
STREAM_X, STREAM_W, STREAM_BIAS, STREAM_MOD = 5, 6, 7, 8


@dataclass(frozen=True)
class Workload:
    """Shape of one wave round.

    L: tokens per chunk (= F * gh * gw); n_wave: chunks in the wave (denoising
    chunks + 1 refresh chunk); n_hist: history chunks in the ring; H, D: heads
    and head_dim; F, gh, gw: latent frames per chunk and the patch grid.
    """
    name: str
    H: int
    D: int
    F: int
    gh: int
    gw: int
    n_wave: int
    n_hist: int
    layers: int = 1
    rounds: int = 1

    @property
    def L(self) -> int:
        return self.F * self.gh * self.gw

    @property
    def T(self) -> int:
        return self.n_wave * self.L

    @property
    def R(self) -> int:
        return self.n_hist + self.n_wave


# The five workloads of the wave-round hot path.
WORKLOADS = {
    "tiny": Workload("tiny: 2x64, 3 chunks x 32 tokens (2x4x4), no history",
                     H=2, D=64, F=2, gh=4, gw=4, n_wave=3, n_hist=0),
    "wan13b_4step": Workload("wan1.3b 4-step wave: 12x128, 5 chunks x 4680 (3x30x52), history 2",
                             H=12, D=128, F=3, gh=30, gw=52, n_wave=5, n_hist=2),
    "wan13b_5step": Workload("wan1.3b 5-step wave: 12x128, 6 chunks x 4680, history 3",
                             H=12, D=128, F=3, gh=30, gw=52, n_wave=6, n_hist=3),
    "wan13b_round": Workload("wan1.3b full round: 30 layers of the 4-step wave, 20 rounds",
                             H=12, D=128, F=3, gh=30, gw=52, n_wave=5, n_hist=2,
                             layers=30, rounds=20),
    "wan14b_4step": Workload("wan14b 4-step wave: 40x128, 5 chunks x 4680, history 3",
                             H=40, D=128, F=3, gh=30, gw=52, n_wave=5, n_hist=3),
}


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 16 + int(stream))
    return g


def bf16_normal(shape, seed: int, stream: int) -> torch.Tensor:
    """bf16 CPU tensor of N(0,1) draws, rounded from float32."""
    x = torch.randn(tuple(shape), generator=_gen(seed, stream), dtype=torch.float32)
    return x.to(torch.bfloat16)


def gains(H: int, D: int, seed: int) -> "tuple[torch.Tensor, torch.Tensor]":
    """(gamma_q, gamma_k) float32 [H, D], each 1 + 0.1*N(0,1)."""
    g = torch.randn((2, H, D), generator=_gen(seed, STREAM_GAMMA), dtype=torch.float32)
    return (1.0 + 0.1 * g[0]).contiguous(), (1.0 + 0.1 * g[1]).contiguous()


@dataclass
class WaveInputs:
    q: torch.Tensor          # bf16 [T, H, D]
    k: torch.Tensor          # bf16 [T, H, D]
    v: torch.Tensor          # bf16 [T, H, D]
    gamma_q: torch.Tensor    # f32 [H, D]
    gamma_k: torch.Tensor    # f32 [H, D]


def wave_inputs(w: Workload, seed: int = 0, salt: int = 0) -> WaveInputs:
    """q, k, v of one wave round plus the RMSNorm gains.

    ``salt`` gives further independent draws (other layers, other rounds).
    """
    s = seed + 1009 * salt
    shape = (w.T, w.H, w.D)
    gq, gk = gains(w.H, w.D, seed)
    return WaveInputs(bf16_normal(shape, s, STREAM_Q), bf16_normal(shape, s, STREAM_K),
                      bf16_normal(shape, s, STREAM_V), gq, gk)


def history_prefill(w: Workload, n_chunks: Optional[int] = None, seed: int = 0,
                    salt: int = 0) -> "tuple[torch.Tensor, torch.Tensor]":
    """Clean history K/V [n_chunks, L, H, D] bf16 to seed the ring before round n_hist."""
    n = w.n_hist if n_chunks is None else n_chunks
    g = torch.randn((2, n, w.L, w.H, w.D), generator=_gen(seed + 1009 * salt, STREAM_CACHE),
                    dtype=torch.float32).to(torch.bfloat16)
    return g[0].contiguous(), g[1].contiguous()


def bf16_weight(out_features: int, in_features: int, seed: int, salt: int = 0) -> torch.Tensor:
    """A random-init linear weight [out, in]: N(0, 1/in) draws rounded to bf16."""
    g = _gen(seed + 1009 * salt, STREAM_W)
    w = torch.randn((out_features, in_features), generator=g, dtype=torch.float32)
    return (w * in_features ** -0.5).to(torch.bfloat16)


def f32_vector(shape, scale: float, seed: int, stream: int, salt: int = 0) -> torch.Tensor:
    """float32 N(0, scale^2) draws (biases, modulation tables)."""
    g = _gen(seed + 1009 * salt, stream)
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32) * scale


# Hidden and feed-forward widths of the Wan2.1-T2V-1.3B block (12 heads x 128 = 1536).
WAN13B_HIDDEN = 1536
WAN13B_FFN = 8960
# (hidden, feed-forward) widths of the block by attention width H*D: the 1.3B model
# (12 x 128) and the 14B model (40 x 128).
BLOCK_WIDTHS = {12 * 128: (WAN13B_HIDDEN, WAN13B_FFN), 40 * 128: (5120, 13824)}


@dataclass
class BlockInputs:
    x: torch.Tensor          # bf16 [T, C] residual stream entering the block
    w_qkv: torch.Tensor      # bf16 [3HD, C]
    b_qkv: torch.Tensor      # f32 [3HD]
    w_o: torch.Tensor        # bf16 [C, HD]
    b_o: torch.Tensor        # f32 [C]
    w_1: torch.Tensor        # bf16 [F, C]
    b_1: torch.Tensor        # f32 [F]
    w_2: torch.Tensor        # bf16 [C, F]
    b_2: torch.Tensor        # f32 [C]
    mod: torch.Tensor        # f32 [6, n_wave, C]: shift/scale/gate of attention, then of the FFN
    gamma_q: torch.Tensor    # f32 [H, D]
    gamma_k: torch.Tensor    # f32 [H, D]


def block_inputs(w: Workload, hidden: int, ffn: int, seed: int = 0) -> BlockInputs:
    """Random-init weights and one wave's residual stream for a DiT block of width
    ``hidden`` (= H*D for the Wan shapes) and feed-forward width ``ffn``.  Each wave
    chunk gets its own modulation rows (its own denoising step)."""
    HD = w.H * w.D
    gq, gk = gains(w.H, w.D, seed)
    return BlockInputs(
        x=bf16_normal((w.T, hidden), seed, STREAM_X),
        w_qkv=bf16_weight(3 * HD, hidden, seed, 1), b_qkv=f32_vector((3 * HD,), 0.02, seed, STREAM_BIAS, 1),
        w_o=bf16_weight(hidden, HD, seed, 2), b_o=f32_vector((hidden,), 0.02, seed, STREAM_BIAS, 2),
        w_1=bf16_weight(ffn, hidden, seed, 3), b_1=f32_vector((ffn,), 0.02, seed, STREAM_BIAS, 3),
        w_2=bf16_weight(hidden, ffn, seed, 4), b_2=f32_vector((hidden,), 0.02, seed, STREAM_BIAS, 4),
        mod=f32_vector((6, w.n_wave, hidden), 0.1, seed, STREAM_MOD),
        gamma_q=gq, gamma_k=gk)


def block_weights_on(device, w: Workload, hidden: int, ffn: int, seed: int, layer: int):
    """Random-init weights of one block drawn on `device` from a seeded generator
    there (faster than host draws for many layers): the same recipe as
    ``block_inputs`` (weights N(0, 1/in) in bf16, biases 0.02 N(0,1), modulation
    0.1 N(0,1) per wave chunk), a different stream of numbers."""
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1009 + int(layer)) * 16 + STREAM_W)
    HD = w.H * w.D

    def wt(o, i):
        return (torch.randn((o, i), generator=g, device=device) * i ** -0.5).to(torch.bfloat16)

    def vec(shape, scale):
        return torch.randn(shape, generator=g, device=device) * scale
    return dict(w_qkv=wt(3 * HD, hidden), b_qkv=vec((3 * HD,), 0.02),
                w_o=wt(hidden, HD), b_o=vec((hidden,), 0.02),
                w_1=wt(ffn, hidden), b_1=vec((ffn,), 0.02),
                w_2=wt(hidden, ffn), b_2=vec((hidden,), 0.02),
                mod=vec((6, w.n_wave, hidden), 0.1),
                gamma_q=(1.0 + 0.1 * torch.randn((w.H, w.D), generator=g, device=device)),
                gamma_k=(1.0 + 0.1 * torch.randn((w.H, w.D), generator=g, device=device)))


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (same memory order)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
