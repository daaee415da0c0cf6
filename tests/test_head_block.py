"""Host logic of the attention's unit order (wf_attn_head_block, the plan's
head-block setting), on the CPU.

The choice is checked against an independent Python playthrough of the same
dynamic schedule (a priority queue of CTA finish times), and against the rules
the header states: at least 1 and at most `heads`; a block's visible keys and
values within half of L2 when more than one head; `heads` when every unit has a
CTA of its own.
"""
import heapq

import pytest

from chunk_causal_dit_b200 import build as wf_build


@pytest.fixture(scope="module")
def wf():
    wf_build.build()
    from chunk_causal_dit_b200 import wf as mod
    return mod


def _makespan(H, W, h_valid, L, g, n_ctas):
    n_kt = (L + 127) // 128
    n_qp = (n_kt + 1) // 2
    free = [0.0] * n_ctas
    for hb in range(0, H, g):
        for c in reversed(range(W)):
            for h in range(hb, min(H, hb + g)):
                for pair in range(n_qp):
                    single = (2 * pair + 1) * 128 >= L
                    d = (h_valid + c + 1) * n_kt * (0.93 if single else 1.0) + 3.0
                    t = heapq.heappop(free)
                    heapq.heappush(free, t + d)
    return max(free)


def _choice(H, W, h_valid, L, D, kb, l2, n_ctas):
    per_head = (h_valid + W) * L * D * (kb + 2)
    g_max = H if l2 <= 0 else max(1, min(H, int(0.5 * l2 / per_head)))
    best_g, best = g_max, None
    for g in range(g_max, 0, -1):
        m = _makespan(H, W, h_valid, L, g, n_ctas)
        if best is None or m < best * (1 - 2e-3):
            best_g, best = g, m
    return best_g


B200_L2 = 126 * 1024 * 1024

CASES = [
    # heads, wave chunks, valid history chunks, chunk tokens, head_dim, key bytes
    (12, 5, 2, 4680, 128, 2),     # Wan-1.3B 4-step wave
    (12, 5, 2, 4680, 128, 1),     # the same with E4M3 keys
    (12, 6, 3, 4680, 128, 2),     # 5-step wave
    (40, 5, 3, 4680, 128, 2),     # 14B wave
    (12, 5, 0, 4680, 128, 2),     # round 0: no history yet
    (7, 3, 2, 1000, 64, 2),
]


@pytest.mark.parametrize("H,W,hv,L,D,kb", CASES)
def test_choice_matches_an_independent_schedule_playthrough(wf, H, W, hv, L, D, kb):
    g = wf.wf_attn_head_block(H, W, hv, L, D, kb, B200_L2, 148)
    assert g == _choice(H, W, hv, L, D, kb, B200_L2, 148)
    assert 1 <= g <= H
    if g > 1:
        assert g * (hv + W) * L * D * (kb + 2) <= B200_L2 / 2


def test_headline_shape_takes_three_heads_per_block(wf):
    # 16.8 MB of visible keys and values per head: three heads fit in half of L2
    assert wf.wf_attn_head_block(12, 5, 2, 4680, 128, 2, B200_L2, 148) == 3


def test_small_problems_keep_all_heads_in_one_block(wf):
    # every unit has a CTA of its own, so every order ends at the same time
    assert wf.wf_attn_head_block(3, 4, 2, 300, 128, 2, B200_L2, 148) == 3
    assert wf.wf_attn_head_block(2, 3, 0, 32, 64, 2, B200_L2, 148) == 2
    # no L2 size known and one CTA: nothing to choose between
    assert wf.wf_attn_head_block(12, 5, 2, 4680, 128, 2, 0, 1) == 12


def test_large_heads_fall_back_to_one_head_per_block(wf):
    # one head's keys and values alone exceed half of a small L2
    assert wf.wf_attn_head_block(8, 5, 2, 4680, 128, 2, 16 << 20, 148) == 1


def test_argument_validation(wf):
    assert wf.wf_attn_head_block(0, 5, 2, 4680, 128, 2, B200_L2, 148) == -1
    assert wf.wf_attn_head_block(12, 0, 2, 4680, 128, 2, B200_L2, 148) == -1
    assert wf.wf_attn_head_block(12, 5, -1, 4680, 128, 2, B200_L2, 148) == -1
    assert wf.wf_attn_head_block(12, 5, 2, 0, 128, 2, B200_L2, 148) == -1
    assert wf.wf_attn_head_block(12, 5, 2, 4680, 128, 3, B200_L2, 148) == -1
    # outside 1..1024 CTAs: the L2 cap alone
    assert wf.wf_attn_head_block(12, 5, 2, 4680, 128, 2, B200_L2, 0) == 3
    assert wf.wf_attn_head_block(12, 5, 2, 4680, 128, 2, B200_L2, 2000) == 3


def test_plan_setting(wf):
    plan = wf.Plan(300, 4, 2, 5, 128)
    # without a device the plan knows no L2 size and no SM count: all heads
    assert plan.head_block(3) in (1, 2, 3, 4, 5)
    for g in (1, 2, 5):
        plan.set_head_block(g)
        assert plan.head_block(3) == g and plan.head_block(0, fp8_keys=True) == g
    plan.set_head_block(0)
    for bad in (-1, 6):
        with pytest.raises(wf.WFError) as e:
            plan.set_head_block(bad)
        assert e.value.status == wf.WF_ERR_INVALID_ARG
    assert plan.head_block(-1) == -1
    plan.destroy()
