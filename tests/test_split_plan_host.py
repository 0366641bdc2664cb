"""The library's split plan for split-KV attention (wf_attn_split_plan), on the host.

A plan gives every unit (256 query rows x one head) S parts and the last units of the dispatch
order S + 1, chosen from a model of the grid on a given number of SMs.  These tests need the
library but no GPU: the plan is host logic when the SM count is given."""
import pytest

from block_causal_streaming_b200 import (WF_ERR_INVALID_ARG, WF_ERR_SHAPE, WavefrontDesc,
                                         WfError, attn_split_plan)
from block_causal_streaming_b200.workloads import WORKLOADS, small_case


def _desc(wl):
    return WavefrontDesc(wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks, wl.num_pages)


def _units(wl):
    return -(-wl.t_q // 256) * wl.heads


@pytest.mark.parametrize("name", ["wan13b_5step", "wan13b_4step", "wan14b", "wan13b_round30"])
def test_grids_of_two_waves_or_more_are_not_split(name):
    wl = WORKLOADS[name]
    assert _units(wl) >= 2 * 148
    assert attn_split_plan(_desc(wl), wl.heads, 0, 148) == (1, 0)


def test_the_rank_call_fills_whole_waves():
    """One Wave-Parallelism rank's call (228 units on 148 SMs): split, and when the plan has a
    tail its CTAs fill whole waves."""
    wl = WORKLOADS["wp_rank0"]
    parts, tail = attn_split_plan(_desc(wl), wl.heads, 0, 148)
    assert parts >= 2
    ctas = (_units(wl) - tail) * parts + tail * (parts + 1)
    if tail:
        assert 0 < tail <= _units(wl) and ctas % 148 == 0


def test_plans_change_with_the_sm_count_and_repeat():
    wl = WORKLOADS["wp_rank0"]
    d = _desc(wl)
    a = attn_split_plan(d, wl.heads, 0, 148)
    assert attn_split_plan(d, wl.heads, 0, 148) == a                # cached, same answer
    assert attn_split_plan(d, wl.heads, 0, 100) == (1, 0)           # 228 units: two waves
    for sms in (120, 132, 264, 456):
        parts, tail = attn_split_plan(d, wl.heads, 0, sms)
        assert 1 <= parts <= 16 and 0 <= tail <= _units(wl)
        assert tail == 0 or parts >= 2                  # no plan mixes whole and split units


def test_explicit_splits_are_uniform_and_capped_by_the_smallest_unit():
    wl = small_case("plan_cap", 2, 128, (100,), (300, 60), 64, seed=1)
    d = _desc(wl)
    # parts never exceed the key tiles of the smallest unit (its rows see 100 + 300 keys) or 16
    for s in (1, 2, 3):
        assert attn_split_plan(d, wl.heads, s, 148) == (s, 0)
    parts, tail = attn_split_plan(d, wl.heads, 16, 148)
    assert tail == 0 and 1 <= parts <= 16 and parts <= -(-(100 + 300) // 128)


def test_invalid_arguments():
    wl = WORKLOADS["wp_rank0"]
    d = _desc(wl)
    with pytest.raises(WfError) as e:
        attn_split_plan(d, wl.heads, -1, 148)
    assert e.value.code == WF_ERR_INVALID_ARG
    with pytest.raises(WfError) as e:
        attn_split_plan(d, 0, 0, 148)
    assert e.value.code == WF_ERR_INVALID_ARG
    ctx_only = WavefrontDesc([0, 64], [0], 1, 4)
    with pytest.raises(WfError) as e:
        attn_split_plan(ctx_only, 2, 0, 148)
    assert e.value.code == WF_ERR_SHAPE
