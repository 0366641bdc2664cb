"""The input recipe (block_causal_streaming_b200.workloads) on the CPU.

The named workloads must have the sizes, stages and page geometry the benchmark configurations
state.  Inputs must be reproducible from the seed, page tables must be valid permutations, and
the value distributions must be the stated ones.  Statistical checks use tolerances far wider
than their sampling error at these sizes.
"""
import math

import pytest
import torch

from block_causal_streaming_b200.workloads import (CHUNK_TOKENS, TINY, WAN13B_4STEP, WAN13B_5STEP,
                                                   WAN13B_ROUND30, WAN14B, WORKLOADS, WP_RANK0,
                                                   make_inputs, make_layers, small_case)


def test_chunk_is_three_latent_frames_of_30_by_52_patches():
    assert CHUNK_TOKENS == 3 * 30 * 52 == 4680


@pytest.mark.parametrize("wl,h,d,t_q,t_kv,ps,stages", [
    (TINY, 2, 64, 144, 144, 16, (200, 600, 1000)),
    (WAN13B_5STEP, 12, 128, 23400, 32760, 64, (200, 400, 600, 800, 1000)),
    (WAN13B_4STEP, 12, 128, 18720, 37440, 64, (250, 500, 750, 1000)),
    (WAN13B_ROUND30, 12, 128, 23400, 32760, 64, (200, 400, 600, 800, 1000)),
    (WAN14B, 40, 128, 23400, 51480, 128, (200, 400, 600, 800, 1000)),
    (WP_RANK0, 12, 128, 4680, 37440, 64, (1000,)),
], ids=lambda x: getattr(x, "name", None))
def test_named_workloads_have_the_stated_geometry(wl, h, d, t_q, t_kv, ps, stages):
    assert (wl.heads, wl.head_dim, wl.t_q, wl.t_kv, wl.page_size) == (h, d, t_q, t_kv, ps)
    off = wl.chunk_offsets
    assert off[0] == 0 and off[-1] == t_kv and all(a <= b for a, b in zip(off, off[1:]))
    assert off[-1] - off[wl.num_ctx_chunks] == t_q
    assert tuple(wl.chunk_stage[wl.num_ctx_chunks:]) == stages
    assert all(s == 0 for s in wl.chunk_stage[:wl.num_ctx_chunks])
    assert wl.pages_needed == math.ceil(t_kv / ps)


def test_workload_table_names_every_bench_workload():
    assert WORKLOADS["wan13b_5step"] is WAN13B_5STEP and WORKLOADS["wp_rank0"] is WP_RANK0
    assert len({w.seed for w in WORKLOADS.values()}) == len(WORKLOADS)   # one seed each


def test_inputs_are_reproducible_from_the_seed_and_differ_between_seeds():
    a, b = make_inputs(TINY), make_inputs(TINY)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.page_table, b.page_table)):
        assert torch.equal(x, y)
    other = small_case("other", TINY.heads, TINY.head_dim, (), (48, 48, 48), 16, seed=99)
    assert not torch.equal(make_inputs(other).q, a.q)


def test_shapes_dtypes_and_identity_pages_of_the_tiny_workload():
    inp = make_inputs(TINY)
    assert inp.q.shape == (144, 2, 64) and inp.k.shape == (144, 2, 64) == inp.v.shape
    assert inp.q.dtype == inp.k.dtype == inp.v.dtype == torch.bfloat16
    assert torch.equal(inp.page_table, torch.arange(9, dtype=torch.int32))


def test_five_step_values_are_half_a_standard_normal_and_pages_a_permutation():
    inp = make_inputs(WAN13B_5STEP)
    for x in (inp.q, inp.k, inp.v):
        x = x.float()
        assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 0.5) < 0.01
    pt = inp.page_table
    assert pt.dtype == torch.int32 and torch.equal(pt.sort().values, torch.arange(512, dtype=torch.int32))
    assert not torch.equal(pt, torch.arange(512, dtype=torch.int32))


def test_four_step_keys_carry_one_mean_vector_per_head():
    inp = make_inputs(WAN13B_4STEP)
    k, q = inp.k.float(), inp.q.float()
    assert abs(q.std().item() - 1.0) < 0.01
    mu = k.mean(dim=0)                                     # [H, D], one offset per head
    resid = k - mu
    assert abs(resid.std().item() - 1.0) < 0.01            # N(0,1) around the offset
    assert 0.8 < mu.std().item() < 1.2                     # the offset itself is ~N(0,1)
    assert len(set(inp.page_table.tolist())) == 585


def test_the_round_draws_distinct_layers_with_pages_from_one_pool():
    layers = make_layers(WAN13B_ROUND30, layers=2)         # the first two of the 30 layers
    a, b = layers
    assert not torch.equal(a.q, b.q)
    for inp in layers:
        pt = inp.page_table.tolist()
        assert len(pt) == 512 and len(set(pt)) == 512 and 0 <= min(pt) and max(pt) < 4096
    assert torch.equal(make_layers(WAN13B_ROUND30, layers=1)[0].page_table, a.page_table)
