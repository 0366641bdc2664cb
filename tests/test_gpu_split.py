"""wf_attn_forward_split (split-KV) on the GPU against the oracle.

Each unit's key range is cut into S consecutive parts run by S CTAs whose partial results a
second kernel merges.  The result must meet the same parity bar as the single pass, whatever S,
including splits in which some rows of a unit see no key at all (their partial is empty)."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_streaming_b200 import (WF_ERR_CAPACITY, WF_OK, WfError, attn_forward_split,
                                         attn_workspace_size, check_status)
from block_causal_streaming_b200.workloads import WP_RANK0, make_inputs, small_case
from gpu_util import assert_parity, place, run, sample_rows, scale_of

pytestmark = pytest.mark.gpu

CASES = [
    # units straddle chunk edges: early rows see fewer keys than later splits start at
    small_case("split_d128_straddle", 2, 128, (300,), (20, 300, 129, 700), 64, seed=31),
    small_case("split_d64_ps16", 3, 64, (128, 64), (200, 333), 16, seed=32),
    small_case("split_d128_one_chunk_long_ctx", 2, 128, (1500, 900), (260,), 48, seed=33),
    small_case("split_d128_kmean", 1, 128, (700,), (500,), 128, seed=34, k_mean_offset=True),
]


def oracle_of(wl, inp):
    return oracle.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks,
                            scale_of(wl), with_lse=True)


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [2, 3, 5])
def test_forced_splits_every_element(wl, splits):
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
    layer.forward(q, out, lse=lse, splits=splits)
    assert check_status() == WF_OK
    ref, ref_lse = oracle_of(wl, inp)
    assert_parity(out.float().cpu().numpy(), ref, f"{wl.name} S={splits}")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)


def test_one_split_is_the_single_pass_bitwise():
    wl = CASES[0]
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    out1 = torch.empty_like(q)
    layer.forward(q, out1, splits=1)
    assert torch.equal(out1, run(layer, q))


def test_split_results_are_deterministic():
    wl = CASES[2]
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    a, b = torch.empty_like(q), torch.empty_like(q)
    layer.forward(q, a, splits=4)
    layer.forward(q, b, splits=4)
    assert torch.equal(a, b)


def test_too_small_workspace_is_rejected():
    wl = CASES[0]
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    need = attn_workspace_size(layer.desc, wl.heads, wl.head_dim, 3)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device=q.device)
    with pytest.raises(WfError) as e:
        attn_forward_split(q, layer.pool.k, layer.pool.v, layer.page_tables[0], layer.desc,
                           scale_of(wl), torch.empty_like(q), 3, ws)
    assert e.value.code == WF_ERR_CAPACITY


def test_wave_parallel_rank_call_library_choice_sampled_parity():
    """One rank's chunk (4680 queries) against its 37 440-key prefix: the library splits it."""
    wl = WP_RANK0
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    assert attn_workspace_size(layer.desc, wl.heads, wl.head_dim, 0) > 0   # split chosen
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
    layer.forward(q, out, lse=lse, splits=0)
    out2 = torch.empty_like(q)
    layer.forward(q, out2, splits=0)
    assert check_status() == WF_OK
    assert torch.equal(out, out2)
    assert torch.isfinite(out.float()).all()
    rows, heads = sample_rows(wl, per_chunk=24, seed=5)
    ref, ref_lse = oracle.attention_rows(inp.q, inp.k, inp.v, wl.chunk_offsets,
                                         wl.num_ctx_chunks, scale_of(wl), rows, heads,
                                         with_lse=True)
    assert_parity(out[rows, heads].float().cpu().numpy(), ref, wl.name)
    np.testing.assert_allclose(lse[heads, rows].cpu().numpy(), ref_lse, rtol=0, atol=2e-3)
    # the single pass agrees within the parity bar too
    single = run(layer, q)
    assert_parity(single[rows, heads].float().cpu().numpy(), ref, wl.name + " single pass")


def test_sixteen_splits_the_maximum():
    """A unit of 20 key tiles split 16 ways (and a request for more is capped at 16)."""
    wl = small_case("split_16", 1, 128, (2300,), (200,), 64, seed=35)
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    assert attn_workspace_size(layer.desc, 1, 128, 40) == \
        attn_workspace_size(layer.desc, 1, 128, 16)
    ref, ref_lse = oracle_of(wl, inp)
    for splits in (16, 40):
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
        layer.forward(q, out, lse=lse, splits=splits)
        assert check_status() == WF_OK
        assert_parity(out.float().cpu().numpy(), ref, f"S={splits}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)


def test_library_plan_with_a_tail_of_units_split_once_more_every_element():
    """A wavefront for which the library's plan (on a 148-SM B200) gives every unit 3 parts and
    the last units of the dispatch order 4, so that the CTAs fill whole waves: every element and
    every lse against the oracle, and rows of the units left whole by another plan equal too."""
    from block_causal_streaming_b200 import attn_split_plan
    wl = small_case("split_tail", 6, 128, (1200,), (2800, 300), 64, seed=91)
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    parts, tail = attn_split_plan(layer.desc, wl.heads, 0)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert (parts, tail) == attn_split_plan(layer.desc, wl.heads, 0, 148)
        assert tail > 0
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
    layer.forward(q, out, lse=lse, splits=0)
    assert check_status() == WF_OK
    ref, ref_lse = oracle_of(wl, inp)
    assert_parity(out.float().cpu().numpy(), ref, f"{wl.name} plan ({parts}, {tail})")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)

