"""wf_attn_forward_split_noalloc: the split attention with the library's static scratch.

Collected last on purpose: it exercises the device-wide scratch array after every other test.
The entry point must give exactly what wf_attn_forward_split gives with a caller workspace, on
two calls in a row (the second reuses the scratch the first left behind), and must reject plans
larger than its 128 MiB."""
import ctypes

import pytest
import torch

from block_causal_streaming_b200 import (WF_ERR_CAPACITY, WF_ERR_INVALID_ARG, WF_OK, WfError,
                                         attn_forward_split_noalloc, attn_workspace_size,
                                         check_status)
from block_causal_streaming_b200.workloads import WP_RANK0, make_inputs, small_case

SCRATCH_BYTES = 128 << 20
FAKE = 0x10000


def test_noalloc_validation_without_a_gpu():
    from block_causal_streaming_b200 import _abi
    desc = _abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    pool = _abi.KvPool(k_pool=FAKE, v_pool=FAKE, num_pages=8, page_size=64, num_heads=2,
                       head_dim=128)
    pt = ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32))
    assert _abi.lib.wf_attn_forward_split_noalloc(FAKE, ctypes.byref(pool), pt,
                                                  ctypes.byref(desc.c), 0.1, FAKE, None, -1,
                                                  None) == WF_ERR_INVALID_ARG
    bad = _abi.KvPool(k_pool=FAKE, v_pool=FAKE, num_pages=8, page_size=24, num_heads=2,
                      head_dim=128)
    assert _abi.lib.wf_attn_forward_split_noalloc(FAKE, ctypes.byref(bad), pt,
                                                  ctypes.byref(desc.c), 0.1, FAKE, None, 2,
                                                  None) != WF_OK


def _compare_two_calls(wl, splits, rows=None, heads=None):
    """Two calls of the no-alloc entry point must equal the workspace entry point bit for bit,
    and the result must meet the parity bar against the oracle on its own (every element, or
    the given (row, head) pairs)."""
    import oracle
    from gpu_util import assert_parity, place
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    # the plan really splits, so the static scratch is in use
    assert attn_workspace_size(layer.desc, wl.heads, wl.head_dim, splits) > 0
    ref = torch.empty_like(q)
    ref_lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
    layer.forward(q, ref, lse=ref_lse, splits=splits)          # caller-workspace entry point
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        attn_forward_split_noalloc(q, layer.pool.k, layer.pool.v, layer.page_tables[0],
                                   layer.desc, 1.0 / wl.head_dim ** 0.5, out, splits, lse)
        assert check_status() == WF_OK
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
    scale = 1.0 / wl.head_dim ** 0.5
    if rows is None:
        want = oracle.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, scale)
        assert_parity(out.float().cpu().numpy(), want, f"{wl.name} no-alloc")
    else:
        want = oracle.attention_rows(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks,
                                     scale, rows, heads)
        assert_parity(out[rows, heads].float().cpu().numpy(), want, f"{wl.name} no-alloc")


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [2, 3])
def test_noalloc_matches_workspace_entry_on_two_calls(splits):
    _compare_two_calls(small_case("noalloc_d128", 2, 128, (300,), (20, 300, 129, 700), 64,
                                  seed=41), splits)


@pytest.mark.gpu
def test_noalloc_matches_on_the_wave_parallel_rank_call():
    wl = WP_RANK0
    assert 0 < attn_workspace_size(_desc(wl), wl.heads, wl.head_dim, 0) <= SCRATCH_BYTES
    from gpu_util import sample_rows
    rows, heads = sample_rows(wl, per_chunk=16, seed=41)
    _compare_two_calls(wl, 0, rows, heads)


@pytest.mark.gpu
def test_noalloc_rejects_plans_larger_than_its_scratch():
    from gpu_util import place
    wl = WP_RANK0
    assert attn_workspace_size(_desc(wl), wl.heads, wl.head_dim, 8) > SCRATCH_BYTES
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    with pytest.raises(WfError) as e:
        attn_forward_split_noalloc(q, layer.pool.k, layer.pool.v, layer.page_tables[0],
                                   layer.desc, 1.0 / wl.head_dim ** 0.5, torch.empty_like(q), 8)
    assert e.value.code == WF_ERR_CAPACITY
    assert check_status() == WF_OK


def _desc(wl):
    from block_causal_streaming_b200 import WavefrontDesc
    return WavefrontDesc(wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks, wl.pages_needed)
