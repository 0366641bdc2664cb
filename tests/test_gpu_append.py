"""wf_kv_append on the GPU against the oracle's paged layout: bit-exact, nothing else touched."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_streaming_b200 import WF_ERR_PAGE_OOB, WF_OK, check_status
from block_causal_streaming_b200.layer import PagedPool, WavefrontLayer
from block_causal_streaming_b200.workloads import TINY, make_inputs, small_case

pytestmark = pytest.mark.gpu

SENTINEL = -12345.0   # exact in bf16 (0xC641)


def as_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("wl", [
    TINY,
    small_case("append_ps48_shared_pages", 3, 128, (37, 11), (100, 5, 64), 48, seed=31,
               pool_pages=40),
    small_case("append_ps256", 2, 64, (300,), (513,), 256, seed=32, pool_pages=9),
], ids=lambda w: w.name)
def test_append_is_bit_exact_and_touches_nothing_else(wl):
    inp = make_inputs(wl)
    pool = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, "cuda", fill=SENTINEL)
    pt = inp.page_table.cuda().reshape(1, -1)
    layer = WavefrontLayer(pool, pt, 0, wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks)
    k, v = inp.k.cuda(), inp.v.cuda()
    # append in a scrambled chunk order: the result must not depend on it
    order = list(range(wl.num_chunks))[::-1]
    layer.append_range(k, v, order)
    assert check_status() == WF_OK
    for name, src, dev in (("k", inp.k, pool.k), ("v", inp.v, pool.v)):
        expect = np.full(tuple(pool.k.shape), 0, dtype=np.int16)
        expect[...] = as_bits(torch.full((1,), SENTINEL, dtype=torch.bfloat16))[0]
        off = wl.chunk_offsets
        src_bits = as_bits(src)
        for c in order:
            oracle.scatter_chunk(expect, inp.page_table.numpy(), off[c], src_bits[off[c]:off[c + 1]])
        assert np.array_equal(as_bits(dev), expect), f"{name} pool differs from the oracle layout"


def test_append_into_shared_pool_with_two_layers():
    """Two layers, disjoint page-table rows into one pool: each layer's rows land in its pages."""
    wl = small_case("two_layers", 2, 128, (64,), (100, 27), 64, seed=33, pool_pages=12)
    inp = make_inputs(wl)
    pool = PagedPool(12, 64, 2, 128, "cuda", fill=SENTINEL)
    pt = torch.tensor([[3, 7, 1], [0, 11, 5]], dtype=torch.int32, device="cuda")
    expect = np.full(tuple(pool.k.shape), as_bits(torch.full((1,), SENTINEL,
                                                             dtype=torch.bfloat16))[0], np.int16)
    kb = as_bits(inp.k)
    for layer_idx in (0, 1):
        layer = WavefrontLayer(pool, pt, layer_idx, wl.chunk_offsets, wl.chunk_stage,
                               wl.num_ctx_chunks)
        k = (inp.k.float() + layer_idx).to(torch.bfloat16)
        layer.append_range(k.cuda(), inp.v.cuda(), range(wl.num_chunks))
        oracle.scatter_chunk(expect, pt[layer_idx].cpu().numpy(), 0, as_bits(k))
    assert check_status() == WF_OK
    assert np.array_equal(as_bits(pool.k), expect)
    del kb


def test_out_of_range_page_is_reported_not_written():
    wl = small_case("oob", 1, 64, (), (40,), 16, seed=34)
    inp = make_inputs(wl)
    pool = PagedPool(3, 16, 1, 64, "cuda", fill=SENTINEL)
    pt = torch.tensor([[0, 3, 2]], dtype=torch.int32, device="cuda")   # 3 is outside the pool
    layer = WavefrontLayer(pool, pt, 0, wl.chunk_offsets, wl.chunk_stage, 0)
    layer.append(0, inp.k.cuda(), inp.v.cuda())
    assert check_status() == WF_ERR_PAGE_OOB
    assert check_status() == WF_OK                     # cleared by the first read
    bits = as_bits(pool.k)
    sentinel = as_bits(torch.full((1,), SENTINEL, dtype=torch.bfloat16))[0]
    assert np.all(bits[1] == sentinel)                 # page 1 is nobody's: untouched
    assert np.array_equal(bits[0], as_bits(inp.k)[0:16])
    assert np.array_equal(bits[2, :8], as_bits(inp.k)[32:40])
