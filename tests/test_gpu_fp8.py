"""FP8 (e4m3) K/V pages on the GPU: wf_kv_append_fp8 and wf_kv_dequant against the oracle.

The codes and the scales written by the quantizing append must equal the oracle's bit for bit,
through a permuted page table with chunks that straddle pages; rows the chunks do not own keep
their sentinel.  Dequantization must reproduce the oracle's bf16 rows bit for bit, and attention
over the dequantized pages must meet the parity bar against the oracle run on the oracle's own
dequantized K/V.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as ofp8
from block_causal_streaming_b200 import (WF_ERR_PAGE_OOB, WF_OK, check_status, kv_append_fp8,
                                         kv_dequant)
from block_causal_streaming_b200.layer import PagedPoolFp8
from block_causal_streaming_b200.workloads import make_inputs, small_case
from gpu_util import assert_parity, place, run, scale_of

pytestmark = pytest.mark.gpu

CASES = [
    small_case("fp8_d128_ps64", 3, 128, (130, 64), (200, 77, 300), 64, seed=61),
    small_case("fp8_d64_ps16", 2, 64, (100,), (90, 150), 16, seed=62),
]
SENTINEL_CODE = 0xA5


def _with_special_rows(inp):
    """A row of zeros, a row of large values and a row of small ones in K (token 5, 6, 7)."""
    k = inp.k.clone()
    k[5, 0] = 0
    k[6, 0] = (k[6, 0].float() * 3000).bfloat16()
    k[7, 0] = (k[7, 0].float() * 1e-20).bfloat16()
    inp.k = k
    return inp


def _expected(wl, inp):
    """The FP8 pool the oracle writes: quantize each chunk's rows, scatter them by page table."""
    H, D, ps = wl.heads, wl.head_dim, wl.page_size
    pages = wl.num_pages
    pt = inp.page_table.numpy()
    out = {}
    for name, x in (("k", inp.k), ("v", inp.v)):
        codes = np.full((pages, ps, H, D), SENTINEL_CODE, np.uint8)
        scale = np.full((pages, ps, H), np.nan, np.float32)
        q_codes, q_scale = ofp8.quantize_rows(x.float().numpy())
        off = wl.chunk_offsets
        for c in range(wl.num_chunks):
            oracle.scatter_chunk(codes, pt, off[c], q_codes[off[c]:off[c + 1]])
            oracle.scatter_chunk(scale, pt, off[c], q_scale[off[c]:off[c + 1]])
        out[name] = (codes, scale, q_codes, q_scale)
    return out


def _fp8_pool(wl):
    pool = PagedPoolFp8(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, "cuda")
    pool.k_codes.fill_(SENTINEL_CODE)
    pool.v_codes.fill_(SENTINEL_CODE)
    pool.k_scale.fill_(float("nan"))
    pool.v_scale.fill_(float("nan"))
    return pool


def _append_all(wl, layer, fp, k, v):
    off = wl.chunk_offsets
    for c in reversed(range(wl.num_chunks)):          # any order: chunks own disjoint rows
        kv_append_fp8(*fp.tensors, 0, c, k[off[c]:off[c + 1]], v[off[c]:off[c + 1]],
                      layer.page_tables, layer.desc)


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_quantized_append_is_bit_exact(wl):
    inp = _with_special_rows(make_inputs(wl))
    layer, _, k, v = place(wl, inp, append=False)
    fp = _fp8_pool(wl)
    _append_all(wl, layer, fp, k, v)
    assert check_status() == WF_OK
    want = _expected(wl, inp)
    for name, codes, scale in (("k", fp.k_codes, fp.k_scale), ("v", fp.v_codes, fp.v_scale)):
        w_codes, w_scale, _, _ = want[name]
        assert np.array_equal(codes.cpu().numpy(), w_codes), f"{name} codes"
        assert np.array_equal(scale.cpu().numpy().view(np.int32), w_scale.view(np.int32)), \
            f"{name} scales"


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_dequantized_pages_are_bit_exact_and_attention_meets_the_bar(wl):
    inp = _with_special_rows(make_inputs(wl))
    layer, q, k, v = place(wl, inp, append=False, fill=float("nan"))
    fp = _fp8_pool(wl)
    _append_all(wl, layer, fp, k, v)
    for c in range(wl.num_chunks):
        kv_dequant(*fp.tensors, layer.pool.k, layer.pool.v, 0, c, layer.page_tables, layer.desc)
    assert check_status() == WF_OK
    want = _expected(wl, inp)
    pt = inp.page_table.numpy()
    deq = {}
    for name, pool in (("k", layer.pool.k), ("v", layer.pool.v)):
        _, _, q_codes, q_scale = want[name]
        deq[name] = ofp8.dequantize_rows(q_codes, q_scale)              # logical order, bf16
        got = oracle.gather_logical(pool.cpu().view(torch.int16).numpy(), pt, wl.t_kv)
        assert np.array_equal(got, deq[name].view(torch.int16).numpy()), f"{name} dequantized"
    out = run(layer, q)
    ref = oracle.attention(inp.q, deq["k"], deq["v"], wl.chunk_offsets, wl.num_ctx_chunks,
                           scale_of(wl))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)


def test_a_page_outside_the_fp8_pool_is_reported():
    wl = CASES[1]
    inp = make_inputs(wl)
    layer, _, k, v = place(wl, inp, append=False)
    bad = layer.page_tables.clone()
    bad[0, 1] = wl.num_pages + 3
    fp = _fp8_pool(wl)
    off = wl.chunk_offsets
    kv_append_fp8(*fp.tensors, 0, 0, k[off[0]:off[1]], v[off[0]:off[1]], bad, layer.desc)
    assert check_status() == WF_ERR_PAGE_OOB
    assert check_status() == WF_OK
