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
    small_case("fp8_d128_h12_ps64", 12, 128, (70,), (130, 45), 64, seed=63),
    small_case("fp8_d64_h5_ps32", 5, 64, (33,), (64, 100), 32, seed=64),
]
SENTINEL_CODE = 0xA5


def _with_special_rows(inp):
    """Special K rows of head 0: zeros (token 5), large values (6), small ones (7), a row whose
    448 / amax overflows fp32 (8, stored as zeros) and one just above that threshold, with a
    subnormal fp32 scale (9)."""
    k = inp.k.clone()
    k[5, 0] = 0
    k[6, 0] = (k[6, 0].float() * 3000).bfloat16()
    k[7, 0] = (k[7, 0].float() * 1e-20).bfloat16()
    row = k[8, 0].float()
    k[8, 0] = (row / row.abs().max() * 1e-37).bfloat16()
    row = k[9, 0].float()
    k[9, 0] = (row / row.abs().max() * 3e-36).bfloat16()
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


# ------------------------------------------------------------------------- FP8 publication
# The "peers" are further FP8 pools on the same device: the kernel writes them through plain
# device pointers, exactly as it writes another GPU's pools mapped by IPC.
LAYER, GEN = 1, 11


class PublishedFp8:
    def __init__(self, wl, n_peers=2):
        from block_causal_streaming_b200.wave import new_flags
        from block_causal_streaming_b200 import WavefrontDesc
        self.wl = wl
        self.inp = _with_special_rows(make_inputs(wl))
        self.pools = [_fp8_pool(wl) for _ in range(1 + n_peers)]
        self.flags = [new_flags(2, "cuda") for _ in range(1 + n_peers)]
        pt = self.inp.page_table.cuda()
        self.pt = torch.stack([torch.zeros_like(pt), pt]).contiguous()    # row LAYER is used
        self.desc = WavefrontDesc(wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks,
                                  self.pt.shape[1])
        self.peers = [(p.k_codes.data_ptr(), p.v_codes.data_ptr(), p.k_scale.data_ptr(),
                       p.v_scale.data_ptr(), f.data_ptr())
                      for p, f in zip(self.pools[1:], self.flags[1:])]
        self.k, self.v = self.inp.k.cuda(), self.inp.v.cuda()

    def publish(self, chunks, gen=GEN):
        from block_causal_streaming_b200 import kv_append_publish_fp8
        off = self.wl.chunk_offsets
        for c in chunks:
            kv_append_publish_fp8(*self.pools[0].tensors, self.flags[0], self.peers, LAYER, c,
                                  self.k[off[c]:off[c + 1]], self.v[off[c]:off[c + 1]],
                                  self.pt, self.desc, gen)

    def dequant_into(self, i, bf16_pool, chunks, gen=GEN):
        from block_causal_streaming_b200 import kv_dequant_published
        for c in chunks:
            kv_dequant_published(*self.pools[i].tensors, bf16_pool.k, bf16_pool.v, LAYER, c,
                                 self.pt, self.desc, self.flags[i][LAYER], gen)


def test_fp8_publication_is_bit_exact_in_every_pool_and_raises_every_flag():
    wl = CASES[0]
    P = PublishedFp8(wl, n_peers=2)
    P.publish(reversed(range(wl.num_chunks)))
    assert check_status() == WF_OK
    want = _expected(wl, P.inp)
    for i, pool in enumerate(P.pools):
        for name, codes, scale in (("k", pool.k_codes, pool.k_scale),
                                   ("v", pool.v_codes, pool.v_scale)):
            w_codes, w_scale, _, _ = want[name]
            assert np.array_equal(codes.cpu().numpy(), w_codes), f"pool {i} {name} codes"
            assert np.array_equal(scale.cpu().numpy().view(np.int32), w_scale.view(np.int32)), \
                f"pool {i} {name} scales"
    for f in P.flags:
        expect = torch.zeros_like(f)
        expect[LAYER, :wl.num_chunks] = GEN
        assert torch.equal(f, expect)


@pytest.mark.parametrize("wl", [CASES[0], CASES[3]], ids=lambda w: w.name)
def test_published_fp8_chunks_convert_and_attend(wl):
    """Each consumer converts the published codes back (after the flag) into its own bf16 pool;
    the rows are the oracle's bit for bit and attention meets the parity bar."""
    from block_causal_streaming_b200.layer import PagedPool, WavefrontLayer
    P = PublishedFp8(wl, n_peers=1)
    P.publish(range(wl.num_chunks))
    bf = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, "cuda", fill=float("nan"))
    P.dequant_into(1, bf, range(wl.num_chunks))
    assert check_status() == WF_OK
    want = _expected(wl, P.inp)
    deq = {n: ofp8.dequantize_rows(want[n][2], want[n][3]) for n in ("k", "v")}
    pt = P.inp.page_table.numpy()
    for name, pool in (("k", bf.k), ("v", bf.v)):
        got = oracle.gather_logical(pool.cpu().view(torch.int16).numpy(), pt, wl.t_kv)
        assert np.array_equal(got, deq[name].view(torch.int16).numpy()), f"{name} dequantized"
    layer = WavefrontLayer(bf, P.pt, LAYER, wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks)
    out = run(layer, P.inp.q.cuda())
    ref = oracle.attention(P.inp.q, deq["k"], deq["v"], wl.chunk_offsets, wl.num_ctx_chunks,
                           scale_of(wl))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)


def test_converting_a_chunk_never_published_times_out_and_writes_nothing():
    from block_causal_streaming_b200 import WF_ERR_TIMEOUT
    from block_causal_streaming_b200.layer import PagedPool
    import time
    wl = CASES[1]
    P = PublishedFp8(wl, n_peers=1)
    last = wl.num_chunks - 1
    P.publish(range(last))                          # the last chunk is never published
    bf = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, "cuda", fill=float("nan"))
    t = time.perf_counter()
    P.dequant_into(1, bf, [last])
    assert check_status() == WF_ERR_TIMEOUT
    assert time.perf_counter() - t < 10.0
    assert check_status() == WF_OK
    assert torch.isnan(bf.k.float()).all() and torch.isnan(bf.v.float()).all()
    P.publish([last])                               # published late: the conversion now runs
    P.dequant_into(1, bf, [last])
    assert check_status() == WF_OK
    off = wl.chunk_offsets
    got = oracle.gather_logical(bf.k.cpu().view(torch.int16).numpy(), P.inp.page_table.numpy(),
                                wl.t_kv)[off[last]:off[last + 1]]
    want = _expected(wl, P.inp)["k"]
    deq = ofp8.dequantize_rows(want[2], want[3])[off[last]:off[last + 1]]
    assert np.array_equal(got, deq.view(torch.int16).numpy())


def test_an_fp8_chunk_with_a_page_outside_the_pool_is_not_published():
    wl = CASES[0]
    P = PublishedFp8(wl, n_peers=1)
    off, ps = wl.chunk_offsets, wl.page_size
    c = wl.num_chunks - 1
    P.pt[LAYER, (off[c] + 1) // ps] = wl.num_pages + 2
    P.publish([c])
    assert check_status() == WF_ERR_PAGE_OOB
    assert check_status() == WF_OK
    for f in P.flags:
        assert int(f[LAYER, c]) == 0


@pytest.mark.parametrize("wl", CASES[:2], ids=lambda w: w.name)
def test_chunk_range_forms_equal_the_oracle_and_touch_only_their_rows(wl):
    """wf_kv_append_fp8_chunks over chunks [1, num_chunks) in one launch: codes and scales of those
    chunks bit-exact, chunk 0's rows keep the sentinel; wf_kv_dequant_chunks of the same range
    then writes exactly the oracle's bf16 rows of those chunks and leaves chunk 0's rows alone."""
    from block_causal_streaming_b200 import kv_append_fp8_chunks, kv_dequant_chunks
    inp = _with_special_rows(make_inputs(wl))
    layer, _, k, v = place(wl, inp, append=False, fill=float("nan"))
    fp = _fp8_pool(wl)
    off, c0, c1 = wl.chunk_offsets, 1, wl.num_chunks
    kv_append_fp8_chunks(*fp.tensors, 0, c0, c1, k[off[c0]:off[c1]], v[off[c0]:off[c1]],
                         layer.page_tables, layer.desc)
    assert check_status() == WF_OK
    want = _expected(wl, inp)
    pt = inp.page_table.numpy()
    H, D, ps = wl.heads, wl.head_dim, wl.page_size
    for name, codes, scale in (("k", fp.k_codes, fp.k_scale), ("v", fp.v_codes, fp.v_scale)):
        _, _, q_codes, q_scale = want[name]
        w_codes = np.full((wl.num_pages, ps, H, D), SENTINEL_CODE, np.uint8)
        w_scale = np.full((wl.num_pages, ps, H), np.nan, np.float32)
        oracle.scatter_chunk(w_codes, pt, off[c0], q_codes[off[c0]:off[c1]])
        oracle.scatter_chunk(w_scale, pt, off[c0], q_scale[off[c0]:off[c1]])
        assert np.array_equal(codes.cpu().numpy(), w_codes), f"{name} codes"
        assert np.array_equal(scale.cpu().numpy().view(np.int32), w_scale.view(np.int32)), \
            f"{name} scales"
    kv_dequant_chunks(*fp.tensors, layer.pool.k, layer.pool.v, 0, c0, c1, layer.page_tables,
                      layer.desc)
    assert check_status() == WF_OK
    for name, pool in (("k", layer.pool.k), ("v", layer.pool.v)):
        _, _, q_codes, q_scale = want[name]
        deq = ofp8.dequantize_rows(q_codes, q_scale).view(torch.int16).numpy()
        got = oracle.gather_logical(pool.cpu().view(torch.int16).numpy(), pt, wl.t_kv)
        assert np.array_equal(got[off[c0]:off[c1]], deq[off[c0]:off[c1]]), f"{name} dequantized"
        assert np.all(got[:off[c0]] == np.int16(0x7FC0)), f"{name}: chunk 0 rows were written"


def test_chunk_range_forms_reject_empty_and_reversed_ranges():
    from block_causal_streaming_b200 import (WF_ERR_INVALID_ARG, WfError, kv_append_fp8_chunks,
                                             kv_dequant_chunks)
    wl = CASES[0]
    inp = make_inputs(wl)
    layer, _, k, v = place(wl, inp, append=False)
    fp = _fp8_pool(wl)
    for c0, c1 in ((1, 1), (2, 1), (0, wl.num_chunks + 1)):
        with pytest.raises(WfError) as e:
            kv_append_fp8_chunks(*fp.tensors, 0, c0, c1, k[:0], v[:0], layer.page_tables,
                                 layer.desc)
        assert e.value.code == WF_ERR_INVALID_ARG
        with pytest.raises(WfError) as e:
            kv_dequant_chunks(*fp.tensors, layer.pool.k, layer.pool.v, 0, c0, c1,
                              layer.page_tables, layer.desc)
        assert e.value.code == WF_ERR_INVALID_ARG
    assert check_status() == WF_OK
