"""One-way K/V publication on one GPU: wf_kv_append_publish and wf_attn_forward_published.

The "peers" here are further pools on the same device (the kernels write them through plain
device pointers, exactly as they write a peer GPU's memory mapped by IPC).  Publication must put
the chunk bit for bit into every pool's pages and raise its flag in every flag array; attention
on a published pool must wait for the flags -- also for a flag that arrives while the kernel is
already running -- and must stop with WF_ERR_TIMEOUT, leaving the device usable, when a chunk is
never published."""
import time

import numpy as np
import pytest
import torch

import oracle
from block_causal_streaming_b200 import (WF_ERR_PAGE_OOB, WF_ERR_TIMEOUT, WF_OK,
                                         attn_forward_published,
                                         attn_workspace_size, check_status, kv_append_publish)
from block_causal_streaming_b200.layer import PagedPool
from block_causal_streaming_b200.wave import new_flags
from block_causal_streaming_b200.workloads import WP_RANK0, make_inputs, small_case
from block_causal_streaming_b200 import WavefrontDesc
from gpu_util import assert_parity, sample_rows, scale_of

pytestmark = pytest.mark.gpu

SENTINEL = -12345.0
LAYER = 1            # publish into layer 1 of a 2-layer flag array / page table
GEN = 7


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy()


class Published:
    """A source pool and `n_peers` destination pools (same device), with flag arrays."""

    def __init__(self, wl, n_peers=2):
        self.wl = wl
        self.inp = make_inputs(wl)
        H, D, ps = wl.heads, wl.head_dim, wl.page_size
        self.pools = [PagedPool(wl.num_pages, ps, H, D, "cuda", fill=SENTINEL)
                      for _ in range(1 + n_peers)]
        self.flags = [new_flags(2, "cuda") for _ in range(1 + n_peers)]
        pt = self.inp.page_table.cuda()
        self.pt = torch.stack([torch.zeros_like(pt), pt]).contiguous()   # row LAYER is used
        self.desc = WavefrontDesc(wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks,
                                  self.pt.shape[1])
        self.peers = [(p.k.data_ptr(), p.v.data_ptr(), f.data_ptr())
                      for p, f in zip(self.pools[1:], self.flags[1:])]
        self.k, self.v = self.inp.k.cuda(), self.inp.v.cuda()

    def publish(self, chunks, gen=GEN):
        off = self.wl.chunk_offsets
        for c in chunks:
            kv_append_publish(self.pools[0].k, self.pools[0].v, self.flags[0], self.peers,
                              LAYER, c, self.k[off[c]:off[c + 1]], self.v[off[c]:off[c + 1]],
                              self.pt, self.desc, gen)

    def attend(self, i, splits=0, lse=None, stream=None, gen=GEN):
        q = self.inp.q.cuda()
        out = torch.empty_like(q)
        need = attn_workspace_size(self.desc, self.wl.heads, self.wl.head_dim, splits)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
        attn_forward_published(q, self.pools[i].k, self.pools[i].v, self.pt[LAYER], self.desc,
                               scale_of(self.wl), out, self.flags[i][LAYER], gen, splits, ws,
                               lse, stream)
        return out


CASE = small_case("publish_d128", 2, 128, (130, 64), (200, 77, 300), 64, seed=51)


def test_publish_is_bit_exact_in_every_pool_and_raises_every_flag():
    P = Published(CASE, n_peers=2)
    P.publish(reversed(range(CASE.num_chunks)))
    assert check_status() == WF_OK
    off = CASE.chunk_offsets
    for name, src in (("k", P.inp.k), ("v", P.inp.v)):
        expect = np.full(tuple(P.pools[0].k.shape),
                         _bits(torch.full((1,), SENTINEL, dtype=torch.bfloat16))[0], np.int16)
        for c in range(CASE.num_chunks):
            oracle.scatter_chunk(expect, P.inp.page_table.numpy(), off[c],
                                 _bits(src)[off[c]:off[c + 1]])
        for i, pool in enumerate(P.pools):
            got = _bits(pool.k if name == "k" else pool.v)
            assert np.array_equal(got, expect), f"{name} of pool {i}"
    for f in P.flags:
        want = torch.zeros_like(f)
        want[LAYER, :CASE.num_chunks] = GEN
        assert torch.equal(f, want)


@pytest.mark.parametrize("splits", [1, 3])
def test_attention_on_a_published_pool_matches_the_oracle(splits):
    P = Published(CASE, n_peers=1)
    P.publish(range(CASE.num_chunks))
    lse = torch.empty(CASE.heads, CASE.t_q, dtype=torch.float32, device="cuda")
    out = P.attend(1, splits=splits, lse=lse)
    assert check_status() == WF_OK
    ref, ref_lse = oracle.attention(P.inp.q, P.inp.k, P.inp.v, CASE.chunk_offsets,
                                    CASE.num_ctx_chunks, scale_of(CASE), with_lse=True)
    assert_parity(out.float().cpu().numpy(), ref, f"published S={splits}")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)


def test_a_flag_that_arrives_during_the_kernel_is_waited_for():
    """The last chunk's flag is stale when the kernel starts; a copy on another stream raises
    it ~50 ms later.  The kernel must wait (not time out) and then read the published data."""
    P = Published(WP_RANK0, n_peers=1)
    P.publish(range(WP_RANK0.num_chunks))
    last = WP_RANK0.num_chunks - 1
    P.flags[1][LAYER, last] = GEN - 1                  # not yet published (older generation)
    torch.cuda.synchronize()
    raise_flag = torch.tensor([GEN], dtype=torch.int32).pin_memory()
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(main)
    out = P.attend(1, splits=0, stream=main)
    t1.record(main)
    time.sleep(0.05)
    with torch.cuda.stream(side):
        P.flags[1][LAYER, last:last + 1].copy_(raise_flag, non_blocking=True)
    assert check_status() == WF_OK
    torch.cuda.synchronize()
    assert t0.elapsed_time(t1) > 20.0, "the kernel did not wait for the flag"
    rows, heads = sample_rows(WP_RANK0, per_chunk=8, seed=7)
    ref = oracle.attention_rows(P.inp.q, P.inp.k, P.inp.v, WP_RANK0.chunk_offsets,
                                WP_RANK0.num_ctx_chunks, scale_of(WP_RANK0), rows, heads)
    assert_parity(out[rows, heads].float().cpu().numpy(), ref, "late flag")


def test_a_chunk_never_published_times_out_and_the_device_stays_usable():
    P = Published(CASE, n_peers=1)
    P.publish(range(CASE.num_chunks - 1))              # the last chunk is never published
    t = time.perf_counter()
    P.attend(1, splits=1)
    assert check_status() == WF_ERR_TIMEOUT
    assert time.perf_counter() - t < 10.0
    assert check_status() == WF_OK
    P.publish([CASE.num_chunks - 1])
    out = P.attend(1, splits=1)
    assert check_status() == WF_OK
    ref = oracle.attention(P.inp.q, P.inp.k, P.inp.v, CASE.chunk_offsets, CASE.num_ctx_chunks,
                           scale_of(CASE))
    assert_parity(out.float().cpu().numpy(), ref, "after a timeout")


def test_publication_at_head_dim_64_with_splits():
    wl = small_case("publish_d64", 3, 64, (100,), (90, 150), 16, seed=52)
    P = Published(wl, n_peers=2)
    P.publish(range(wl.num_chunks))
    ref = oracle.attention(P.inp.q, P.inp.k, P.inp.v, wl.chunk_offsets, wl.num_ctx_chunks,
                           scale_of(wl))
    for i in (1, 2):
        out = P.attend(i, splits=2)
        assert check_status() == WF_OK
        assert_parity(out.float().cpu().numpy(), ref, f"pool {i}")


def test_a_chunk_with_a_page_outside_the_pool_is_not_published():
    """A page-table entry outside the pool makes the writer skip those rows; the chunk is then
    incomplete, so its flag must stay down in every pool (a consumer would wait, not read stale
    pages), while the other chunks publish normally."""
    P = Published(CASE, n_peers=2)
    off, ps = CASE.chunk_offsets, CASE.page_size
    bad_chunk = CASE.num_chunks - 2
    P.pt[LAYER, (off[bad_chunk] + 3) // ps] = CASE.num_pages + 5
    P.publish(range(CASE.num_chunks))
    assert check_status() == WF_ERR_PAGE_OOB
    assert check_status() == WF_OK
    for f in P.flags:
        row = f[LAYER, :CASE.num_chunks].cpu().tolist()
        # a chunk that shares the bad page is incomplete too
        bad = {c for c in range(CASE.num_chunks)
               if off[c] // ps <= (off[bad_chunk] + 3) // ps <= (off[c + 1] - 1) // ps
               and off[c + 1] > off[c]}
        assert bad_chunk in bad
        assert row == [0 if c in bad else GEN for c in range(CASE.num_chunks)]
