"""wf_attn_forward on the GPU against the oracle.

Parity bar: max-abs <= 1e-2 and mean-abs <= 1e-3 on bf16 outputs
with fp32 accumulation.  Small cases are compared element by element on every output; the five
benchmark workloads are compared on sampled rows (chunk edges, tile edges, the tail) plus
properties that hold at any size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_causal_streaming_b200 import WF_ERR_PAGE_OOB, WF_OK, check_status
from block_causal_streaming_b200.workloads import (TINY, WAN13B_4STEP, WAN13B_5STEP,
                                                   WAN13B_ROUND30, WAN14B, LayerInputs,
                                                   make_inputs, make_layers,
                                                   small_case)
from gpu_util import assert_parity, place, run, sample_rows, scale_of, whole_units

pytestmark = pytest.mark.gpu

SMALL = [
    small_case("d128_ps64_ctx2_act3", 2, 128, (300, 200), (257, 300, 129), 64, seed=11),
    small_case("d64_ps16_noctx", 3, 64, (), (48, 48, 48, 100), 16, seed=12),
    small_case("d128_ps48_short_chunks", 1, 128, (37,), (5, 1, 130, 70), 48, seed=13),
    small_case("d128_ps256_single_chunk", 2, 128, (), (700,), 256, seed=14),
    small_case("d128_ps128_tq_below_tile", 2, 128, (500,), (20,), 128, seed=15),
    small_case("d64_ps32_many_chunks", 2, 64, (64, 64, 64), (33, 95, 128, 256, 1), 32, seed=16),
    small_case("d128_kmean", 2, 128, (400, 400), (300, 300), 64, seed=17, k_mean_offset=True),
    small_case("d128_empty_active_chunk", 2, 128, (90,), (100, 0, 50), 16, seed=18),
    small_case("d64_ps128_pool_larger", 4, 64, (130,), (250, 260), 128, seed=19, pool_pages=20),
]


def full_oracle(wl, inp, with_lse=True):
    return oracle.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks,
                            scale_of(wl), with_lse=with_lse)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_parity_every_element(wl):
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"), extra_pages=2)
    out, lse = run(layer, q, with_lse=True)
    assert check_status() == WF_OK
    ref, ref_lse = full_oracle(wl, inp)
    assert_parity(out.float().cpu().numpy(), ref, wl.name)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)


def test_tiny_wavefront_every_element():
    wl = TINY
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    out = run(layer, q)
    assert check_status() == WF_OK
    assert_parity(out.float().cpu().numpy(), full_oracle(wl, inp, with_lse=False), wl.name)


@pytest.mark.parametrize("wl", [WAN13B_5STEP, WAN13B_4STEP, WAN14B], ids=lambda w: w.name)
def test_full_size_wavefront_parity_on_whole_units(wl):
    """Full-size wavefronts: every head of every row of whole 256-row units (two per query chunk
    at least, the units that straddle chunk boundaries, and the longest unit) element by
    element, plus sampled rows at chunk and tile edges; lse on all of them; two runs bitwise
    equal."""
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    out, lse = run(layer, q, with_lse=True)
    out2 = run(layer, q)
    assert check_status() == WF_OK
    assert torch.equal(out, out2), "two identical runs differ"
    assert torch.isfinite(out.float()).all()
    # 40 heads: the boundary units alone (still two per query chunk) keep the oracle to minutes
    u_rows, u_heads, units = whole_units(wl, seed=wl.seed, interior=wl.heads <= 12)
    s_rows, s_heads = sample_rows(wl, per_chunk=4, seed=wl.seed)
    rows = np.concatenate([u_rows, np.asarray(s_rows, np.int32)])
    heads = np.concatenate([u_heads, np.asarray(s_heads, np.int32)])
    ref, ref_lse = oracle.attention_rows(inp.q, inp.k, inp.v, wl.chunk_offsets,
                                         wl.num_ctx_chunks, scale_of(wl), rows, heads,
                                         with_lse=True)
    got = out[rows, heads].float().cpu().numpy()
    mx, mean = assert_parity(got, ref, wl.name)
    np.testing.assert_allclose(lse[heads, rows].cpu().numpy(), ref_lse, rtol=0, atol=2e-3)
    print(f"{wl.name}: {len(units)} whole units {units} x {wl.heads} heads + "
          f"{len(s_rows)} sampled rows = {len(rows)} (row, head) pairs, "
          f"{got.size} outputs: max-abs {mx:.3e}, mean-abs {mean:.3e}")


def test_thirty_layer_round_parity():
    """30 layers share one 4096-page pool; each layer appends its chunks, then attends.  Three
    layers (first, middle, last) are compared on whole units over every head, the others on
    sampled rows."""
    wl = WAN13B_ROUND30
    layers = make_layers(wl)
    from block_causal_streaming_b200.layer import PagedPool, WavefrontLayer
    pool = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, "cuda")
    pts = torch.stack([l.page_table for l in layers]).cuda()
    outs = []
    for i, inp in enumerate(layers):
        layer = WavefrontLayer(pool, pts, i, wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks)
        layer.append_range(inp.k.cuda(), inp.v.cuda(), range(wl.num_chunks))
        outs.append(run(layer, inp.q.cuda()).cpu())
    assert check_status() == WF_OK
    full = {0, len(layers) // 2, len(layers) - 1}
    for i, inp in enumerate(layers):
        if i in full:
            rows, heads, units = whole_units(wl, seed=100 + i)
        else:
            rows, heads = sample_rows(wl, per_chunk=1, seed=100 + i)
        ref = oracle.attention_rows(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks,
                                    scale_of(wl), rows, heads)
        mx, mean = assert_parity(outs[i][rows, heads].float().numpy(), ref, f"layer {i}")
        if i in full:
            print(f"layer {i}: {len(units)} whole units x {wl.heads} heads = {len(rows)} pairs: "
                  f"max-abs {mx:.3e}, mean-abs {mean:.3e}")


# ------------------------------------------------------------------------------- invariants
MED = small_case("invariants", 2, 128, (300,), (200, 300, 250), 64, seed=21)


def test_later_chunks_are_invisible_bitwise():
    wl = MED
    inp = make_inputs(wl)
    layer, q, k, v = place(wl, inp)
    base = run(layer, q)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    for i in range(nctx, wl.num_chunks - 1):
        k2, v2 = k.clone(), v.clone()
        k2[off[i + 1]:] = torch.randn_like(k2[off[i + 1]:].float()).to(torch.bfloat16) * 5
        v2[off[i + 1]:] = torch.randn_like(v2[off[i + 1]:].float()).to(torch.bfloat16) * 5
        layer.append_range(k2, v2, range(i + 1, wl.num_chunks))
        got = run(layer, q)
        rows = off[i + 1] - off[nctx]
        assert torch.equal(got[:rows], base[:rows]), f"chunk <= {i} changed"
        assert not torch.equal(got[rows:], base[rows:])
        layer.append_range(k, v, range(i + 1, wl.num_chunks))   # restore
    assert check_status() == WF_OK


def test_values_of_later_chunks_never_leak():
    wl = MED
    inp = make_inputs(wl)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    for j in range(nctx + 1, wl.num_chunks):
        v = torch.zeros_like(inp.v)
        v[off[j]:off[j + 1]] = inp.v[off[j]:off[j + 1]]
        layer, q, _, _ = place(wl, LayerInputs(inp.q, inp.k, v, inp.page_table))
        out = run(layer, q)
        before = off[j] - off[nctx]
        assert torch.all(out[:before] == 0), f"chunk {j}'s values leaked into earlier chunks"
        assert torch.any(out[before:off[j + 1] - off[nctx]] != 0)
    assert check_status() == WF_OK


def test_zero_queries_give_prefix_mean():
    wl = MED
    inp = make_inputs(wl)
    inp = LayerInputs(torch.zeros_like(inp.q), inp.k, inp.v, inp.page_table)
    layer, q, _, _ = place(wl, inp)
    out, lse = run(layer, q, with_lse=True)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    csum = torch.cat([torch.zeros(1, wl.heads, wl.head_dim, dtype=torch.float64),
                      inp.v.double().cumsum(0)])
    for c in range(nctx, wl.num_chunks):
        n = off[c + 1]
        rows = slice(off[c] - off[nctx], off[c + 1] - off[nctx])
        mean = (csum[n] / n).float()
        err = (out[rows].float().cpu() - mean).abs().max().item()
        assert err <= 1e-2, f"chunk {c}: prefix-mean error {err}"
        assert (lse[:, rows].cpu() - math.log(n)).abs().max().item() <= 1e-3


def test_unit_values_give_unit_outputs():
    """V = 1: every softmax row used by P.V must sum to 1, so every output is 1 within 1e-3.

    The kernel divides O = sum_j bf16(p_j) by the sum of the same bf16-rounded weights, so the
    result is 1 up to fp32 summation error (about 1e-6), which rounds to exactly 1.0 in bf16.
    (Dividing by the fp32 sum of the unrounded p_j instead would leave the bf16 rounding of the
    weights, up to 2^-8 relative, in the output: with a stale reference maximum a single
    dominant weight is itself rounded, and rows with one dominant key then come out at
    1 - 2^-8.)  The logits here have standard deviation ~4, so such rows occur.  A missed key
    or a tile counted twice would move the output by far more than 1e-3."""
    wl = small_case("unit_v", 3, 128, (1000,), (600, 700), 64, seed=22, value_scale=2.0)
    inp = make_inputs(wl)
    inp = LayerInputs(inp.q, inp.k, torch.ones_like(inp.v), inp.page_table)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    out = run(layer, q)
    dev = (out.float() - 1).abs().max().item()
    print(f"V = 1: max |out - 1| = {dev:.3e} over {out.numel()} outputs")
    assert dev <= 1e-3


def test_page_permutation_is_invisible_bitwise():
    wl = MED
    inp = make_inputs(wl)
    ident = LayerInputs(inp.q, inp.k, inp.v, torch.arange(wl.pages_needed, dtype=torch.int32))
    perm = LayerInputs(inp.q, inp.k, inp.v,
                       torch.randperm(wl.pages_needed + 9,
                                      generator=torch.Generator().manual_seed(3))[
                           :wl.pages_needed].to(torch.int32))
    layer_a, q, _, _ = place(wl, ident)
    layer_b, _, _, _ = place(wl, perm, extra_pages=9, fill=float("nan"))
    assert torch.equal(run(layer_a, q), run(layer_b, q))


def test_out_of_range_page_in_attention_is_reported():
    wl = small_case("oob_attn", 1, 128, (64,), (64,), 64, seed=23)
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    layer.page_tables[0, 1] = 99                     # outside the 2-page pool
    run(layer, q)
    assert check_status() == WF_ERR_PAGE_OOB
    assert check_status() == WF_OK


def test_bounded_wait_runs_out_and_context_survives():
    """A kernel wait that nothing completes gives up after its limit, reports WF_ERR_TIMEOUT,
    and the device keeps working: the next attention call is still correct."""
    from block_causal_streaming_b200 import WF_ERR_TIMEOUT, selftest_timeout
    import time
    t0 = time.perf_counter()
    selftest_timeout(20000)                     # 20 ms
    assert check_status() == WF_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert check_status() == WF_OK
    wl = TINY
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp)
    out = run(layer, q)
    assert check_status() == WF_OK
    assert_parity(out.float().cpu().numpy(), full_oracle(wl, inp, with_lse=False), "after timeout")


def test_sixty_four_chunks_the_descriptor_maximum():
    """WF_MAX_CHUNKS chunks: 4 context + 60 query chunks of 1..40 tokens, every element."""
    import random
    rnd = random.Random(64)
    ctx = tuple(rnd.randint(5, 30) for _ in range(4))
    act = tuple(rnd.randint(1, 40) for _ in range(60))
    wl = small_case("sixty_four_chunks", 2, 128, ctx, act, 16, seed=64)
    assert wl.num_chunks == 64
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    out, lse = run(layer, q, with_lse=True)
    assert check_status() == WF_OK
    ref, ref_lse = full_oracle(wl, inp)
    assert_parity(out.float().cpu().numpy(), ref, wl.name)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)
