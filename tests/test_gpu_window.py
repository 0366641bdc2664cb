"""A rolling window streamed round after round through the CUDA path (wf_kv_append and
wf_attn_forward), checked against the oracle.

Every round draws fresh K/V for the store pass and for the chunks in flight; a stored chunk keeps
the K/V of its store pass.  The planner keeps the history as a ring of slots, while the oracle gets
the same chunks in chronological order (anchor, history oldest first, store, in flight), so the
check also covers the reading that the order of the context does not matter.  After the last round,
the pool must equal, bit for bit, a CPU replay of the same appends through the oracle's scatter.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_causal_streaming_b200 import WF_OK, check_status
from block_causal_streaming_b200.window import ACTIVE, STORE, RollingCache, RollingWindow
from gpu_util import assert_parity

pytestmark = pytest.mark.gpu


def _draw(layer, chunk, rnd, rows, heads, dim):
    g = torch.Generator().manual_seed(1_000_003 * layer + 1009 * chunk + rnd)
    return [torch.randn(rows, heads, dim, generator=g).bfloat16() for _ in range(3)]   # q, k, v


@pytest.mark.parametrize("copy_free", [False, True], ids=["hand_over", "copy_free_ring"])
@pytest.mark.parametrize("chunk_len,stages,history,page_size,dim", [
    (200, (1000, 600, 200), 2, 64, 128),     # slots straddle pages; ring fills, then rolls
    (72, (1000, 500), 3, 16, 64),
    (130, (1000,), 1, 32, 128),              # one stage: every round stores and evicts
])
def test_rolling_window_rounds_match_the_oracle(chunk_len, stages, history, page_size, dim,
                                                copy_free):
    """hand_over: the store chunk is appended past the ring and handed into the evicted slot after
    attention.  copy_free_ring: a ring of history + 1 slots; the store pass writes its ring slot
    once and its rows are a query segment that sees the whole ring (wf_attn_forward_segments)."""
    heads, layers = 2, 2
    win = RollingWindow(chunk_len, stages, history, page_size, copy_free=copy_free)
    rng = np.random.default_rng(11)
    pt = torch.from_numpy(rng.permutation(win.pages * layers).astype(np.int32))
    pt = pt.view(layers, win.pages)
    cache = RollingCache(win, heads, dim, layers, "cuda", page_tables=pt, fill=float("nan"))
    nan_bits = torch.full((1,), float("nan"), dtype=torch.bfloat16).view(torch.int16).item()
    replay = {name: np.full((win.pages * layers, page_size, heads, dim), nan_bits, np.int16)
              for name in ("k", "v")}
    stored = [dict() for _ in range(layers)]          # chunk -> (k, v) of its store pass
    scale = 1.0 / math.sqrt(dim)
    L = chunk_len
    rounds = len(stages) + history + 6
    for t in range(rounds):
        view = win.view(t)
        for layer in range(layers):
            qslots = view.query_rows_slots
            qs, ks, vs = zip(*(_draw(layer, view.chunk_ids[s], t, L, heads, dim)
                               for s in qslots))
            q, k, v = torch.cat(qs), torch.cat(ks), torch.cat(vs)
            out = torch.empty_like(q, device="cuda")
            cache.run_layer(view, layer, q.cuda(), k.cuda(), v.cuda(), out, scale=scale)
            assert check_status() == WF_OK

            # oracle: the same chunks in chronological order
            ctx = sorted(c for c, r in zip(view.chunk_ids, view.roles)
                         if r not in (STORE, ACTIVE))
            k_all = torch.cat([stored[layer][c][0] for c in ctx] + [k]) if ctx else k
            v_all = torch.cat([stored[layer][c][1] for c in ctx] + [v]) if ctx else v
            offsets = [i * L for i in range(view.num_chunks + 1)]
            ref = oracle.attention(q, k_all, v_all, offsets, len(ctx), scale)
            assert_parity(out.float().cpu().numpy(), ref, f"round {t} layer {layer}")

            # the replay of the same appends, and the hand-over of the store chunk
            row = pt[layer].numpy()
            for name, src in (("k", k), ("v", v)):
                bits = src.view(torch.int16).numpy()
                for i, s in enumerate(qslots):
                    oracle.scatter_chunk(replay[name], row, view.chunk_offsets[s],
                                         bits[i * L:(i + 1) * L])
                if view.store_to is not None:
                    oracle.scatter_chunk(replay[name], row, view.chunk_offsets[view.store_to],
                                         bits[:L])
            if STORE in view.roles:
                c = view.chunk_ids[view.roles.index(STORE)]
                stored[layer][c] = (k[:L], v[:L])
                if view.evicted is not None:
                    del stored[layer][view.evicted]
    torch.cuda.synchronize()
    # rows never written keep the NaN fill on both sides; every row is compared bit for bit
    for name, pool in (("k", cache.pool.k), ("v", cache.pool.v)):
        assert np.array_equal(pool.cpu().view(torch.int16).numpy(), replay[name]), name


def test_segments_that_restate_the_wavefront_give_the_same_bits():
    """Query segments equal to the descriptor's query chunks (rows of chunk i see the prefix up to
    its own end) reproduce wf_attn_forward bit for bit, with and without key splits."""
    from block_causal_streaming_b200 import Segments, attn_forward_segments, \
        attn_segments_workspace_size
    from block_causal_streaming_b200.workloads import make_inputs, small_case
    from gpu_util import place, run
    wl = small_case("segments", 2, 128, (300, 200), (257, 300, 129), 64, seed=91)
    inp = make_inputs(wl)
    layer, q, _, _ = place(wl, inp, fill=float("nan"))
    ref = run(layer, q)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    seg = Segments([off[c + 1] - off[nctx] for c in range(nctx, wl.num_chunks)],
                   [off[c + 1] for c in range(nctx, wl.num_chunks)], off[-1],
                   layer.page_tables.shape[1])
    for splits in (1, 3):
        out = torch.empty_like(q)
        need = attn_segments_workspace_size(seg, wl.heads, wl.head_dim, splits)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
        attn_forward_segments(q, layer.pool.k, layer.pool.v, layer.page_tables[0], seg,
                              1.0 / math.sqrt(wl.head_dim), out, None, splits, ws)
        assert check_status() == WF_OK
        if splits == 1:
            assert torch.equal(out, ref)
        else:
            ref32 = ref.float()
            assert (out.float() - ref32).abs().max().item() <= 1e-2
