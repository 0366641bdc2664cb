"""The rolling-window planner (block_causal_streaming_b200.window) on the CPU.

* Visible sets: for every round and every query chunk, the chunks its keys come from must be those
  the pages name.  These are the anchor, the clean history, the live store and every earlier, cleaner
  chunk in flight, and never a later, noisier one (KipQuest summary of arXiv 2611.00859, "The deep
  dive").  The history is the ``history`` most recently stored chunks after the anchor.  The expected
  set is written from the stream's chronology, not from the planner's slots.
* Nothing that persists moves: a stored chunk keeps its logical token range from round to round.
* Data flow: the appends the planner prescribes, replayed round after round with the oracle's
  own paged scatter and gather, leave in every slot exactly the chunk the round's descriptor names,
  bit for bit.
"""
import ctypes

import numpy as np
import pytest

import oracle
from block_causal_streaming_b200 import build as wf_build

wf_build.build()                      # the planner is the library's wf_window_round
from block_causal_streaming_b200 import _abi  # noqa: E402
from block_causal_streaming_b200 import window as W  # noqa: E402

SHAPES = [(1, 0), (1, 2), (2, 1), (4, 2), (5, 1), (5, 3), (3, 5)]   # (stages, history)


def _stages(n):
    return [1000 - i * (800 // max(n - 1, 1)) for i in range(n)] if n > 1 else [1000]


def expected_visible(t, S, H, c, is_store):
    """Stream indices visible to chunk ``c`` at round ``t``, from the chronology alone: chunk d
    entered at round d, was in flight at rounds d..d+S-1, stored at round d+S."""
    stored = [d for d in range(0, t - S)]                  # store pass finished before round t
    history = [d for d in stored if d >= 1][-H:] if H > 0 else []
    anchor = [0] if stored else []
    if is_store:
        return set(anchor) | set(history) | {c}
    live_store = [t - S] if t - S >= 0 else []
    in_flight_cleaner = [d for d in range(max(0, t - S + 1), t + 1) if d < c]
    return set(anchor) | set(history) | set(live_store) | set(in_flight_cleaner) | {c}


@pytest.mark.parametrize("S,H", SHAPES)
def test_every_query_chunk_sees_exactly_what_the_pages_name(S, H):
    win = W.RollingWindow(48, _stages(S), H, 16)
    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        assert v.chunk_offsets == [i * 48 for i in range(v.num_chunks + 1)]
        assert all(a <= b for a, b in zip(v.chunk_stage, v.chunk_stage[1:]))
        assert v.num_chunks <= win.slots and v.chunk_offsets[-1] <= win.pages * 16
        assert len(set(v.chunk_ids)) == v.num_chunks
        for slot in v.query_slots:
            c = v.chunk_ids[slot]
            visible = set(v.chunk_ids[:slot + 1])       # the prefix rule of the descriptor
            assert visible == expected_visible(t, S, H, c, v.roles[slot] == W.STORE), (t, c)
            r = v.rank_view(slot)                        # the same set as one rank's own call
            assert set(r.chunk_ids) == visible and r.num_ctx_chunks == slot
            assert r.t_q == 48


@pytest.mark.parametrize("S,H", SHAPES)
def test_stored_chunks_never_move(S, H):
    win = W.RollingWindow(40, _stages(S), H, 16)
    prev = None
    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        if prev is not None:
            for slot in range(v.num_ctx_chunks):
                c = v.chunk_ids[slot]
                if prev.store_to is not None and c == prev.chunk_ids[prev.num_ctx_chunks]:
                    assert slot == prev.store_to           # handed over into the evicted slot
                elif c in prev.chunk_ids[:prev.num_ctx_chunks]:
                    assert slot == prev.slot_of(c)         # stayed where it was
                else:                                      # stored last round: no copy needed
                    assert prev.roles[prev.slot_of(c)] == W.STORE and prev.slot_of(c) == slot
                    assert prev.store_to is None
        if v.evicted is not None:
            assert v.store_to == v.slot_of(v.evicted)
        prev = v


@pytest.mark.parametrize("S,H,ps", [(2, 2, 16), (3, 1, 32), (1, 3, 16), (4, 0, 48)])
def test_appends_replayed_with_the_oracle_leave_the_named_chunk_in_every_slot(S, H, ps):
    """K/V content is a tag per (chunk, round, token); a stored chunk keeps its store-round tag."""
    L, heads, D = 24, 1, 2                                   # 24 tokens: slots straddle pages
    win = W.RollingWindow(L, _stages(S), H, ps)
    rng = np.random.default_rng(3)
    page_table = rng.permutation(win.pages)
    pool = np.full((win.pages, ps, heads, D), -1, np.int64)
    stored = {}                                              # chunk -> its store-round K rows

    def rows(c, t):
        base = (c * 1000 + t) * 100
        return (base + np.arange(L * heads * D)).reshape(L, heads, D)

    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        fresh = {v.chunk_ids[s]: rows(v.chunk_ids[s], t) for s in v.query_slots}
        for s in v.query_slots:                              # the round's appends
            oracle.scatter_chunk(pool, page_table, v.chunk_offsets[s], fresh[v.chunk_ids[s]])
        logical = oracle.gather_logical(pool, page_table, v.chunk_offsets[-1])
        for s, c in enumerate(v.chunk_ids):                  # what attention reads
            want = fresh[c] if s >= v.num_ctx_chunks else stored[c]
            got = logical[v.chunk_offsets[s]:v.chunk_offsets[s + 1]]
            assert np.array_equal(got, want), (t, s, c)
        if STORE_SLOT(v) is not None:
            c = v.chunk_ids[STORE_SLOT(v)]
            stored[c] = fresh[c]
            if v.store_to is not None:                       # hand-over after attention
                oracle.scatter_chunk(pool, page_table, v.chunk_offsets[v.store_to], fresh[c])
                del stored[v.evicted]


def STORE_SLOT(v):
    return v.roles.index(W.STORE) if W.STORE in v.roles else None


def test_pipeline_fill_and_steady_state_counts():
    """4-step layout with two history chunks: the critical consumer (the noisiest chunk) sees
    8 chunks in steady state, the cleanest chunk in flight 5 and the store pass 4 (project page,
    "02 Interactive pipeline", "Inside one diffusion tick": r0 sees 8 chunks, r1-store about 5)."""
    win = W.RollingWindow(4680, [1000, 750, 500, 250], 2, 64)
    v = win.view(20)
    assert v.roles == [W.ANCHOR, W.HISTORY, W.HISTORY, W.STORE] + [W.ACTIVE] * 4
    assert [v.rank_view(s).num_chunks for s in v.query_slots] == [4, 5, 6, 7, 8]
    assert v.chunk_stage == [0, 0, 0, 0, 250, 500, 750, 1000]
    assert win.view(0).roles == [W.ACTIVE] and win.view(0).chunk_stage == [1000]
    assert win.view(4).roles == [W.STORE] + [W.ACTIVE] * 4            # the anchor's store pass
    assert win.slots == 8 and win.pages == 585


def test_planner_argument_checks():
    with pytest.raises(ValueError):
        W.RollingWindow(48, [200, 1000], 1, 16)            # stages must decrease
    with pytest.raises(ValueError):
        W.RollingWindow(48, [1000], 63, 16)                # 65 slots > 64 chunks
    with pytest.raises(ValueError):
        W.RollingWindow(0, [1000], 1, 16)
    v = W.RollingWindow(48, [1000, 500], 1, 16).view(5)
    with pytest.raises(ValueError):
        v.rank_view(0)                                     # the anchor carries no queries


def test_max_chunks_matches_the_library():
    assert W.MAX_CHUNKS == _abi.WF_MAX_CHUNKS


def _plan_written_out(chunk_len, stages, history, t):
    """A second, independent statement of the layout (sorting kept chunks by ring slot), used to
    cross-check the native planner's slot assignment."""
    S, H = len(stages), history
    ring = lambda c: 0 if c == 0 else 1 + (c - 1) % H                       # noqa: E731
    ids, roles, stage = [], [], []
    last_stored = t - S - 1
    if last_stored >= 0:
        kept = list(range(max(1, last_stored - H + 1), last_stored + 1)) if H else []
        ids += [0] + sorted(kept, key=ring)
        roles += [W.ANCHOR] + [W.HISTORY] * len(kept)
        stage += [0] * (1 + len(kept))
    n_ctx, store_to, evicted = len(ids), None, None
    if t - S >= 0:
        ids.append(t - S)
        roles.append(W.STORE)
        stage.append(0)
        if H and t - S - H >= 1:
            evicted, store_to = t - S - H, ring(t - S)
    for c in range(max(0, t - S + 1), t + 1):
        ids.append(c)
        roles.append(W.ACTIVE)
        stage.append(stages[t - c])
    return ids, roles, stage, n_ctx, store_to, evicted


@pytest.mark.parametrize("S,H", SHAPES + [(2, 7), (6, 4), (1, 1), (3, 2), (2, 3)])
def test_native_planner_matches_the_written_out_layout(S, H):
    win = W.RollingWindow(33, _stages(S), H, 16)
    for t in range(0, 4 * (S + H) + 9):
        v = win.view(t)
        ids, roles, stage, n_ctx, store_to, evicted = _plan_written_out(33, _stages(S), H, t)
        assert (v.chunk_ids, v.roles, v.chunk_stage, v.num_ctx_chunks, v.store_to, v.evicted) == \
            (ids, roles, stage, n_ctx, store_to, evicted), t


def test_native_planner_argument_checks():
    w = _abi.Window(48, [1000, 500], 2)
    out = _abi.RoundC()
    assert _abi.lib.wf_window_round(None, 0, ctypes.byref(out)) == _abi.WF_ERR_INVALID_ARG
    assert _abi.lib.wf_window_round(ctypes.byref(w.c), 0, None) == _abi.WF_ERR_INVALID_ARG
    assert _abi.lib.wf_window_round(ctypes.byref(w.c), -1, ctypes.byref(out)) == \
        _abi.WF_ERR_INVALID_ARG
    assert _abi.window_slots(w) == (5 + 1, 6 * 48)
    for bad in (_abi.Window(48, [500, 1000], 2), _abi.Window(48, [1000, 0], 2),
                _abi.Window(0, [1000], 2), _abi.Window(48, [1000], -1),
                _abi.Window(48, [1000], 62), _abi.Window(2 ** 26, [1000], 62 - 30)):
        with pytest.raises(_abi.WfError) as e:
            _abi.window_slots(bad)
        assert e.value.code == _abi.WF_ERR_SHAPE
    assert _abi.window_slots(_abi.Window(48, [1000], 61)) == (64, 64 * 48)
    big = _abi.window_round(w, 10 ** 12)                 # far into a stream: 64-bit chunk ids
    assert big.chunk_id[big.num_chunks - 1] == 10 ** 12


# ----------------------------------------------------------------- copy-free ring (history + 1)
def _segment_visible(v, slot):
    """Chunks whose keys the query chunk in `slot` reads in the round's segment call."""
    rows_end, kv_end = v.segments()
    i = v.query_rows_slots.index(slot)
    n = kv_end[i]
    return {v.chunk_ids[s] for s in range(v.num_chunks) if v.chunk_offsets[s + 1] <= n}


@pytest.mark.parametrize("S,H", SHAPES)
def test_ring_every_query_chunk_sees_exactly_what_the_pages_name(S, H):
    win = W.RollingWindow(48, _stages(S), H, 16, copy_free=True)
    assert (win.slots, win.tokens) == W.RollingWindow(48, _stages(S), H, 16).slots_and_tokens()
    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        assert v.store_to is None                          # nothing is handed over
        assert v.chunk_offsets == [i * 48 for i in range(v.num_chunks + 1)]
        assert v.num_chunks <= win.slots and len(set(v.chunk_ids)) == v.num_chunks
        rows_end, kv_end = v.segments()
        assert rows_end == [48 * (i + 1) for i in range(len(rows_end))]
        assert all(a <= b for a, b in zip(kv_end, kv_end[1:]))   # one segment call per round
        for slot in v.query_rows_slots:
            c = v.chunk_ids[slot]
            assert _segment_visible(v, slot) == \
                expected_visible(t, S, H, c, v.roles[slot] == W.STORE), (t, c)


@pytest.mark.parametrize("S,H", SHAPES)
def test_ring_chunks_are_written_once_and_never_move(S, H):
    """A stored chunk is written once, by its store pass, straight into the slot it keeps: no
    round's append ever lands in a slot that holds the anchor or a history chunk."""
    win = W.RollingWindow(40, _stages(S), H, 16, copy_free=True)
    home = {}                                              # stored chunk -> its slot
    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        for slot, (c, role) in enumerate(zip(v.chunk_ids, v.roles)):
            if role in (W.ANCHOR, W.HISTORY):
                assert home[c] == slot, (t, c)             # where its store pass wrote it
            if role == W.STORE:
                assert c not in home
                written = {s for s in v.query_rows_slots}
                held = {home[d] for d in v.chunk_ids if d in home}
                assert slot not in held                    # it overwrites no live history
                home[c] = slot
                assert not (written - {slot}) & held       # nor does any other append
        if v.evicted is not None:
            assert v.evicted not in v.chunk_ids


@pytest.mark.parametrize("S,H,ps", [(2, 2, 16), (3, 1, 32), (1, 3, 16), (4, 0, 48)])
def test_ring_appends_replayed_with_the_oracle_leave_the_named_chunk_in_every_slot(S, H, ps):
    """Copy-free: the round's appends (store pass into its ring slot, chunks in flight after the
    ring), replayed with the oracle's scatter and gather, leave every slot holding the chunk the
    round names -- stored chunks their store-round rows, with no hand-over."""
    L, heads, D = 24, 1, 2
    win = W.RollingWindow(L, _stages(S), H, ps, copy_free=True)
    rng = np.random.default_rng(4)
    page_table = rng.permutation(win.pages)
    pool = np.full((win.pages, ps, heads, D), -1, np.int64)
    stored = {}

    def rows(c, t):
        base = (c * 1000 + t) * 100
        return (base + np.arange(L * heads * D)).reshape(L, heads, D)

    for t in range(0, 3 * (S + H) + 6):
        v = win.view(t)
        fresh = {v.chunk_ids[s]: rows(v.chunk_ids[s], t) for s in v.query_rows_slots}
        for s in v.query_rows_slots:
            oracle.scatter_chunk(pool, page_table, v.chunk_offsets[s], fresh[v.chunk_ids[s]])
        logical = oracle.gather_logical(pool, page_table, v.chunk_offsets[-1])
        for s, c in enumerate(v.chunk_ids):
            want = fresh[c] if s in v.query_rows_slots else stored[c]
            assert np.array_equal(logical[v.chunk_offsets[s]:v.chunk_offsets[s + 1]], want), \
                (t, s, c)
        if STORE_SLOT(v) is not None:
            c = v.chunk_ids[STORE_SLOT(v)]
            stored[c] = fresh[c]
