"""Rolling context window for a streaming wavefront over one fixed paged layout.

What a round contains (KipQuest summary of arXiv 2611.00859, "The deep dive"): chunks and
denoising stages form a grid whose active cells lie on a diagonal that moves one chunk per round;
the oldest active chunk is on its last stage and the newest has just left pure noise.  A chunk that
has finished its last stage gets one more forward pass at the clean timestep, the *store* pass,
whose keys and values become the history later chunks read.  Within a chunk attention is full;
across chunks a chunk sees the anchor, the clean history, the live store and every earlier,
cleaner chunk in flight, and never a later, noisier one.  The GitHub README ("Quick start",
"Run the 4-step checkpoint") gives one store rank beside the denoising stages.  The project page
("03 End-to-end KV transport", item 03 "Layout") has every producer write into its fixed slot of
the consumer's attention buffer, with attention reading the prefix in place.

Readings taken here, where the pages say no more:

* The anchor is the first chunk ever stored.  It is kept for the whole stream.
* The clean history holds the ``history`` most recently stored chunks after the anchor.  When a
  newer one is stored, the oldest leaves.
* Every chunk has the same number of tokens, ``chunk_len``: three latent frames in the Wan
  configurations.

Layout.  One layer's K/V occupy ``slots`` consecutive chunk slots of ``chunk_len`` tokens:

    [anchor][history ring: ``history`` slots][live store][in flight, cleanest first]

One page table per layer maps them, and it never changes.  Chunk slots are not page-aligned
(4680 tokens is not a multiple of any page size the kernels take), so a slot's logical position
cannot be moved by editing page-table entries.  Nothing that persists is moved, then:

* The anchor and history chunks stay in their slots.  Every query sees all of them, and attention
  over a set of keys does not depend on their order.  So the history is a ring: a newly stored chunk
  takes the slot of the chunk it evicts.
* The store chunk and the chunks in flight get new K/V every round.  They are appended each round
  right after the last occupied history slot.
* While the ring is filling, the store chunk already sits in the slot it keeps as history: nothing
  is copied.  Once the ring is full, the store chunk sits past the ring.  After the round's
  attention at a layer, its K/V are appended a second time, into the ring slot of the chunk that
  leaves (``RoundView.store_to``).  That is one extra chunk append per layer per round.

:class:`RollingWindow` is the host-side planner: a pure function from the round number to that
round's descriptor, computed by the library's native planner (``wf_window_round``).

Copy-free form (``copy_free=True``, ``wf_window_round_ring``).  With one GPU per chunk (Wave
Parallelism), the hand-over append would overwrite a ring slot in the very round in which other
GPUs may still read the chunk that leaves it.  The copy-free form gives the ring ``history + 1``
slots instead of ``history`` plus a separate store slot:

    [anchor][ring: ``history + 1`` slots][in flight, cleanest first]

The store pass writes its chunk once, straight into the ring slot it keeps (the slot of the chunk
that left the history at the end of the previous round), and never moves again.  Its rows see the
anchor and the whole occupied ring, although their own slot is not the last one, so a round is one
attention call over query segments (``wf_attn_forward_segments``): the store pass's rows with the
ring's end as their key limit, then each chunk in flight with its own end.
:class:`RollingCache` holds the device pools and page tables.  Through the C ABI it runs one
layer of a round: appends, attention and the hand-over into the ring.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch

ANCHOR, HISTORY, STORE, ACTIVE = "anchor", "history", "store", "active"
_ROLE_NAMES = {0: ANCHOR, 1: HISTORY, 2: STORE, 3: ACTIVE}   # WF_ROLE_* of include/wf.h
MAX_CHUNKS = 64   # chunks per descriptor (WF_MAX_CHUNKS)


@dataclasses.dataclass(frozen=True)
class RoundView:
    """One round's chunks in logical order (the order of the descriptor and of the slots)."""

    round: int
    chunk_ids: List[int]        # stream index of the chunk in each slot
    roles: List[str]            # ANCHOR | HISTORY | STORE | ACTIVE per slot
    chunk_stage: List[int]      # 0 for anchor, history and store; the timestep for chunks in flight
    chunk_offsets: List[int]    # slot i holds logical tokens [i * chunk_len, (i + 1) * chunk_len)
    num_ctx_chunks: int         # anchor + history: K/V only, no queries this round
    store_to: Optional[int]     # slot that must also receive the store chunk's K/V after attention
    evicted: Optional[int]      # stream index of the history chunk leaving after this round
    store_kv_end: Optional[int] = None   # keys the store pass's rows see (None: no store pass)

    @property
    def num_chunks(self) -> int:
        return len(self.chunk_ids)

    @property
    def query_slots(self) -> List[int]:
        return list(range(self.num_ctx_chunks, self.num_chunks))

    @property
    def t_q(self) -> int:
        return self.chunk_offsets[-1] - self.chunk_offsets[self.num_ctx_chunks]

    def slot_of(self, chunk_id: int) -> int:
        return self.chunk_ids.index(chunk_id)

    @property
    def query_rows_slots(self) -> List[int]:
        """Slots whose chunks carry queries this round, in the order of the query rows: the
        store pass, then the chunks in flight (slot order in both forms)."""
        return [i for i, r in enumerate(self.roles) if r in (STORE, ACTIVE)]

    def segments(self):
        """(rows_end, kv_end) of the round's query segments: one per query chunk, in the order
        of the query rows; the store pass sees ``store_kv_end`` keys, a chunk in flight the
        slots up to its own."""
        rows_end, kv_end, rows = [], [], 0
        for i in self.query_rows_slots:
            rows += self.chunk_offsets[i + 1] - self.chunk_offsets[i]
            rows_end.append(rows)
            kv_end.append(self.store_kv_end if self.roles[i] == STORE
                          else self.chunk_offsets[i + 1])
        return rows_end, kv_end

    def rank_view(self, slot: int) -> "RoundView":
        """The call of the one rank whose query chunk is in ``slot`` (Wave Parallelism: one stage,
        or the store pass, per GPU).  Its keys are the prefix up to and including that chunk, and
        every earlier chunk is K/V only for it."""
        if not self.num_ctx_chunks <= slot < self.num_chunks:
            raise ValueError(f"slot {slot} carries no queries this round")
        n = slot + 1
        return dataclasses.replace(
            self, chunk_ids=self.chunk_ids[:n], roles=self.roles[:n],
            chunk_stage=self.chunk_stage[:n], chunk_offsets=self.chunk_offsets[:n + 1],
            num_ctx_chunks=slot, store_to=None, evicted=None)


class RollingWindow:
    """Round-by-round plan of a streaming wavefront with a rolling history (wf_window_round).

    ``stages`` are the denoising timesteps of the in-flight positions, noisiest first (e.g.
    1000, 800, 600, 400, 200).  Chunk ``c`` enters at round ``c``.  At round ``t`` it is on step
    ``t - c``, and in the store pass at round ``c + len(stages)``.  The plan comes from the
    library's native planner; this class only converts it.
    """

    def __init__(self, chunk_len: int, stages: Sequence[int], history: int, page_size: int,
                 copy_free: bool = False):
        from . import _abi
        self.copy_free = bool(copy_free)
        self.chunk_len = int(chunk_len)
        self.stages = [int(x) for x in stages]
        self.history = int(history)
        self.page_size = int(page_size)
        if not self.stages or self.page_size < 1:
            raise ValueError("at least one stage and a positive page size are required")
        self._w = _abi.Window(self.chunk_len, self.stages, self.history)
        try:
            self.slots, self.tokens = _abi.window_slots(self._w)
        except _abi.WfError as e:
            raise ValueError(f"invalid window (chunk_len >= 1, history >= 0, stages positive and "
                             f"strictly decreasing, at most {MAX_CHUNKS} slots): {e}") from None
        self.pages = math.ceil(self.tokens / self.page_size)

    def slots_and_tokens(self):
        return self.slots, self.tokens

    def view(self, t: int) -> RoundView:
        from . import _abi
        if t < 0:
            raise ValueError("rounds start at 0")
        r = _abi.window_round(self._w, t, ring=self.copy_free)
        n = r.num_chunks
        return RoundView(round=int(r.round), chunk_ids=[int(x) for x in r.chunk_id[:n]],
                         roles=[_ROLE_NAMES[x] for x in r.role[:n]],
                         chunk_stage=[int(x) for x in r.chunk_stage[:n]],
                         chunk_offsets=[int(x) for x in r.chunk_offsets[:n + 1]],
                         num_ctx_chunks=int(r.num_ctx_chunks),
                         store_to=None if r.store_to < 0 else int(r.store_to),
                         evicted=None if r.evicted < 0 else int(r.evicted),
                         store_kv_end=None if r.store_kv_end < 0 else int(r.store_kv_end))


class RollingCache:
    """Device state of a rolling window: one K/V pool holding ``num_layers`` layers of
    ``window.pages`` pages, and one fixed page-table row per layer.

    Each round, for every layer: :meth:`run_layer` appends the round's query chunks (store pass
    first, then the chunks in flight, in the order of :meth:`RollingWindow.view`).  It then runs
    attention for all of them in one launch and, once the ring is full, hands the store chunk into
    the slot of the chunk that leaves.
    """

    def __init__(self, window: RollingWindow, heads: int, head_dim: int, num_layers: int = 1,
                 device="cuda", page_tables: Optional[torch.Tensor] = None,
                 fill: Optional[float] = None):
        from .layer import PagedPool
        self.window = window
        self.num_layers = int(num_layers)
        self.pool = PagedPool(window.pages * self.num_layers, window.page_size, heads, head_dim,
                              device, fill=fill)
        if page_tables is None:
            page_tables = torch.arange(window.pages * self.num_layers, dtype=torch.int32)
            page_tables = page_tables.view(self.num_layers, window.pages)
        if tuple(page_tables.shape) != (self.num_layers, window.pages):
            raise ValueError("page_tables must be [num_layers, window.pages]")
        self.page_tables = page_tables.to(device=device, dtype=torch.int32).contiguous()

    def layer_view(self, view: RoundView, layer: int):
        from .layer import WavefrontLayer
        return WavefrontLayer(self.pool, self.page_tables, layer, view.chunk_offsets,
                              view.chunk_stage, view.num_ctx_chunks)

    def run_layer(self, view: RoundView, layer: int, q: torch.Tensor, k: torch.Tensor,
                  v: torch.Tensor, out: torch.Tensor, scale: Optional[float] = None,
                  lse: Optional[torch.Tensor] = None, stream=None) -> None:
        """One layer of round ``view.round``.  ``q``, ``k``, ``v``, ``out``: bf16 [T_q, H, D], the
        rows of the round's query chunks in logical order (store pass, then in flight)."""
        if view.t_q == 0:
            return
        lay = self.layer_view(view, layer)
        L = self.window.chunk_len
        if self.window.copy_free:
            self._run_segments(view, layer, lay, q, k, v, out, scale, lse, stream)
            return
        for i, slot in enumerate(view.query_slots):
            lay.append(slot, k[i * L:(i + 1) * L], v[i * L:(i + 1) * L], stream)
        lay.forward(q, out, scale=scale, lse=lse, stream=stream)
        if view.store_to is not None:
            # the store chunk is the first query chunk; after this layer's attention the evicted
            # chunk is no longer read, so its slot takes the store chunk's clean K/V
            lay.append(view.store_to, k[:L], v[:L], stream)

    def _run_segments(self, view: RoundView, layer: int, lay, q, k, v, out, scale, lse,
                      stream) -> None:
        """Copy-free round: every query chunk is appended once, into its own slot (the store pass
        into its ring slot), then one attention call over the round's query segments."""
        from . import _abi
        L = self.window.chunk_len
        for i, slot in enumerate(view.query_rows_slots):
            lay.append(slot, k[i * L:(i + 1) * L], v[i * L:(i + 1) * L], stream)
        rows_end, kv_end = view.segments()
        seg = _abi.Segments(rows_end, kv_end, view.chunk_offsets[-1],
                            self.page_tables.shape[1])
        if scale is None:
            scale = 1.0 / math.sqrt(self.pool.head_dim)
        _abi.attn_forward_segments(q, self.pool.k, self.pool.v, self.page_tables[layer], seg,
                                   scale, out, lse, 1, None, stream)
