"""Wave Parallelism plumbing: every rank's paged pool and flag array, mapped into every process.

In Wave Parallelism each GPU (one process per GPU) owns one chunk of the wavefront and attends to
every chunk before it; each producer publishes its chunk's K/V, right after projection, straight
into the consumers' attention buffers, one way (project page, "03 End-to-end KV transport",
items 01-03).  :class:`PublishedPools` exchanges CUDA IPC handles of each rank's K pool, V pool
and flag array over a ``torch.distributed`` group (any backend: only handles and integers cross
it) and maps the other ranks' allocations into this process with ``wf_ipc_import``.  The data
path is the library's: ``wf_kv_append_publish`` writes the chunk into the local pool and the
consumers' pools and raises the chunk's flag everywhere, and ``wf_attn_forward_published`` waits
for the flags before reading.  The FP8 form does the same with e4m3 codes and scales
(``wf_kv_append_publish_fp8``), and the consumer converts a chunk once its flag is up
(``wf_kv_dequant_published``).

All ranks must create their pools with the same geometry and use the same page table, so a chunk
lands in the same pages everywhere.  Every rank takes the same collective steps in the same
order.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import _abi

WF_MAX_CHUNKS = 64


def new_flags(num_layers: int, device) -> torch.Tensor:
    """A zeroed flag array int32 [num_layers, WF_MAX_CHUNKS] (word = last published generation)."""
    return torch.zeros(num_layers, WF_MAX_CHUNKS, dtype=torch.int32, device=device)


def consumers_of(rank: int, world: int) -> List[int]:
    """Ranks that attend to rank's chunk: in Wave Parallelism every later chunk sees it."""
    return list(range(rank + 1, world))


class PublishedPools:
    """The pools and flag arrays of all ranks, mapped into this process.

    ``peer(r)`` is rank r's (k_pool, v_pool, flags) as device pointers valid here (this rank's own
    allocations for r == rank).  With ``fp8`` -- this rank's FP8 pool as (k_codes, v_codes,
    k_scale, v_scale) tensors -- ``peer_fp8(r)`` is rank r's (k_codes, v_codes, k_scale, v_scale,
    flags), the destination form of ``wf_kv_append_publish_fp8``.  Call :meth:`close` (all ranks)
    before the process group goes.
    """

    def __init__(self, k_pool: torch.Tensor, v_pool: torch.Tensor, flags: torch.Tensor,
                 group=None, fp8: Optional[Sequence[torch.Tensor]] = None):
        import torch.distributed as dist
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        own = [k_pool.data_ptr(), v_pool.data_ptr(), flags.data_ptr()]
        if fp8 is not None:
            own += [t.data_ptr() for t in fp8]
        handles = tuple(_abi.ipc_export(p) for p in own)
        gathered: List[Optional[Tuple[bytes, ...]]] = [None] * self.world
        dist.all_gather_object(gathered, handles, group=group)
        if any(len(hs) != len(own) for hs in gathered):
            raise ValueError("every rank must pass an FP8 pool, or none")
        self._mapped: List[int] = []
        self._ptrs: Dict[int, Tuple[int, ...]] = {self.rank: tuple(own)}
        # Several tensors may live in one allocation of the owner's caching allocator, so they
        # share an IPC handle: each allocation is mapped (and later closed) once.
        opened: Dict[bytes, Tuple[int, int]] = {}      # handle -> (pointer, offset) first mapped
        for r, hs in enumerate(gathered):
            if r == self.rank:
                continue
            ptrs = []
            for handle, off in hs:
                if handle in opened:
                    p0, off0 = opened[handle]
                    ptrs.append(p0 - off0 + off)
                    continue
                p = _abi.ipc_import((handle, off))
                opened[handle] = (p, off)
                self._mapped.append(p)
                ptrs.append(p)
            self._ptrs[r] = tuple(ptrs)

    def peer(self, r: int) -> Tuple[int, int, int]:
        return self._ptrs[r][:3]

    def peer_fp8(self, r: int) -> Tuple[int, int, int, int, int]:
        p = self._ptrs[r]
        if len(p) < 7:
            raise ValueError("no FP8 pools were exchanged")
        return p[3], p[4], p[5], p[6], p[2]

    def destinations(self, ranks: Sequence[int]) -> List[Tuple[int, int, int]]:
        """The (k_pool, v_pool, flags) triples of ``ranks`` (this rank excluded)."""
        return [self.peer(r) for r in ranks if r != self.rank]

    def destinations_fp8(self, ranks: Sequence[int]) -> List[Tuple[int, int, int, int, int]]:
        """The FP8 destinations (k_codes, v_codes, k_scale, v_scale, flags) of ``ranks`` (this
        rank excluded)."""
        return [self.peer_fp8(r) for r in ranks if r != self.rank]

    def close(self) -> None:
        for p in self._mapped:
            _abi.ipc_close(p)
        self._mapped = []
