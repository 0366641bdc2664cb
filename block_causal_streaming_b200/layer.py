"""Device-side state of one wavefront layer: paged K/V pools, page table and descriptor.

PyTorch provides the device memory and the stream; every step of the hot path runs through the
C ABI (:mod:`._abi`).  A pool may be shared by several layers (each with its own page-table row),
which is how the 30-layer round reuses one 4096-page pool.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import torch

from . import _abi


class PagedPool:
    """K and V pools, bf16 [num_pages, page_size, H, D] each, on one device."""

    def __init__(self, num_pages: int, page_size: int, heads: int, head_dim: int,
                 device="cuda", fill: Optional[float] = None):
        shape = (num_pages, page_size, heads, head_dim)
        self.k = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.empty(shape, dtype=torch.bfloat16, device=device)
        if fill is not None:
            self.k.fill_(fill)
            self.v.fill_(fill)
        self.num_pages, self.page_size, self.heads, self.head_dim = shape


class PagedPoolFp8:
    """FP8 K/V pool with the geometry of a :class:`PagedPool`: e4m3 codes uint8
    [num_pages, page_size, H, D] and one fp32 scale per (token, head) row [num_pages, page_size, H]
    for K and for V.  Filled by wf_kv_append_fp8, read back by wf_kv_dequant."""

    def __init__(self, num_pages: int, page_size: int, heads: int, head_dim: int,
                 device="cuda"):
        shape = (num_pages, page_size, heads, head_dim)
        self.k_codes = torch.zeros(shape, dtype=torch.uint8, device=device)
        self.v_codes = torch.zeros(shape, dtype=torch.uint8, device=device)
        self.k_scale = torch.zeros(shape[:3], dtype=torch.float32, device=device)
        self.v_scale = torch.zeros(shape[:3], dtype=torch.float32, device=device)
        self.num_pages, self.page_size, self.heads, self.head_dim = shape

    @property
    def tensors(self):
        return self.k_codes, self.v_codes, self.k_scale, self.v_scale


class QkI8Buffers:
    """The device buffers of the INT8 attention tier for one wavefront shape (see
    ``wf_qk_quantize_i8``): int8 Q and K' codes, their per-128-row scales, the key mean and its
    fp64 scratch."""

    def __init__(self, desc, heads: int, head_dim: int, device="cuda"):
        from . import _abi
        sizes = _abi.qk_i8_sizes(desc, heads, head_dim)
        off = desc.chunk_offsets
        t_kv, t_q = off[-1], off[-1] - off[desc.num_ctx_chunks]
        self.q_codes = torch.empty(t_q, heads, head_dim, dtype=torch.int8, device=device)
        self.q_scale = torch.empty(sizes[1] // 4, dtype=torch.float32, device=device)
        self.k_codes = torch.empty(t_kv, heads, head_dim, dtype=torch.int8, device=device)
        self.k_scale = torch.empty(sizes[3] // 4, dtype=torch.float32, device=device)
        self.k_mean = torch.empty(heads, head_dim, dtype=torch.float32, device=device)
        self.k_sum = torch.empty(heads, head_dim, dtype=torch.float64, device=device)
        self.heads = heads


class QkE4m3Buffers:
    """The device buffers of the FP8 (e4m3) attention tier for one wavefront shape (see
    ``wf_qk_quantize_e4m3``): e4m3 Q and K codes (uint8) and their per-128-row scales."""

    def __init__(self, desc, heads: int, head_dim: int, device="cuda"):
        from . import _abi
        sizes = _abi.qk_e4m3_sizes(desc, heads, head_dim)
        off = desc.chunk_offsets
        t_kv, t_q = off[-1], off[-1] - off[desc.num_ctx_chunks]
        self.q_codes = torch.empty(t_q, heads, head_dim, dtype=torch.uint8, device=device)
        self.q_scale = torch.empty(sizes[1] // 4, dtype=torch.float32, device=device)
        self.k_codes = torch.empty(t_kv, heads, head_dim, dtype=torch.uint8, device=device)
        self.k_scale = torch.empty(sizes[3] // 4, dtype=torch.float32, device=device)
        self.heads = heads


class WavefrontLayer:
    """One layer of a wavefront: its descriptor and its page-table rows.

    ``page_tables`` is int32 [num_layers, max_pages_per_seq] on the device (row ``layer`` is this
    layer's); ``chunk_offsets`` / ``chunk_stage`` / ``num_ctx_chunks`` describe the chunks in
    logical order (context first, then active chunks cleanest to noisiest).
    """

    def __init__(self, pool: PagedPool, page_tables: torch.Tensor, layer: int,
                 chunk_offsets: Sequence[int], chunk_stage: Sequence[int], num_ctx_chunks: int):
        self.pool = pool
        self.page_tables = page_tables
        self.layer = int(layer)
        self.desc = _abi.WavefrontDesc(chunk_offsets, chunk_stage, num_ctx_chunks,
                                       page_tables.shape[1])
        self.chunk_offsets = list(chunk_offsets)
        self.num_ctx_chunks = int(num_ctx_chunks)
        self._workspace: Optional[torch.Tensor] = None   # split-KV partial results
        self._ws_bytes: dict = {}                          # workspace bytes per `splits`

    @property
    def t_q(self) -> int:
        return self.chunk_offsets[-1] - self.chunk_offsets[self.num_ctx_chunks]

    def append(self, chunk: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        _abi.kv_append(self.pool.k, self.pool.v, self.layer, chunk, k, v, self.page_tables,
                       self.desc, stream)

    def append_range(self, k_all: torch.Tensor, v_all: torch.Tensor, chunks: Sequence[int],
                     stream=None) -> None:
        """Append the given chunks, slicing their rows out of logical-order K/V tensors."""
        for c in chunks:
            a, b = self.chunk_offsets[c], self.chunk_offsets[c + 1]
            self.append(c, k_all[a:b], v_all[a:b], stream)

    def forward_i8(self, q: torch.Tensor, out: torch.Tensor, qk: "QkI8Buffers",
                   scale: Optional[float] = None, lse: Optional[torch.Tensor] = None,
                   stream=None) -> None:
        """The INT8 tier: quantize q and this layer's keys into ``qk``, then attend."""
        from . import _abi
        if scale is None:
            scale = 1.0 / math.sqrt(self.pool.head_dim)
        row = self.page_tables[self.layer]
        _abi.qk_quantize_i8(q, self.pool.k, self.pool.v, row, self.desc, qk, stream)
        _abi.attn_forward_i8(qk, self.pool.k, self.pool.v, row, self.desc, scale, out, lse,
                             stream)

    def forward_e4m3(self, q: torch.Tensor, out: torch.Tensor, qk: "QkE4m3Buffers",
                     scale: Optional[float] = None, lse: Optional[torch.Tensor] = None,
                     stream=None) -> None:
        """The FP8 tier: quantize q and this layer's keys into ``qk`` as e4m3, then attend."""
        from . import _abi
        if scale is None:
            scale = 1.0 / math.sqrt(self.pool.head_dim)
        row = self.page_tables[self.layer]
        _abi.qk_quantize_e4m3(q, self.pool.k, self.pool.v, row, self.desc, qk, stream)
        _abi.attn_forward_e4m3(qk, self.pool.k, self.pool.v, row, self.desc, scale, out, lse,
                               stream)

    def forward(self, q: torch.Tensor, out: torch.Tensor, scale: Optional[float] = None,
                lse: Optional[torch.Tensor] = None, stream=None,
                splits: Optional[int] = None) -> None:
        """Attention of ``q`` over this layer's pages.  ``splits`` None: wf_attn_forward; an int:
        wf_attn_forward_split with that many key splits (0: the library's choice), with a
        workspace this layer allocates once and reuses."""
        if scale is None:
            scale = 1.0 / math.sqrt(self.pool.head_dim)
        if splits is None:
            _abi.attn_forward(q, self.pool.k, self.pool.v, self.page_tables[self.layer],
                              self.desc, scale, out, lse, stream)
            return
        need = self._ws_bytes.get(splits)
        if need is None:
            need = _abi.attn_workspace_size(self.desc, self.pool.heads, self.pool.head_dim,
                                            splits)
            self._ws_bytes[splits] = need
        ws = None
        if need > 0:
            if self._workspace is None or self._workspace.numel() < need:
                self._workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
            ws = self._workspace
        _abi.attn_forward_split(q, self.pool.k, self.pool.v, self.page_tables[self.layer],
                                self.desc, scale, out, splits, ws, lse, stream)
