"""Helpers shared by the GPU tests: put a seeded workload on the device through the C ABI."""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from block_causal_streaming_b200.layer import PagedPool, WavefrontLayer
from block_causal_streaming_b200.workloads import LayerInputs, Workload

MAX_ABS = 1e-2   # bf16 outputs, fp32 accumulation: the stated parity bar
MEAN_ABS = 1e-3


def place(wl: Workload, inp: LayerInputs, device="cuda", fill: Optional[float] = None,
          pool: Optional[PagedPool] = None, append: bool = True, extra_pages: int = 0):
    """Allocate pools (or reuse ``pool``), upload q/k/v and the page table, append every chunk."""
    if pool is None:
        pool = PagedPool(wl.num_pages + extra_pages, wl.page_size, wl.heads, wl.head_dim,
                         device, fill)
    pt = inp.page_table.to(device).reshape(1, -1).contiguous()
    layer = WavefrontLayer(pool, pt, 0, wl.chunk_offsets, wl.chunk_stage, wl.num_ctx_chunks)
    q = inp.q.to(device)
    k = inp.k.to(device)
    v = inp.v.to(device)
    if append:
        layer.append_range(k, v, range(wl.num_chunks))
    return layer, q, k, v


def run(layer: WavefrontLayer, q: torch.Tensor, with_lse: bool = False, scale=None):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device) \
        if with_lse else None
    layer.forward(q, out, scale=scale, lse=lse)
    return (out, lse) if with_lse else out


def scale_of(wl: Workload) -> float:
    return 1.0 / math.sqrt(wl.head_dim)


def assert_parity(got: np.ndarray, ref: np.ndarray, what: str = ""):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e} > {MEAN_ABS}"
    return float(err.max()), float(err.mean())


def sample_rows(wl: Workload, per_chunk: int = 3, seed: int = 0):
    """Query rows worth checking: chunk edges, tile edges next to them, the tail, random rows."""
    rng = np.random.default_rng(seed)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    t_ctx, t_q = off[nctx], wl.t_q
    rows = {0, t_q - 1}
    for c in range(nctx, wl.num_chunks):
        a, b = off[c] - t_ctx, off[c + 1] - t_ctx
        if b <= a:
            continue
        rows.update({a, b - 1, min(b, t_q - 1)})
        for edge in (a - a % 128, a - a % 256 + 255, b - b % 128):
            if 0 <= edge < t_q:
                rows.add(edge)
        rows.update(int(x) for x in rng.integers(a, b, size=per_chunk))
    rows = sorted(r for r in rows if 0 <= r < t_q)
    heads = [int(h) for h in rng.integers(0, wl.heads, size=len(rows))]
    heads[0], heads[-1] = 0, wl.heads - 1
    return rows, heads


UNIT_ROWS = 256   # query rows of one attention work unit (two 128-row Q tiles)


def whole_units(wl: Workload, seed: int = 0, interior: bool = True):
    """Every head of every row of whole 256-row work units: for each query chunk the unit that
    holds its first row and the one that holds its last row (these straddle chunk boundaries
    unless a boundary falls on a unit edge) and, with `interior`, one interior unit drawn at
    random; the last unit of the wavefront, whose rows see the most keys, is always among them.
    Returns
    (rows, heads, units), rows/heads flattened so that pair i is (rows[i], heads[i])."""
    rng = np.random.default_rng(seed)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    t_ctx, t_q = off[nctx], wl.t_q
    units = {(t_q - 1) // UNIT_ROWS}
    for c in range(nctx, wl.num_chunks):
        a, b = off[c] - t_ctx, off[c + 1] - t_ctx
        if b <= a:
            continue
        first, last = a // UNIT_ROWS, (b - 1) // UNIT_ROWS
        units.update({first, last})
        if interior and last - first > 1:
            units.add(int(rng.integers(first + 1, last)))
    units = sorted(units)
    rows = np.concatenate([np.arange(u * UNIT_ROWS, min((u + 1) * UNIT_ROWS, t_q))
                           for u in units]).astype(np.int32)
    heads = np.tile(np.arange(wl.heads, dtype=np.int32), len(rows))
    rows = np.repeat(rows, wl.heads)
    return rows, heads, units
