"""Seeded synthetic wavefront inputs (shared by the CUDA path's tests, the bench and the oracle tests).

This module only *draws* inputs: chunk layouts, q/k/v values and page tables. It holds none of the
attention arithmetic, so the oracle and the CUDA path can both take their inputs from here without
sharing any of the computation they are compared on.

Workload shapes follow the Wave Forcing pages: a chunk is three latent frames (GitHub README,
"Quick start", note on ``--num-frames``); a Wan2.1 latent frame at 832x480 is 30x52 patches, so a
chunk is 4680 tokens; the 5-step wavefront has stages 1000/800/600/400/200 and the 4-step one
1000/750/500/250 (README, "Launch WaveRT" and "Run the 4-step checkpoint"); the critical consumer
sees 8 chunks of context in the 4-step layout (project page, "02 Interactive pipeline", the
"Inside one diffusion tick" panel: r0 sees 8 chunks, r3 sees 5).

Logical K/V order is oldest (cleanest) first: context chunks (stage 0), then active chunks from the
cleanest to the noisiest.  Queries exist only for the active chunks, packed in the same order.

Recipe (every workload): a CPU ``torch.Generator`` seeded with the workload's seed draws, in this
order, q ~ N(0,1) of shape [T_q, H, D], k ~ N(0,1) of shape [T_kv, H, D], v ~ N(0,1) of shape
[T_kv, H, D] (each multiplied by ``value_scale``), then (if ``k_mean_offset``) one mean vector
mu ~ N(0,1) of shape [H, D] added to every k row of that head, then the page permutation.  Values
are drawn in fp32 and rounded to bf16.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

CHUNK_TOKENS = 3 * 30 * 52  # 3 latent frames x 30x52 patches = 4680 tokens


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    head_dim: int
    ctx_lens: tuple            # token counts of the KV-only context chunks, oldest first
    active_lens: tuple         # token counts of the query-carrying chunks, cleanest first
    active_stages: tuple       # diffusion timestep of each active chunk, cleanest first
    page_size: int
    value_scale: float = 1.0
    k_mean_offset: bool = False
    seed: int = 0
    page_order: str = "perm"   # "identity" | "perm"
    pool_pages: Optional[int] = None  # pages in the pool (default: exactly the pages needed)
    layers: int = 1            # >1: independent layers sharing one pool (the 30-layer round)

    @property
    def num_chunks(self) -> int:
        return len(self.ctx_lens) + len(self.active_lens)

    @property
    def num_ctx_chunks(self) -> int:
        return len(self.ctx_lens)

    @property
    def chunk_lens(self) -> List[int]:
        return list(self.ctx_lens) + list(self.active_lens)

    @property
    def chunk_offsets(self) -> List[int]:
        off = [0]
        for n in self.chunk_lens:
            off.append(off[-1] + n)
        return off

    @property
    def chunk_stage(self) -> List[int]:
        return [0] * len(self.ctx_lens) + list(self.active_stages)

    @property
    def t_kv(self) -> int:
        return sum(self.chunk_lens)

    @property
    def t_ctx(self) -> int:
        return sum(self.ctx_lens)

    @property
    def t_q(self) -> int:
        return sum(self.active_lens)

    @property
    def pages_needed(self) -> int:
        return (self.t_kv + self.page_size - 1) // self.page_size

    @property
    def num_pages(self) -> int:
        return self.pool_pages if self.pool_pages is not None else self.pages_needed


def _ramp(n: int, lo: int, hi: int) -> tuple:
    """n stage values from the cleanest (lo) to the noisiest (hi)."""
    if n == 1:
        return (hi,)
    return tuple(lo + (hi - lo) * i // (n - 1) for i in range(n))


# A tiny wavefront and synthetic wavefronts of the Wan2.1 1.3B and 14B shapes.
TINY = Workload("tiny_3x48_h2_d64", heads=2, head_dim=64, ctx_lens=(),
                active_lens=(48, 48, 48), active_stages=(200, 600, 1000), page_size=16,
                value_scale=1.0, seed=0, page_order="identity")
WAN13B_5STEP = Workload("wan1.3b_5step_2ctx+5x4680_h12_d128", heads=12, head_dim=128,
                        ctx_lens=(CHUNK_TOKENS,) * 2, active_lens=(CHUNK_TOKENS,) * 5,
                        active_stages=(200, 400, 600, 800, 1000), page_size=64,
                        value_scale=0.5, seed=1, page_order="perm")
WAN13B_4STEP = Workload("wan1.3b_4step_4ctx+4x4680_h12_d128_kmean", heads=12, head_dim=128,
                        ctx_lens=(CHUNK_TOKENS,) * 4, active_lens=(CHUNK_TOKENS,) * 4,
                        active_stages=(250, 500, 750, 1000), page_size=64,
                        value_scale=1.0, k_mean_offset=True, seed=2, page_order="perm")
WAN13B_ROUND30 = Workload("wan1.3b_5step_round_30_layers", heads=12, head_dim=128,
                          ctx_lens=(CHUNK_TOKENS,) * 2, active_lens=(CHUNK_TOKENS,) * 5,
                          active_stages=(200, 400, 600, 800, 1000), page_size=64,
                          value_scale=0.5, seed=3, page_order="perm", pool_pages=4096, layers=30)
WAN14B = Workload("wan14b_6ctx+5x4680_h40_d128_ps128", heads=40, head_dim=128,
                  ctx_lens=(CHUNK_TOKENS,) * 6, active_lens=(CHUNK_TOKENS,) * 5,
                  active_stages=(200, 400, 600, 800, 1000), page_size=128,
                  value_scale=0.5, seed=4, page_order="perm")

# One Wave-Parallelism rank's call: the critical consumer's single query chunk against a context
# of 7 earlier chunks (8 chunks visible; project page, "02 Interactive pipeline", "Inside one
# diffusion tick").  Seed 5; otherwise the 1.3B shapes above.
WP_RANK0 = Workload("wp_rank0_7ctx+1x4680_h12_d128", heads=12, head_dim=128,
                    ctx_lens=(CHUNK_TOKENS,) * 7, active_lens=(CHUNK_TOKENS,),
                    active_stages=(1000,), page_size=64, value_scale=0.5, seed=5,
                    page_order="perm")

# The workloads by short name (bench.py --workload).
WORKLOADS = {"tiny": TINY, "wan13b_5step": WAN13B_5STEP, "wan13b_4step": WAN13B_4STEP,
             "wan13b_round30": WAN13B_ROUND30, "wan14b": WAN14B, "wp_rank0": WP_RANK0}


def small_case(name: str, heads: int, head_dim: int, ctx_lens, active_lens, page_size: int,
               seed: int, value_scale: float = 1.0, k_mean_offset: bool = False,
               page_order: str = "perm", pool_pages: Optional[int] = None) -> Workload:
    """A parity-sized workload: several tiles, ragged tails, any chunk mix."""
    return Workload(name, heads=heads, head_dim=head_dim, ctx_lens=tuple(ctx_lens),
                    active_lens=tuple(active_lens),
                    active_stages=_ramp(len(active_lens), 200, 1000), page_size=page_size,
                    value_scale=value_scale, k_mean_offset=k_mean_offset, seed=seed,
                    page_order=page_order, pool_pages=pool_pages)


@dataclasses.dataclass
class LayerInputs:
    q: torch.Tensor            # bf16 [T_q, H, D]
    k: torch.Tensor            # bf16 [T_kv, H, D], logical order
    v: torch.Tensor            # bf16 [T_kv, H, D], logical order
    page_table: torch.Tensor   # int32 [pages_needed]: logical page -> physical page


def _draw_layer(wl: Workload, g: torch.Generator) -> LayerInputs:
    H, D = wl.heads, wl.head_dim
    q = torch.randn(wl.t_q, H, D, generator=g, dtype=torch.float32) * wl.value_scale
    k = torch.randn(wl.t_kv, H, D, generator=g, dtype=torch.float32) * wl.value_scale
    v = torch.randn(wl.t_kv, H, D, generator=g, dtype=torch.float32) * wl.value_scale
    if wl.k_mean_offset:
        mu = torch.randn(H, D, generator=g, dtype=torch.float32)
        k = k + mu.unsqueeze(0)
    if wl.page_order == "identity":
        pt = torch.arange(wl.pages_needed, dtype=torch.int32)
    else:
        pt = torch.randperm(wl.num_pages, generator=g)[: wl.pages_needed].to(torch.int32)
    return LayerInputs(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16),
                       v=v.to(torch.bfloat16), page_table=pt.contiguous())


def make_layers(wl: Workload, layers: Optional[int] = None) -> List[LayerInputs]:
    """Draw ``layers`` (default: all of the workload's) layers from one seeded generator."""
    g = torch.Generator().manual_seed(wl.seed)
    n = wl.layers if layers is None else layers
    return [_draw_layer(wl, g) for _ in range(n)]


def make_inputs(wl: Workload) -> LayerInputs:
    """The first (for single-layer workloads: the only) layer of a workload."""
    g = torch.Generator().manual_seed(wl.seed)
    return _draw_layer(wl, g)
