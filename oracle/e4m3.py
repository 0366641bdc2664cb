"""Oracle for the FP8 (e4m3) attention tier -- TEST INFRASTRUCTURE ONLY (imported by ``tests/``
alone).

The project page ("03 End-to-end KV transport", item 01 "Precision") measures K/V in FP8, and the
pages name FP8 tensor-core attention only as a direction; they give no scale granularity for
attention operands.  The tier built here is this project's reading, the e4m3 twin of the INT8
tier (``oracle/int8.py``):

* **Blocks.**  One fp32 scale per (128 consecutive query rows, head) for Q and per (128
  consecutive keys in logical order, head) for K, counted from row / key 0 (the last block may
  be shorter).  One scale per S tile of the attention kernel, as in the INT8 tier.  No key
  smoothing: the floating format keeps each value's relative precision however far the block
  sits from zero.
* **Quantization** of a block with largest magnitude ``a``: ``inv = 448 / a`` and
  ``scale = a / 448`` (fp32 divisions; both 0 for a block of zeros or when ``448 / a``
  overflows), ``code = e4m3(x * inv)`` with an fp32 product, rounded to nearest even and
  saturated at 448 -- the encoder of the FP8 K/V pages (``oracle/fp8.py``).
* **Logits.**  ``s = softmax_scale * scale_q * scale_k * sum_d decode(q_d) * decode(k_d)``.  A
  product of two e4m3 values has at most 8 significant bits and lies in [2^-18, 2^17.6], so the
  sum of 128 of them is exact in fp64; the scales multiply in fp64.
* **The rest** is the block-causal attention of the bf16 path over the unquantized V, fp64.

Every function is pinned by ``tests/test_oracle_e4m3.py`` (the quantizer against its rounding
bound, saturation and zero blocks; the logits against a library matrix product of values decoded
through PyTorch's float8_e4m3fn type; a closed-form bound on the logit error; and planted
mistakes).
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

from oracle import fp8 as _fp8

QMAX = 448.0
Q_ROWS = 128      # query rows per Q scale block
K_KEYS = 128      # keys per K scale block


def _f32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def quantize_blocks(x, block: int):
    """x: [T, H, D] float32 -> (codes uint8 e4m3 [T, H, D], scale float32 [H, ceil(T / block)]).
    Block b of head h is rows [b * block, (b + 1) * block) of that head."""
    x = _f32(x)
    T, H, D = x.shape
    nb = (T + block - 1) // block
    codes = np.zeros((T, H, D), np.uint8)
    scale = np.zeros((H, nb), np.float32)
    for b in range(nb):
        rows = slice(b * block, min((b + 1) * block, T))
        xb = x[rows]                                            # [rows, H, D]
        a = np.max(np.abs(xb), axis=(0, 2)).astype(np.float32)  # [H]
        safe = np.where(a > 0, a, np.float32(1)).astype(np.float32)
        with np.errstate(over="ignore"):
            inv = (np.float32(QMAX) / safe).astype(np.float32)
        live = (a > 0) & np.isfinite(inv)
        inv = np.where(live, inv, np.float32(0)).astype(np.float32)
        scale[:, b] = np.where(live, safe / np.float32(QMAX), np.float32(0))
        codes[rows] = _fp8.e4m3_encode((xb * inv[None, :, None]).astype(np.float32))
    return codes, scale


def quantize_qk(q, k):
    """The whole quantization step: (q_codes, q_scale, k_codes, k_scale)."""
    k_codes, k_scale = quantize_blocks(_f32(k), K_KEYS)
    q_codes, q_scale = quantize_blocks(_f32(q), Q_ROWS)
    return q_codes, q_scale, k_codes, k_scale


def logits_rows(q_codes, q_scale, k_codes, k_scale, rows: Sequence[int], h: int, n: int,
                softmax_scale: float) -> np.ndarray:
    """fp64 logits [len(rows), n] of query rows `rows` of head h against keys [0, n)."""
    rows = np.asarray(rows)
    qv = _fp8.e4m3_decode(q_codes[rows, h, :]).astype(np.float64)
    kv = _fp8.e4m3_decode(k_codes[:n, h, :]).astype(np.float64)
    dots = qv @ kv.T                                   # exact: see the module docstring
    sq = q_scale[h, rows // Q_ROWS].astype(np.float64)[:, None]
    sk = k_scale[h, np.arange(n) // K_KEYS].astype(np.float64)[None, :]
    return softmax_scale * sq * sk * dots


def attention(q, k, v, chunk_offsets: Sequence[int], num_ctx_chunks: int, softmax_scale: float,
              rows: Sequence[int] = None, heads: Sequence[int] = None, quantized=None):
    """FP8-tier attention.  q [T_q, H, D] (query rows of chunks num_ctx_chunks..), k, v [T_kv, H, D]
    in logical order.  With rows/heads: outputs [n_sel, D] for the (row, head) pairs; else
    [T_q, H, D].  `quantized`: a quantize_qk result to reuse."""
    v64 = _f32(v).astype(np.float64)
    qc, qs, kc, ks = quantized if quantized is not None else quantize_qk(q, k)
    off = list(chunk_offsets)
    t_ctx, T_q, H = off[num_ctx_chunks], qc.shape[0], qc.shape[1]
    kv_end = np.empty(T_q, np.int64)
    for c in range(num_ctx_chunks, len(off) - 1):
        kv_end[off[c] - t_ctx:off[c + 1] - t_ctx] = off[c + 1]
    if rows is None:
        out = np.zeros((T_q, H, v64.shape[2]), np.float64)
        for h in range(H):
            for c in range(num_ctx_chunks, len(off) - 1):
                r = np.arange(off[c] - t_ctx, off[c + 1] - t_ctx)
                if len(r):
                    out[r, h] = _softmax_pv(logits_rows(qc, qs, kc, ks, r, h, off[c + 1],
                                                        softmax_scale), v64[:off[c + 1], h])
        return out.astype(np.float32)
    out = np.zeros((len(rows), v64.shape[2]), np.float64)
    rows, heads = np.asarray(rows), np.asarray(heads)
    # pairs with the same head and the same visible prefix share one matrix product
    groups = {}
    for i, (r, h) in enumerate(zip(rows, heads)):
        groups.setdefault((int(h), int(kv_end[r])), []).append(i)
    for (h, n), idx in groups.items():
        out[idx] = _softmax_pv(logits_rows(qc, qs, kc, ks, rows[idx], h, n, softmax_scale),
                               v64[:n, h])
    return out.astype(np.float32)


def _softmax_pv(s: np.ndarray, v: np.ndarray) -> np.ndarray:
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ v) / p.sum(axis=1, keepdims=True)
