"""Oracle for the INT8 (Sage-like) attention tier -- TEST INFRASTRUCTURE ONLY (imported by ``tests/``
alone).

The pages name SageAttention with W8A8 as the fast attention backend (GitHub README, results table,
"Sage . causal . paged" rows; KipQuest abstract) and give no internals, so the tier is this
project's own reading of that family of methods:

* **Smoothing.**  ``mu[h, :]`` is the mean of the keys of head ``h`` over all ``T_kv`` tokens of the
  layer; quantization sees ``K' = K - mu``.  Subtracting one vector from every key adds the same
  constant ``q . mu`` to every logit of a query row, so the softmax -- and the attention -- of the
  unquantized keys are unchanged; the quantizer then works on centred values.  The sum is taken
  exactly (``math.fsum``) and divided in fp64, then rounded once to fp32; ``K'`` is the fp32
  difference.
* **Blocks.**  One scale per (128 consecutive query rows, head) for Q and per (128 consecutive keys
  in logical order, head) for K, both counted from row / key 0 (the last block may be shorter).
* **Quantization** of a block with largest magnitude ``a``: ``inv = 127 / a`` and
  ``scale = a / 127`` (fp32 divisions; both 0 for a block of zeros or when ``127 / a`` overflows),
  ``code = clamp(round_half_even(x * inv), -127, 127)`` with an fp32 product.  These steps decide
  integer codes, so they are fp32 as on the device.
* **Logits.**  ``s = softmax_scale * scale_q * scale_k * sum_d qcode * kcode``: the integer sum is
  exact; the product of the scales is taken in fp64 here.
* **The rest** is the block-causal attention of the bf16 path: each query chunk sees the keys
  ``[0, kv_end)`` of its prefix, softmax over them, ``O = P V`` with V unquantized.  fp64
  throughout.

Every function is pinned by ``tests/test_oracle_int8.py`` (quantizer bounds and ties, the exact
integer logits against a library matrix product, the smoothing invariance of exact attention, a
closed-form bound on the logit error, and planted mistakes).
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np

QMAX = 127
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


def key_mean(k) -> np.ndarray:
    """k: [T, H, D] (bf16 values) -> mu float32 [H, D]: exact sum, fp64 division, fp32 rounding."""
    k = _f32(k).astype(np.float64)
    T, H, D = k.shape
    cols = k.reshape(T, H * D)
    mu = np.array([math.fsum(cols[:, i]) for i in range(H * D)], dtype=np.float64) / T
    return mu.astype(np.float32).reshape(H, D)


def smooth(k, mu) -> np.ndarray:
    """K' = K - mu (fp32 subtraction), mu broadcast over tokens."""
    return (_f32(k) - np.asarray(mu, np.float32)[None]).astype(np.float32)


def quantize_blocks(x, block: int):
    """x: [T, H, D] float32 -> (codes int8 [T, H, D], scale float32 [H, ceil(T / block)]).
    Block b of head h is rows [b * block, (b + 1) * block) of that head."""
    x = _f32(x)
    T, H, D = x.shape
    nb = (T + block - 1) // block
    codes = np.zeros((T, H, D), np.int8)
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
        y = (xb * inv[None, :, None]).astype(np.float32)
        codes[rows] = np.clip(np.rint(y), -QMAX, QMAX).astype(np.int8)   # rint: half to even
    return codes, scale


def quantize_qk(q, k):
    """The whole quantization step: (q_codes, q_scale, k_codes, k_scale, mu)."""
    mu = key_mean(k)
    k_codes, k_scale = quantize_blocks(smooth(k, mu), K_KEYS)
    q_codes, q_scale = quantize_blocks(_f32(q), Q_ROWS)
    return q_codes, q_scale, k_codes, k_scale, mu


def logits_rows(q_codes, q_scale, k_codes, k_scale, rows: Sequence[int], h: int, n: int,
                softmax_scale: float) -> np.ndarray:
    """fp64 logits [len(rows), n] of query rows `rows` of head h against keys [0, n)."""
    rows = np.asarray(rows)
    # |sum| <= 128 * 127^2 < 2^53 and every partial sum is an integer, so the fp64 product is
    # the exact integer one in any summation order
    dots = q_codes[rows, h, :].astype(np.float64) @ k_codes[:n, h, :].astype(np.float64).T
    sq = q_scale[h, rows // Q_ROWS].astype(np.float64)[:, None]
    sk = k_scale[h, np.arange(n) // K_KEYS].astype(np.float64)[None, :]
    return softmax_scale * sq * sk * dots.astype(np.float64)


def attention(q, k, v, chunk_offsets: Sequence[int], num_ctx_chunks: int, softmax_scale: float,
              rows: Sequence[int] = None, heads: Sequence[int] = None, quantized=None):
    """INT8-tier attention.  q [T_q, H, D] (query rows of chunks num_ctx_chunks..), k, v [T_kv, H, D]
    in logical order.  With rows/heads: outputs [n_sel, D] for the (row, head) pairs; else
    [T_q, H, D].  `quantized`: a quantize_qk result to reuse."""
    v64 = _f32(v).astype(np.float64)
    qc, qs, kc, ks, _ = quantized if quantized is not None else quantize_qk(q, k)
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
