"""Oracle for block-causal chunk attention and paged K/V -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The CUDA library and its Python binding never import it, and it imports nothing from them.

Two parts:

* :func:`attention` / :func:`attention_rows` -- ctypes front end of ``wf_oracle.c``, the plain
  fp64-accumulated definition of block-causal chunk attention with an explicit per-key chunk mask
  (full attention within a chunk, earlier cleaner chunks visible, later noisier chunks never:
  KipQuest summary of arXiv 2611.00859, "The deep dive"; project page, "01 The design gap", panel C).
* :func:`scatter_chunk` / :func:`gather_logical` -- the paged K/V layout written out in NumPy:
  logical token ``t`` of a sequence lives in physical page ``page_table[t // page_size]`` at row
  ``t % page_size`` of a pool shaped ``[num_pages][page_size][H][D]``.  This is the "paged" exchange
  mode of WaveRT, where producers write K/V straight into the consumer's fixed attention slots and
  attention reads the prefix in place (project page, "03 End-to-end KV transport", item 03 "Layout";
  GitHub README, "Runtime layout", ``exchange/`` modes).  The page table generalises the fixed slots.

Every function here is parity-pinned by ``tests/test_oracle_pins.py`` (brute force, closed forms,
invariants, a library routine, hand-derived golden cases and planted-mistake mutants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wf_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle with gcc (-O3, no fast-math, no FMA contraction: IEEE fp64 sums in
    the order the source writes them)."""
    cmd = ["gcc", "-O3", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _load(path: Optional[str] = None):
    global _lib
    if path is None:
        if _lib is not None:
            return _lib
        if (not os.path.exists(_LIB_PATH)
                or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
            build()
        path = _LIB_PATH
    lib = ctypes.CDLL(path)
    i32p = ctypes.POINTER(ctypes.c_int32)
    f32p = ctypes.POINTER(ctypes.c_float)
    lib.oracle_attention.argtypes = [f32p, f32p, f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, i32p, ctypes.c_double, f32p, f32p, ctypes.c_int]
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_attention_rows.argtypes = [f32p, f32p, f32p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, i32p, ctypes.c_double,
                                          i32p, i32p, ctypes.c_int, f32p, f32p, ctypes.c_int]
    lib.oracle_attention_rows.restype = ctypes.c_int
    if path == _LIB_PATH:
        _lib = lib
    return lib


def load_library(path: str):
    """Load an oracle library built from another source file (used by the mutant tests)."""
    return _load(path)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _f32(x) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> contiguous fp32 numpy (bf16 widens exactly)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def attention(q, k, v, chunk_offsets: Sequence[int], num_ctx_chunks: int, scale: float,
              with_lse: bool = False, nthreads: Optional[int] = None, lib=None):
    """Block-causal chunk attention for every query row and head.

    q: [T_q, H, D] (query rows of chunks ``num_ctx_chunks..`` in order); k, v: [T_kv, H, D] in
    logical order.  Returns out [T_q, H, D] fp32 (and lse [H, T_q] fp32 if ``with_lse``).
    """
    lib = lib or _load()
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    t_q, H, D = qf.shape
    off = np.ascontiguousarray(np.asarray(chunk_offsets, dtype=np.int32))
    out = np.zeros((t_q, H, D), dtype=np.float32)
    lse = np.zeros((H, t_q), dtype=np.float32) if with_lse else None
    rc = lib.oracle_attention(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                              _ptr(vf, ctypes.c_float), H, D, len(off) - 1, num_ctx_chunks,
                              _ptr(off, ctypes.c_int32), float(scale), _ptr(out, ctypes.c_float),
                              _ptr(lse, ctypes.c_float) if lse is not None else None,
                              nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attention rejected its arguments (code {rc})")
    return (out, lse) if with_lse else out


def attention_rows(q, k, v, chunk_offsets: Sequence[int], num_ctx_chunks: int, scale: float,
                   rows: Sequence[int], heads: Sequence[int], with_lse: bool = False,
                   nthreads: Optional[int] = None, lib=None):
    """The same attention for selected (row, head) pairs only: out [n, D] (and lse [n])."""
    lib = lib or _load()
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    t_q, H, D = qf.shape
    off = np.ascontiguousarray(np.asarray(chunk_offsets, dtype=np.int32))
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    h = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    assert r.shape == h.shape
    out = np.zeros((len(r), D), dtype=np.float32)
    lse = np.zeros((len(r),), dtype=np.float32) if with_lse else None
    rc = lib.oracle_attention_rows(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                                   _ptr(vf, ctypes.c_float), H, D, len(off) - 1, num_ctx_chunks,
                                   _ptr(off, ctypes.c_int32), float(scale),
                                   _ptr(r, ctypes.c_int32), _ptr(h, ctypes.c_int32), len(r),
                                   _ptr(out, ctypes.c_float),
                                   _ptr(lse, ctypes.c_float) if lse is not None else None,
                                   nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_attention_rows rejected its arguments (code {rc})")
    return (out, lse) if with_lse else out


# ---------------------------------------------------------------------------------------------
# Paged K/V: the reference for the append kernel and for the attention's page-table indexing.
# ---------------------------------------------------------------------------------------------

def scatter_chunk(pool: np.ndarray, page_table: Sequence[int], token_start: int,
                  rows: np.ndarray) -> None:
    """Write ``rows`` ([L, H, D]) as logical tokens token_start..token_start+L-1 into ``pool``.

    pool: [num_pages, page_size, H, D] (any dtype, modified in place); page_table: logical page ->
    physical page.  Raw element copy: the result is compared bit for bit.
    """
    page_size = pool.shape[1]
    for i in range(rows.shape[0]):
        t = token_start + i
        page = int(page_table[t // page_size])
        pool[page, t % page_size] = rows[i]


def gather_logical(pool: np.ndarray, page_table: Sequence[int], num_tokens: int) -> np.ndarray:
    """Read logical tokens 0..num_tokens-1 back out of the pool: [num_tokens, H, D]."""
    page_size = pool.shape[1]
    out = np.empty((num_tokens,) + pool.shape[2:], dtype=pool.dtype)
    for t in range(num_tokens):
        out[t] = pool[int(page_table[t // page_size]), t % page_size]
    return out
