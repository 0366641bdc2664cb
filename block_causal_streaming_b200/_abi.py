"""ctypes binding of ``libwf_b200.so`` (the C ABI in ``include/wf.h``).

Argument marshalling only: every step of append and attention runs in the library's kernels.
There is no CPU fallback; if the library is missing, importing the binding raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
# WF_B200_LIB points the binding at another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("WF_B200_LIB") or os.path.join(HERE, "libwf_b200.so")

WF_OK = 0
WF_ERR_INVALID_ARG = 1
WF_ERR_SHAPE = 2
WF_ERR_STAGE_ORDER = 3
WF_ERR_CAPACITY = 4
WF_ERR_PAGE_OOB = 5
WF_ERR_TIMEOUT = 6
WF_ERR_CUDA = 7
WF_ERR_NO_DEVICE = 8
WF_MAX_CHUNKS = 64

# Every symbol include/wf.h declares (checked by the CPU tests).
EXPORTED = ("wf_kv_append", "wf_attn_forward", "wf_check_status", "wf_strerror", "wf_version",
            "wf_selftest_timeout", "wf_attn_forward_split", "wf_attn_workspace_size",
            "wf_attn_forward_split_noalloc", "wf_kv_append_publish", "wf_attn_forward_published",
            "wf_ipc_export", "wf_ipc_import", "wf_ipc_close", "wf_kv_append_fp8",
            "wf_kv_dequant", "wf_kv_append_fp8_chunks", "wf_kv_dequant_chunks",
            "wf_attn_split_plan", "wf_qk_e4m3_sizes", "wf_qk_quantize_e4m3",
            "wf_attn_forward_e4m3", "wf_kv_append_publish_fp8", "wf_kv_dequant_published",
            "wf_qk_i8_sizes", "wf_qk_quantize_i8", "wf_attn_forward_i8",
            "wf_attn_forward_segments", "wf_attn_segments_workspace_size",
            "wf_window_slots", "wf_window_round", "wf_window_round_ring")


class WfError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)}")


class PoolDst(ctypes.Structure):
    """wf_pool_dst_t: a destination pool (usually another GPU's, mapped by ipc_import)."""
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("flags", ctypes.c_void_p)]


class Fp8Dst(ctypes.Structure):
    """wf_fp8_dst_t: a destination FP8 pool (usually another GPU's, mapped by ipc_import)."""
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("flags", ctypes.c_void_p)]


class QkI8(ctypes.Structure):
    """wf_qk_i8_t: the quantized Q and K' of the INT8 tier (device pointers)."""
    _fields_ = [("q_codes", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("k_mean", ctypes.c_void_p), ("k_sum", ctypes.c_void_p)]


class QkE4m3(ctypes.Structure):
    """wf_qk_e4m3_t: the e4m3 Q and K of the FP8 tier (device pointers)."""
    _fields_ = [("q_codes", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p)]


class KvPool(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class KvPoolFp8(ctypes.Structure):
    """wf_kv_pool_fp8_t: e4m3 codes [pages, page_size, H, D] and fp32 scales [pages, page_size, H]."""
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class WindowC(ctypes.Structure):
    """wf_window_t."""
    _fields_ = [("chunk_len", ctypes.c_int32), ("num_stages", ctypes.c_int32),
                ("stages", ctypes.POINTER(ctypes.c_int32)), ("history", ctypes.c_int32)]


class RoundC(ctypes.Structure):
    """wf_round_t."""
    _fields_ = [("round", ctypes.c_int64), ("num_chunks", ctypes.c_int32),
                ("num_ctx_chunks", ctypes.c_int32), ("chunk_id", ctypes.c_int64 * 64),
                ("role", ctypes.c_int32 * 64), ("chunk_stage", ctypes.c_int32 * 64),
                ("chunk_offsets", ctypes.c_int32 * 65), ("store_to", ctypes.c_int32),
                ("evicted", ctypes.c_int64), ("store_kv_end", ctypes.c_int32)]


class SegmentsC(ctypes.Structure):
    """wf_segments_t."""
    _fields_ = [("num_segments", ctypes.c_int32),
                ("rows_end", ctypes.POINTER(ctypes.c_int32)),
                ("kv_end", ctypes.POINTER(ctypes.c_int32)),
                ("num_keys", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32)]


class Wavefront(ctypes.Structure):
    _fields_ = [("num_chunks", ctypes.c_int32), ("num_ctx_chunks", ctypes.c_int32),
                ("chunk_offsets", ctypes.POINTER(ctypes.c_int32)),
                ("chunk_stage", ctypes.POINTER(ctypes.c_int32)),
                ("max_pages_per_seq", ctypes.c_int32)]


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m block_causal_streaming_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.wf_kv_append.argtypes = [ctypes.POINTER(KvPool), i32, i32, vp, vp,
                                 ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(Wavefront), vp]
    lib.wf_kv_append.restype = i32
    lib.wf_attn_forward.argtypes = [vp, ctypes.POINTER(KvPool), ctypes.POINTER(ctypes.c_int32),
                                    ctypes.POINTER(Wavefront), f32, vp,
                                    ctypes.POINTER(ctypes.c_float), vp]
    lib.wf_attn_forward.restype = i32
    lib.wf_check_status.argtypes = [vp]
    lib.wf_check_status.restype = i32
    lib.wf_strerror.argtypes = [i32]
    lib.wf_strerror.restype = ctypes.c_char_p
    lib.wf_version.argtypes = []
    lib.wf_version.restype = i32
    lib.wf_selftest_timeout.argtypes = [ctypes.c_uint, vp]
    lib.wf_selftest_timeout.restype = i32
    lib.wf_attn_forward_split.argtypes = [vp, ctypes.POINTER(KvPool),
                                          ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(Wavefront), ctypes.c_float, vp,
                                          ctypes.POINTER(ctypes.c_float), i32, vp,
                                          ctypes.c_size_t, vp]
    lib.wf_attn_forward_split.restype = i32
    lib.wf_attn_forward_split_noalloc.argtypes = [vp, ctypes.POINTER(KvPool),
                                                  ctypes.POINTER(ctypes.c_int32),
                                                  ctypes.POINTER(Wavefront), ctypes.c_float, vp,
                                                  ctypes.POINTER(ctypes.c_float), i32, vp]
    lib.wf_attn_forward_split_noalloc.restype = i32
    lib.wf_kv_append_publish.argtypes = [ctypes.POINTER(KvPool), vp, ctypes.POINTER(PoolDst),
                                         i32, i32, i32, vp, vp, ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(Wavefront), ctypes.c_uint32, vp]
    lib.wf_kv_append_publish.restype = i32
    lib.wf_attn_forward_published.argtypes = [vp, ctypes.POINTER(KvPool),
                                              ctypes.POINTER(ctypes.c_int32),
                                              ctypes.POINTER(Wavefront), ctypes.c_float, vp,
                                              ctypes.POINTER(ctypes.c_float), vp,
                                              ctypes.c_uint32, i32, vp, ctypes.c_size_t, vp]
    lib.wf_attn_forward_published.restype = i32
    lib.wf_ipc_export.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_size_t)]
    lib.wf_ipc_export.restype = i32
    lib.wf_ipc_import.argtypes = [vp, ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]
    lib.wf_ipc_import.restype = i32
    lib.wf_ipc_close.argtypes = [vp]
    lib.wf_ipc_close.restype = i32
    lib.wf_attn_workspace_size.argtypes = [ctypes.POINTER(Wavefront), i32, i32, i32]
    lib.wf_attn_workspace_size.restype = ctypes.c_size_t
    lib.wf_attn_split_plan.argtypes = [ctypes.POINTER(Wavefront), i32, i32, i32,
                                       ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_int32)]
    lib.wf_attn_split_plan.restype = i32
    lib.wf_kv_append_fp8.argtypes = [ctypes.POINTER(KvPoolFp8), i32, i32, vp, vp,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(Wavefront), vp]
    lib.wf_kv_append_fp8.restype = i32
    lib.wf_kv_dequant.argtypes = [ctypes.POINTER(KvPoolFp8), ctypes.POINTER(KvPool), i32, i32,
                                  ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(Wavefront), vp]
    lib.wf_kv_dequant.restype = i32
    lib.wf_kv_append_fp8_chunks.argtypes = [ctypes.POINTER(KvPoolFp8), i32, i32, i32, vp, vp,
                                            ctypes.POINTER(ctypes.c_int32),
                                            ctypes.POINTER(Wavefront), vp]
    lib.wf_kv_append_fp8_chunks.restype = i32
    lib.wf_kv_dequant_chunks.argtypes = [ctypes.POINTER(KvPoolFp8), ctypes.POINTER(KvPool), i32,
                                         i32, i32, ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(Wavefront), vp]
    lib.wf_kv_dequant_chunks.restype = i32
    lib.wf_kv_append_publish_fp8.argtypes = [ctypes.POINTER(KvPoolFp8), vp,
                                             ctypes.POINTER(Fp8Dst), i32, i32, i32, vp, vp,
                                             ctypes.POINTER(ctypes.c_int32),
                                             ctypes.POINTER(Wavefront), ctypes.c_uint32, vp]
    lib.wf_kv_append_publish_fp8.restype = i32
    lib.wf_kv_dequant_published.argtypes = [ctypes.POINTER(KvPoolFp8), ctypes.POINTER(KvPool),
                                            i32, i32, ctypes.POINTER(ctypes.c_int32),
                                            ctypes.POINTER(Wavefront), vp, ctypes.c_uint32, vp]
    lib.wf_kv_dequant_published.restype = i32
    lib.wf_qk_i8_sizes.argtypes = [ctypes.POINTER(Wavefront), i32, i32,
                                   ctypes.POINTER(ctypes.c_size_t)]
    lib.wf_qk_i8_sizes.restype = i32
    lib.wf_qk_quantize_i8.argtypes = [vp, ctypes.POINTER(KvPool), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(Wavefront), ctypes.POINTER(QkI8), vp]
    lib.wf_qk_quantize_i8.restype = i32
    lib.wf_attn_forward_i8.argtypes = [ctypes.POINTER(QkI8), ctypes.POINTER(KvPool),
                                       ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(Wavefront),
                                       f32, vp, ctypes.POINTER(ctypes.c_float), vp]
    lib.wf_attn_forward_i8.restype = i32
    lib.wf_qk_e4m3_sizes.argtypes = [ctypes.POINTER(Wavefront), i32, i32,
                                     ctypes.POINTER(ctypes.c_size_t)]
    lib.wf_qk_e4m3_sizes.restype = i32
    lib.wf_qk_quantize_e4m3.argtypes = [vp, ctypes.POINTER(KvPool),
                                        ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(Wavefront), ctypes.POINTER(QkE4m3), vp]
    lib.wf_qk_quantize_e4m3.restype = i32
    lib.wf_attn_forward_e4m3.argtypes = [ctypes.POINTER(QkE4m3), ctypes.POINTER(KvPool),
                                         ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(Wavefront), f32, vp,
                                         ctypes.POINTER(ctypes.c_float), vp]
    lib.wf_attn_forward_e4m3.restype = i32
    lib.wf_window_slots.argtypes = [ctypes.POINTER(WindowC), ctypes.POINTER(ctypes.c_int32),
                                    ctypes.POINTER(ctypes.c_int64)]
    lib.wf_window_slots.restype = i32
    lib.wf_window_round.argtypes = [ctypes.POINTER(WindowC), ctypes.c_int64,
                                    ctypes.POINTER(RoundC)]
    lib.wf_window_round.restype = i32
    lib.wf_window_round_ring.argtypes = [ctypes.POINTER(WindowC), ctypes.c_int64,
                                         ctypes.POINTER(RoundC)]
    lib.wf_window_round_ring.restype = i32
    lib.wf_attn_forward_segments.argtypes = [vp, ctypes.POINTER(KvPool),
                                             ctypes.POINTER(ctypes.c_int32),
                                             ctypes.POINTER(SegmentsC), f32, vp,
                                             ctypes.POINTER(ctypes.c_float), i32, vp,
                                             ctypes.c_size_t, vp]
    lib.wf_attn_forward_segments.restype = i32
    lib.wf_attn_segments_workspace_size.argtypes = [ctypes.POINTER(SegmentsC), i32, i32, i32]
    lib.wf_attn_segments_workspace_size.restype = ctypes.c_size_t
    return lib


lib = _load()


def strerror(code: int) -> str:
    return lib.wf_strerror(int(code)).decode()


class WavefrontDesc:
    """Host copy of a wavefront descriptor; keeps the arrays alive while C reads them."""

    def __init__(self, chunk_offsets: Sequence[int], chunk_stage: Sequence[int],
                 num_ctx_chunks: int, max_pages_per_seq: int):
        n = len(chunk_offsets) - 1
        self._off = (ctypes.c_int32 * (n + 1))(*[int(x) for x in chunk_offsets])
        self._stage = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in chunk_stage])
        self.c = Wavefront(n, int(num_ctx_chunks),
                           ctypes.cast(self._off, ctypes.POINTER(ctypes.c_int32)),
                           ctypes.cast(self._stage, ctypes.POINTER(ctypes.c_int32)),
                           int(max_pages_per_seq))
        self.chunk_offsets = [int(x) for x in chunk_offsets]
        self.num_ctx_chunks = int(num_ctx_chunks)


def _pool_struct(k_pool, v_pool) -> KvPool:
    num_pages, page_size, H, D = (int(x) for x in k_pool.shape)
    return KvPool(k_pool.data_ptr(), v_pool.data_ptr(), num_pages, page_size, H, D)


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ---- shapes.  The C ABI takes plain pointers and cannot see a buffer's size, so these checks
# are what keeps a wrongly shaped tensor from being read or written past its end on the device.
def _pool_shape(k_pool, v_pool, what: str = "pool"):
    if k_pool.dim() != 4 or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError(f"{what}: K and V must both be [num_pages, page_size, H, D], got "
                         f"{tuple(k_pool.shape)} and {tuple(v_pool.shape)}")
    return tuple(int(x) for x in k_pool.shape)


def _check_chunk_rows(wf: "WavefrontDesc", chunk: int, k, v, H: int, D: int):
    off = wf.chunk_offsets
    if not 0 <= int(chunk) < len(off) - 1:
        return                                     # the library answers WF_ERR_INVALID_ARG
    want = (off[chunk + 1] - off[chunk], H, D)
    for t, n in ((k, "k"), (v, "v")):
        if tuple(t.shape) != want and not (want[0] == 0 and t.numel() == 0):
            raise ValueError(f"{n}: chunk {chunk} needs [{want[0]}, {H}, {D}], got {tuple(t.shape)}")


def _check_page_table(page_table, layer: int, wf: "WavefrontDesc"):
    if page_table.dim() != 2 or page_table.shape[1] != wf.c.max_pages_per_seq:
        raise ValueError(f"page_table: expected [num_layers, {wf.c.max_pages_per_seq}], got "
                         f"{tuple(page_table.shape)}")
    if not 0 <= int(layer) < page_table.shape[0]:
        raise ValueError(f"layer {layer} outside the page table's {page_table.shape[0]} rows")


def _check_page_table_row(row, wf: "WavefrontDesc"):
    if row.dim() != 1 or row.shape[0] < wf.c.max_pages_per_seq:
        raise ValueError(f"page_table_row: expected [{wf.c.max_pages_per_seq}], got "
                         f"{tuple(row.shape)}")


def _check_queries(q, out, lse, wf: "WavefrontDesc", H: int, D: int):
    off = wf.chunk_offsets
    t_q = off[-1] - off[wf.num_ctx_chunks] if 0 <= wf.num_ctx_chunks < len(off) else None
    if t_q is None:
        return                                     # the library answers WF_ERR_SHAPE
    if tuple(q.shape) != (t_q, H, D):
        raise ValueError(f"q: expected [{t_q}, {H}, {D}] (the query chunks' rows), got "
                         f"{tuple(q.shape)}")
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"out: expected {tuple(q.shape)}, got {tuple(out.shape)}")
    if lse is not None and tuple(lse.shape) != (H, t_q):
        raise ValueError(f"lse: expected [{H}, {t_q}], got {tuple(lse.shape)}")


def _check_tensor(t, name: str, dtype_name: str):
    import torch
    want = {"bf16": (torch.bfloat16,), "i32": (torch.int32,), "f32": (torch.float32,),
            "u8": (torch.uint8,), "i8": (torch.int8,), "f64": (torch.float64,),
            "u32": (torch.int32, torch.uint32)}[dtype_name]      # flag words: any 32-bit int
    if t.dtype not in want:
        raise TypeError(f"{name}: expected {want[0]}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def _check_qk_buffers(qk, fields, sizes):
    """Every buffer of an 8-bit tier's qk holds at least the bytes the library's sizes call
    gives for this wavefront (the quantize call writes them all, the attention call reads them)."""
    get = (lambda n: qk[n]) if isinstance(qk, dict) else (lambda n: getattr(qk, n))
    for n, sz in zip(fields, sizes):
        t = get(n)
        if t.numel() * t.element_size() < sz:
            raise ValueError(f"{n}: {t.numel() * t.element_size()} bytes, needs {sz}")


class Window:
    """Host copy of a wf_window_t; keeps the stage array alive while C reads it."""

    def __init__(self, chunk_len: int, stages: Sequence[int], history: int):
        self._stages = (ctypes.c_int32 * max(len(stages), 1))(*[int(s) for s in stages])
        self.c = WindowC(int(chunk_len), len(stages),
                         ctypes.cast(self._stages, ctypes.POINTER(ctypes.c_int32)), int(history))


def window_slots(window: Window):
    """wf_window_slots: (slots, tokens) of one layer of the window."""
    slots, tokens = ctypes.c_int32(), ctypes.c_int64()
    rc = lib.wf_window_slots(ctypes.byref(window.c), ctypes.byref(slots), ctypes.byref(tokens))
    if rc != WF_OK:
        raise WfError(rc, "wf_window_slots")
    return slots.value, tokens.value


def window_round(window: Window, round_index: int, ring: bool = False) -> RoundC:
    """wf_window_round (or, with ring, wf_window_round_ring): the plan of one round."""
    out = RoundC()
    fn = lib.wf_window_round_ring if ring else lib.wf_window_round
    rc = fn(ctypes.byref(window.c), int(round_index), ctypes.byref(out))
    if rc != WF_OK:
        raise WfError(rc, "wf_window_round_ring" if ring else "wf_window_round")
    return out


class Segments:
    """Host copy of a wf_segments_t; keeps the arrays alive while C reads them."""

    def __init__(self, rows_end: Sequence[int], kv_end: Sequence[int], num_keys: int,
                 max_pages_per_seq: int):
        n = len(rows_end)
        if n != len(kv_end):
            raise ValueError("rows_end and kv_end need one entry per segment")
        self._rows = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in rows_end])
        self._kv = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in kv_end])
        self.c = SegmentsC(n, ctypes.cast(self._rows, ctypes.POINTER(ctypes.c_int32)),
                           ctypes.cast(self._kv, ctypes.POINTER(ctypes.c_int32)),
                           int(num_keys), int(max_pages_per_seq))
        self.rows_end = [int(x) for x in rows_end]
        self.kv_end = [int(x) for x in kv_end]
        self.num_keys = int(num_keys)

    @property
    def t_q(self) -> int:
        return self.rows_end[-1] if self.rows_end else 0


def attn_segments_workspace_size(seg: Segments, num_heads: int, head_dim: int,
                                 splits: int = 0) -> int:
    return int(lib.wf_attn_segments_workspace_size(ctypes.byref(seg.c), int(num_heads),
                                                   int(head_dim), int(splits)))


def attn_forward_segments(q, k_pool, v_pool, page_table_row, seg: Segments, scale: float, out,
                          lse=None, splits: int = 1, workspace=None, stream=None) -> None:
    """wf_attn_forward_segments: rows of segment i see logical keys [0, kv_end[i])."""
    _, page_size, H, D = _pool_shape(k_pool, v_pool)
    t_q = seg.t_q
    if tuple(q.shape) != (t_q, H, D) or tuple(out.shape) != (t_q, H, D):
        raise ValueError(f"q, out: expected [{t_q}, {H}, {D}], got {tuple(q.shape)}, "
                         f"{tuple(out.shape)}")
    if lse is not None and tuple(lse.shape) != (H, t_q):
        raise ValueError(f"lse: expected [{H}, {t_q}], got {tuple(lse.shape)}")
    if page_table_row.dim() != 1 or page_table_row.numel() < seg.c.max_pages_per_seq:
        raise ValueError(f"page_table_row: needs {seg.c.max_pages_per_seq} entries")
    for t, n, d in ((q, "q", "bf16"), (out, "out", "bf16"), (k_pool, "k_pool", "bf16"),
                    (v_pool, "v_pool", "bf16"), (page_table_row, "page_table_row", "i32")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    need = attn_segments_workspace_size(seg, H, D, splits)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        raise ValueError(f"workspace: {need} bytes needed for {splits} key splits")
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_attn_forward_segments(
        q.data_ptr(), ctypes.byref(pool),
        ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(seg.c), float(scale), out.data_ptr(),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
        if lse is not None else None,
        int(splits), workspace.data_ptr() if workspace is not None else None,
        workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_segments")


def kv_append(k_pool, v_pool, layer: int, chunk: int, k, v, page_table, wf: WavefrontDesc,
              stream=None) -> None:
    """wf_kv_append: write chunk ``chunk``'s K/V ([L, H, D] bf16) into the pools' pages using row
    ``layer`` of ``page_table`` ([num_layers, max_pages_per_seq] int32, on the device)."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_chunk_rows(wf, chunk, k, v, H, D)
    _check_page_table(page_table, layer, wf)
    for t, n, d in ((k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"), (k, "k", "bf16"),
                    (v, "v", "bf16"), (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_kv_append(ctypes.byref(pool), int(layer), int(chunk), k.data_ptr(), v.data_ptr(),
                          ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                      ctypes.POINTER(ctypes.c_int32)),
                          ctypes.byref(wf.c), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_append")


def _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale):
    num_pages, page_size, H, D = _pool_shape(k_codes, v_codes, "FP8 pool codes")
    if tuple(k_scale.shape) != (num_pages, page_size, H) or \
            tuple(v_scale.shape) != (num_pages, page_size, H):
        raise ValueError("FP8 pool: codes [pages, page_size, H, D] and scales [pages, page_size, H]")
    return num_pages, page_size, H, D


def _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale) -> KvPoolFp8:
    num_pages, page_size, H, D = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    for t, n, d in ((k_codes, "k_codes", "u8"), (v_codes, "v_codes", "u8"),
                    (k_scale, "k_scale", "f32"), (v_scale, "v_scale", "f32")):
        _check_tensor(t, n, d)
    return KvPoolFp8(k_codes.data_ptr(), v_codes.data_ptr(), k_scale.data_ptr(),
                     v_scale.data_ptr(), num_pages, page_size, H, D)


def kv_append_fp8(k_codes, v_codes, k_scale, v_scale, layer: int, chunk: int, k, v, page_table,
                  wf: WavefrontDesc, stream=None) -> None:
    """wf_kv_append_fp8: quantize chunk ``chunk``'s K/V ([L, H, D] bf16) to e4m3 codes with one
    fp32 scale per (token, head) row, into an FP8 pool through row ``layer`` of ``page_table``."""
    _, _, H, D = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    _check_chunk_rows(wf, chunk, k, v, H, D)
    _check_page_table(page_table, layer, wf)
    for t, n, d in ((k, "k", "bf16"), (v, "v", "bf16"), (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    pool = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    rc = lib.wf_kv_append_fp8(ctypes.byref(pool), int(layer), int(chunk), k.data_ptr(),
                              v.data_ptr(), ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                                        ctypes.POINTER(ctypes.c_int32)),
                              ctypes.byref(wf.c), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_append_fp8")


def kv_dequant(k_codes, v_codes, k_scale, v_scale, k_pool, v_pool, layer: int, chunk: int,
               page_table, wf: WavefrontDesc, stream=None) -> None:
    """wf_kv_dequant: chunk ``chunk`` of an FP8 pool -> the same rows of a bf16 pool."""
    geo = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    if _pool_shape(k_pool, v_pool) != geo:
        raise ValueError(f"bf16 pool {tuple(k_pool.shape)} differs from the FP8 pool {geo}")
    _check_page_table(page_table, layer, wf)
    for t, n, d in ((k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    src = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    dst = _pool_struct(k_pool, v_pool)
    rc = lib.wf_kv_dequant(ctypes.byref(src), ctypes.byref(dst), int(layer), int(chunk),
                           ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                       ctypes.POINTER(ctypes.c_int32)),
                           ctypes.byref(wf.c), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_dequant")


def kv_append_fp8_chunks(k_codes, v_codes, k_scale, v_scale, layer: int, chunk_begin: int,
                         chunk_end: int, k, v, page_table, wf: WavefrontDesc, stream=None) -> None:
    """wf_kv_append_fp8_chunks: kv_append_fp8 of chunks [chunk_begin, chunk_end) in one launch;
    ``k``, ``v``: those chunks' rows in order, [L, H, D] bf16."""
    _, _, H, D = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    off = wf.chunk_offsets
    if 0 <= int(chunk_begin) < int(chunk_end) <= len(off) - 1:
        want = (off[chunk_end] - off[chunk_begin], H, D)
        for t, n in ((k, "k"), (v, "v")):
            if tuple(t.shape) != want and not (want[0] == 0 and t.numel() == 0):
                raise ValueError(f"{n}: chunks [{chunk_begin}, {chunk_end}) need "
                                 f"[{want[0]}, {H}, {D}], got {tuple(t.shape)}")
    _check_page_table(page_table, layer, wf)
    for t, n, d in ((k, "k", "bf16"), (v, "v", "bf16"), (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    pool = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    rc = lib.wf_kv_append_fp8_chunks(ctypes.byref(pool), int(layer), int(chunk_begin),
                                     int(chunk_end), k.data_ptr(), v.data_ptr(),
                                     ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                                 ctypes.POINTER(ctypes.c_int32)),
                                     ctypes.byref(wf.c), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_append_fp8_chunks")


def kv_dequant_chunks(k_codes, v_codes, k_scale, v_scale, k_pool, v_pool, layer: int,
                      chunk_begin: int, chunk_end: int, page_table, wf: WavefrontDesc,
                      stream=None) -> None:
    """wf_kv_dequant_chunks: kv_dequant of chunks [chunk_begin, chunk_end) in one launch."""
    geo = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    if _pool_shape(k_pool, v_pool) != geo:
        raise ValueError(f"bf16 pool {tuple(k_pool.shape)} differs from the FP8 pool {geo}")
    _check_page_table(page_table, layer, wf)
    for t, n, d in ((k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    src = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    dst = _pool_struct(k_pool, v_pool)
    rc = lib.wf_kv_dequant_chunks(ctypes.byref(src), ctypes.byref(dst), int(layer),
                                  int(chunk_begin), int(chunk_end),
                                  ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                              ctypes.POINTER(ctypes.c_int32)),
                                  ctypes.byref(wf.c), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_dequant_chunks")


def kv_append_publish_fp8(k_codes, v_codes, k_scale, v_scale, flags, peers, layer: int,
                          chunk: int, k, v, page_table, wf: WavefrontDesc, generation: int,
                          stream=None) -> None:
    """wf_kv_append_publish_fp8: quantize one chunk into this FP8 pool and every peer FP8 pool,
    then raise the chunk's flag to ``generation`` here (``flags``: device uint32
    [layers, WF_MAX_CHUNKS] or None) and in every peer.  ``peers``: sequence of
    (k_codes_ptr, v_codes_ptr, k_scale_ptr, v_scale_ptr, flags_ptr)."""
    _, _, H, D = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    _check_chunk_rows(wf, chunk, k, v, H, D)
    _check_page_table(page_table, layer, wf)
    if flags is not None and flags.numel() < (int(layer) + 1) * WF_MAX_CHUNKS:
        raise ValueError(f"flags: layer {layer} needs [>= {int(layer) + 1}, {WF_MAX_CHUNKS}] words, "
                         f"got {tuple(flags.shape)}")
    _check_tensor(page_table, "page_table", "i32")
    if k.numel() > 0:
        _check_tensor(k, "k", "bf16")
        _check_tensor(v, "v", "bf16")
    if flags is not None:
        _check_tensor(flags, "flags", "u32")
    arr = (Fp8Dst * max(1, len(peers)))(*[Fp8Dst(int(a), int(b), int(c), int(d),
                                                 int(f) if f else None)
                                          for a, b, c, d, f in peers])
    pool = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    rc = lib.wf_kv_append_publish_fp8(
        ctypes.byref(pool), flags.data_ptr() if flags is not None else None, arr, len(peers),
        int(layer), int(chunk), k.data_ptr() if k.numel() else None,
        v.data_ptr() if v.numel() else None,
        ctypes.cast(ctypes.c_void_p(page_table.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), int(generation) & 0xFFFFFFFF, _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_append_publish_fp8")


def kv_dequant_published(k_codes, v_codes, k_scale, v_scale, k_pool, v_pool, layer: int,
                         chunk: int, page_table, wf: WavefrontDesc, flags_row, generation: int,
                         stream=None) -> None:
    """wf_kv_dequant_published: kv_dequant that first waits for ``flags_row[chunk]`` (device
    uint32 [WF_MAX_CHUNKS]) to reach ``generation``."""
    geo = _fp8_pool_shape(k_codes, v_codes, k_scale, v_scale)
    if _pool_shape(k_pool, v_pool) != geo:
        raise ValueError(f"bf16 pool {tuple(k_pool.shape)} differs from the FP8 pool {geo}")
    _check_page_table(page_table, layer, wf)
    if flags_row.numel() < len(wf.chunk_offsets) - 1:
        raise ValueError(f"flags_row: needs >= {len(wf.chunk_offsets) - 1} words")
    for t, n, d in ((k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table, "page_table", "i32"), (flags_row, "flags_row", "u32")):
        _check_tensor(t, n, d)
    src = _fp8_pool_struct(k_codes, v_codes, k_scale, v_scale)
    dst = _pool_struct(k_pool, v_pool)
    rc = lib.wf_kv_dequant_published(ctypes.byref(src), ctypes.byref(dst), int(layer),
                                     int(chunk),
                                     ctypes.cast(ctypes.c_void_p(page_table.data_ptr()),
                                                 ctypes.POINTER(ctypes.c_int32)),
                                     ctypes.byref(wf.c), flags_row.data_ptr(),
                                     int(generation) & 0xFFFFFFFF, _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_dequant_published")


QK_I8_FIELDS = ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean", "k_sum")


def qk_i8_sizes(wf: WavefrontDesc, num_heads: int, head_dim: int):
    """wf_qk_i8_sizes: byte sizes of the six buffers of the INT8 tier, in QK_I8_FIELDS order."""
    sizes = (ctypes.c_size_t * 6)()
    rc = lib.wf_qk_i8_sizes(ctypes.byref(wf.c), int(num_heads), int(head_dim), sizes)
    if rc != WF_OK:
        raise WfError(rc, "wf_qk_i8_sizes")
    return [int(x) for x in sizes]


def _qk_struct(qk) -> QkI8:
    """qk: a mapping / object with the six QK_I8_FIELDS device tensors."""
    get = (lambda n: qk[n]) if isinstance(qk, dict) else (lambda n: getattr(qk, n))
    for n, d in zip(QK_I8_FIELDS, ("i8", "f32", "i8", "f32", "f32", "f64")):
        _check_tensor(get(n), n, d)
    return QkI8(*[get(n).data_ptr() for n in QK_I8_FIELDS])


def qk_quantize_i8(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc, qk,
                   stream=None) -> None:
    """wf_qk_quantize_i8: int8 Q (from q) and K' (from the K pool) with their scales into qk."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, q, None, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    _check_qk_buffers(qk, QK_I8_FIELDS, qk_i8_sizes(wf, H, D))
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32")):
        _check_tensor(t, n, d)
    pool = _pool_struct(k_pool, v_pool)
    s = _qk_struct(qk)
    rc = lib.wf_qk_quantize_i8(q.data_ptr(), ctypes.byref(pool),
                               ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()),
                                           ctypes.POINTER(ctypes.c_int32)),
                               ctypes.byref(wf.c), ctypes.byref(s), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_qk_quantize_i8")


def attn_forward_i8(qk, k_pool, v_pool, page_table_row, wf: WavefrontDesc, scale: float, out,
                    lse=None, stream=None) -> None:
    """wf_attn_forward_i8: block-causal attention on the quantized Q / K' of qk, V from v_pool."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(out, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    _check_qk_buffers(qk, QK_I8_FIELDS, qk_i8_sizes(wf, H, D))
    for t, n, d in ((out, "out", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    s = _qk_struct(qk)
    rc = lib.wf_attn_forward_i8(ctypes.byref(s), ctypes.byref(pool),
                                ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()),
                                            ctypes.POINTER(ctypes.c_int32)),
                                ctypes.byref(wf.c), float(scale), out.data_ptr(),
                                ctypes.cast(ctypes.c_void_p(lse.data_ptr()),
                                            ctypes.POINTER(ctypes.c_float))
                                if lse is not None else None,
                                _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_i8")


QK_E4M3_FIELDS = ("q_codes", "q_scale", "k_codes", "k_scale")


def qk_e4m3_sizes(wf: WavefrontDesc, num_heads: int, head_dim: int):
    """wf_qk_e4m3_sizes: byte sizes of the four buffers of the FP8 tier, in QK_E4M3_FIELDS
    order."""
    sizes = (ctypes.c_size_t * 4)()
    rc = lib.wf_qk_e4m3_sizes(ctypes.byref(wf.c), int(num_heads), int(head_dim), sizes)
    if rc != WF_OK:
        raise WfError(rc, "wf_qk_e4m3_sizes")
    return [int(x) for x in sizes]


def _qk_e4m3_struct(qk) -> QkE4m3:
    """qk: a mapping / object with the four QK_E4M3_FIELDS device tensors (codes uint8)."""
    get = (lambda n: qk[n]) if isinstance(qk, dict) else (lambda n: getattr(qk, n))
    for n, d in zip(QK_E4M3_FIELDS, ("u8", "f32", "u8", "f32")):
        _check_tensor(get(n), n, d)
    return QkE4m3(*[get(n).data_ptr() for n in QK_E4M3_FIELDS])


def qk_quantize_e4m3(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc, qk,
                     stream=None) -> None:
    """wf_qk_quantize_e4m3: e4m3 Q (from q) and K (from the K pool) with their scales into qk."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, q, None, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    _check_qk_buffers(qk, QK_E4M3_FIELDS, qk_e4m3_sizes(wf, H, D))
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32")):
        _check_tensor(t, n, d)
    pool = _pool_struct(k_pool, v_pool)
    s = _qk_e4m3_struct(qk)
    rc = lib.wf_qk_quantize_e4m3(q.data_ptr(), ctypes.byref(pool),
                                 ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()),
                                             ctypes.POINTER(ctypes.c_int32)),
                                 ctypes.byref(wf.c), ctypes.byref(s), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_qk_quantize_e4m3")


def attn_forward_e4m3(qk, k_pool, v_pool, page_table_row, wf: WavefrontDesc, scale: float, out,
                      lse=None, stream=None) -> None:
    """wf_attn_forward_e4m3: block-causal attention on the e4m3 Q / K of qk, V from v_pool."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(out, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    _check_qk_buffers(qk, QK_E4M3_FIELDS, qk_e4m3_sizes(wf, H, D))
    for t, n, d in ((out, "out", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    s = _qk_e4m3_struct(qk)
    rc = lib.wf_attn_forward_e4m3(ctypes.byref(s), ctypes.byref(pool),
                                  ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()),
                                              ctypes.POINTER(ctypes.c_int32)),
                                  ctypes.byref(wf.c), float(scale), out.data_ptr(),
                                  ctypes.cast(ctypes.c_void_p(lse.data_ptr()),
                                              ctypes.POINTER(ctypes.c_float))
                                  if lse is not None else None,
                                  _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_e4m3")


def attn_forward(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc, scale: float, out,
                 lse=None, stream=None) -> None:
    """wf_attn_forward: block-causal chunk attention of q ([T_q, H, D] bf16) over the paged K/V
    of one layer (``page_table_row``: [max_pages_per_seq] int32 on the device) into ``out``."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32"), (out, "out", "bf16")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_attn_forward(
        q.data_ptr(), ctypes.byref(pool),
        ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), float(scale), out.data_ptr(),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
        if lse is not None else None,
        _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward")


def attn_workspace_size(wf: WavefrontDesc, num_heads: int, head_dim: int, splits: int = 0) -> int:
    """wf_attn_workspace_size: bytes of workspace attn_forward_split needs (0: none)."""
    return int(lib.wf_attn_workspace_size(ctypes.byref(wf.c), int(num_heads), int(head_dim),
                                          int(splits)))


def attn_split_plan(wf: WavefrontDesc, num_heads: int, splits: int = 0, num_sms: int = 0):
    """wf_attn_split_plan: (parts, tail_units) -- every unit in ``parts`` parts, the last
    ``tail_units`` units of the dispatch order in parts + 1.  ``num_sms`` 0: the current device."""
    parts, tail = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = lib.wf_attn_split_plan(ctypes.byref(wf.c), int(num_heads), int(splits), int(num_sms),
                                ctypes.byref(parts), ctypes.byref(tail))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_split_plan")
    return parts.value, tail.value


def attn_forward_split(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc, scale: float, out,
                       splits: int = 0, workspace=None, lse=None, stream=None) -> None:
    """wf_attn_forward_split: attn_forward with every unit's keys split over ``splits`` CTAs
    (0: the library chooses) and merged; ``workspace`` is a device uint8 tensor of at least
    attn_workspace_size(...) bytes (None when that is 0)."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32"), (out, "out", "bf16")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_attn_forward_split(
        q.data_ptr(), ctypes.byref(pool),
        ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), float(scale), out.data_ptr(),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
        if lse is not None else None,
        int(splits), workspace.data_ptr() if workspace is not None else None,
        workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_split")


def attn_forward_split_noalloc(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc,
                               scale: float, out, splits: int = 0, lse=None, stream=None) -> None:
    """wf_attn_forward_split_noalloc: attn_forward_split with the library's static scratch
    instead of a workspace (calls on one device must be ordered on one stream)."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32"), (out, "out", "bf16")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_attn_forward_split_noalloc(
        q.data_ptr(), ctypes.byref(pool),
        ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), float(scale), out.data_ptr(),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
        if lse is not None else None,
        int(splits), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_split_noalloc")


def kv_append_publish(k_pool, v_pool, flags, peers, layer: int, chunk: int, k, v, page_table,
                      wf: WavefrontDesc, generation: int, stream=None) -> None:
    """wf_kv_append_publish: append one chunk into this pool and every peer pool, then raise the
    chunk's flag to ``generation`` here (``flags``: device uint32 [layers, WF_MAX_CHUNKS] or
    None) and in every peer.  ``peers``: sequence of (k_pool_ptr, v_pool_ptr, flags_ptr)."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_chunk_rows(wf, chunk, k, v, H, D)
    _check_page_table(page_table, layer, wf)
    if flags is not None and flags.numel() < (int(layer) + 1) * WF_MAX_CHUNKS:
        raise ValueError(f"flags: layer {layer} needs [>= {int(layer) + 1}, {WF_MAX_CHUNKS}] words, "
                         f"got {tuple(flags.shape)}")
    for t, n, d in ((k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table, "page_table", "i32")):
        _check_tensor(t, n, d)
    if k.numel() > 0:
        _check_tensor(k, "k", "bf16")
        _check_tensor(v, "v", "bf16")
    if flags is not None:
        _check_tensor(flags, "flags", "u32")
    arr = (PoolDst * max(1, len(peers)))(*[PoolDst(int(a), int(b), int(c) if c else None)
                                          for a, b, c in peers])
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_kv_append_publish(
        ctypes.byref(pool), flags.data_ptr() if flags is not None else None, arr, len(peers),
        int(layer), int(chunk), k.data_ptr() if k.numel() else None,
        v.data_ptr() if v.numel() else None,
        ctypes.cast(ctypes.c_void_p(page_table.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), int(generation) & 0xFFFFFFFF, _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_kv_append_publish")


def attn_forward_published(q, k_pool, v_pool, page_table_row, wf: WavefrontDesc, scale: float,
                           out, flags_row, generation: int, splits: int = 0, workspace=None,
                           lse=None, stream=None) -> None:
    """wf_attn_forward_published: attn_forward_split that waits, chunk by chunk, for the
    publication flags in ``flags_row`` (device uint32 [WF_MAX_CHUNKS]) to reach ``generation``."""
    _, _, H, D = _pool_shape(k_pool, v_pool)
    _check_queries(q, out, lse, wf, H, D)
    _check_page_table_row(page_table_row, wf)
    if flags_row.numel() < len(wf.chunk_offsets) - 1:
        raise ValueError(f"flags_row: one word per chunk needed, got {tuple(flags_row.shape)}")
    for t, n, d in ((q, "q", "bf16"), (k_pool, "k_pool", "bf16"), (v_pool, "v_pool", "bf16"),
                    (page_table_row, "page_table_row", "i32"), (out, "out", "bf16"),
                    (flags_row, "flags_row", "u32")):
        _check_tensor(t, n, d)
    if lse is not None:
        _check_tensor(lse, "lse", "f32")
    pool = _pool_struct(k_pool, v_pool)
    rc = lib.wf_attn_forward_published(
        q.data_ptr(), ctypes.byref(pool),
        ctypes.cast(ctypes.c_void_p(page_table_row.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
        ctypes.byref(wf.c), float(scale), out.data_ptr(),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
        if lse is not None else None,
        flags_row.data_ptr(), int(generation) & 0xFFFFFFFF, int(splits),
        workspace.data_ptr() if workspace is not None else None,
        workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_attn_forward_published")


def ipc_export(device_ptr: int):
    """wf_ipc_export: (64-byte IPC handle of the allocation holding ``device_ptr``, offset)."""
    buf = ctypes.create_string_buffer(64)
    off = ctypes.c_size_t()
    rc = lib.wf_ipc_export(ctypes.c_void_p(int(device_ptr)), buf, ctypes.byref(off))
    if rc != WF_OK:
        raise WfError(rc, "wf_ipc_export")
    return buf.raw, int(off.value)


def ipc_import(exported) -> int:
    """wf_ipc_import: map another process's (handle, offset); returns the device pointer here."""
    handle, offset = exported
    if len(handle) != 64:
        raise ValueError("an IPC handle has 64 bytes")
    out = ctypes.c_void_p()
    rc = lib.wf_ipc_import(ctypes.create_string_buffer(handle, 64), int(offset),
                           ctypes.byref(out))
    if rc != WF_OK:
        raise WfError(rc, "wf_ipc_import")
    return int(out.value)


def ipc_close(device_ptr: int) -> None:
    rc = lib.wf_ipc_close(ctypes.c_void_p(int(device_ptr)))
    if rc != WF_OK:
        raise WfError(rc, "wf_ipc_close")


def selftest_timeout(timeout_us: int, stream=None) -> None:
    """wf_selftest_timeout: make one bounded in-kernel wait run out (read it with check_status)."""
    rc = lib.wf_selftest_timeout(int(timeout_us), _stream_handle(stream))
    if rc != WF_OK:
        raise WfError(rc, "wf_selftest_timeout")


def check_status(stream=None) -> int:
    """wf_check_status: synchronise the stream and return (and clear) the first device error."""
    return int(lib.wf_check_status(_stream_handle(stream)))
