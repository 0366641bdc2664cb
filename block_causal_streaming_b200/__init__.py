"""B200-native (sm_100a) block-causal chunk attention for Wave Forcing wavefronts.

The product is the C-ABI library ``libwf_b200.so`` (declared in ``include/wf.h``):

* ``wf_kv_append``    -- publish one chunk's layer-wise K/V into fixed-size pages;
* ``wf_attn_forward`` -- one block-causal attention over every chunk of the wavefront, one launch;
* ``wf_attn_forward_split`` -- the same with each unit's keys split over several CTAs and merged,
  for wavefronts with few query rows (one Wave-Parallelism rank's chunk against its prefix);
* ``wf_kv_append_publish`` / ``wf_attn_forward_published`` -- one-way publication of a chunk's
  K/V into other GPUs' pools with a generation flag, and attention that waits for the flags
  (:mod:`.wave` maps the peers' pools between processes);
* ``wf_kv_append_fp8`` / ``wf_kv_dequant`` -- a chunk's K/V as e4m3 codes with per-(token, head)
  scales (half the bytes to move), and their conversion back into the bf16 pool (``_chunks``:
  a run of consecutive chunks in one launch);
  ``wf_kv_append_publish_fp8`` / ``wf_kv_dequant_published`` publish those codes into other GPUs'
  FP8 pools with a generation flag, and convert a published chunk once its flag is up;
* ``wf_qk_quantize_i8`` / ``wf_attn_forward_i8`` -- the INT8 tier: smoothed int8 K and int8 Q
  with per-128-row scales, QK^T as an integer product on the tensor core;
  ``wf_qk_quantize_e4m3`` / ``wf_attn_forward_e4m3`` the FP8 tier: e4m3 Q and K with
  per-128-row scales, QK^T on the tensor core's 8-bit floating format.

This package is its thin Python binding (ctypes, argument marshalling only), a small helper that
owns the paged pools of one layer (:mod:`.layer`), the round-by-round planner of a streaming
window with an anchor and a rolling history (:mod:`.window`) and the seeded synthetic workloads
(:mod:`.workloads`).  The binding is loaded on first use of any of its names and fails loudly if
the library has not been built; there is no CPU fallback.
"""
_ABI_NAMES = (
    "WF_OK", "WF_ERR_INVALID_ARG", "WF_ERR_SHAPE", "WF_ERR_STAGE_ORDER", "WF_ERR_CAPACITY",
    "WF_ERR_PAGE_OOB", "WF_ERR_TIMEOUT", "WF_ERR_CUDA", "WF_ERR_NO_DEVICE", "WF_MAX_CHUNKS",
    "WavefrontDesc", "WfError", "attn_forward", "check_status", "kv_append", "strerror",
    "selftest_timeout", "attn_forward_split", "attn_workspace_size",
    "attn_forward_split_noalloc", "kv_append_publish", "attn_forward_published", "ipc_export",
    "ipc_import", "ipc_close", "PoolDst", "kv_append_fp8", "kv_dequant", "KvPoolFp8",
    "kv_append_fp8_chunks", "kv_dequant_chunks", "attn_split_plan", "qk_e4m3_sizes",
    "qk_quantize_e4m3", "attn_forward_e4m3", "QkE4m3",
    "kv_append_publish_fp8", "kv_dequant_published", "Fp8Dst", "qk_i8_sizes", "qk_quantize_i8",
    "attn_forward_i8", "QkI8", "Segments", "attn_forward_segments",
    "attn_segments_workspace_size",
)
__all__ = list(_ABI_NAMES)


def __getattr__(name):
    if name in _ABI_NAMES:
        from . import _abi
        return getattr(_abi, name)
    raise AttributeError(name)
