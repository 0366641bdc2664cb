/*
 * wf.h -- C ABI of the B200 (sm_100a) block-causal chunk-attention library for Wave Forcing.
 *
 * Wave Forcing runs a DiT over a mixed-noise wavefront of video chunks.  Inside every Transformer
 * layer, the queries of each active chunk attend fully within their own chunk and, across chunks,
 * only to earlier, cleaner chunks -- the anchor, the clean history and earlier in-flight chunks --
 * and never to a later, noisier one (KipQuest summary of arXiv 2611.00859, "The deep dive",
 * paragraph on chunk-wise causal attention; project page, "01 The design gap", panel C).
 * The K/V of every chunk is published once per layer into fixed slots of the consumer's attention
 * buffer, and attention reads its visible prefix in place with no concatenation (project page,
 * "03 End-to-end KV transport", item 03 "Layout"; the README's "paged" exchange mode).  This
 * library holds those slots in fixed-size pages addressed through a page table.
 *
 * Logical order.  The K/V sequence of one layer is the chunks in order oldest (cleanest) first:
 * KV-only context chunks (anchor, clean history; stage 0), then the active chunks from the
 * cleanest to the noisiest.  Chunk c owns logical tokens [chunk_offsets[c], chunk_offsets[c+1]).
 * With this order the keys a query of chunk c may see are exactly the prefix
 * [0, chunk_offsets[c+1]).
 *
 * Paged layout.  K and V pools are bf16 arrays [num_pages][page_size][num_heads][head_dim]
 * (row-major, contiguous).  Logical token t of a layer lives in physical page
 * page_table_row[t / page_size] at row t % page_size.  Chunks are packed token-contiguously, so
 * one page may hold the tail of one chunk and the head of the next.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device memory on the current device; "host" pointers are
 *     read during the call only.  The caller owns every buffer; the library keeps no pointer after
 *     a call returns.
 *   - Calls are asynchronous on the given stream (0 = legacy default stream) and never
 *     synchronise, except wf_check_status.
 *   - Every call returns WF_OK (0) or an error code; nothing else crosses the ABI.  Argument
 *     errors are detected on the host before anything is launched.  Errors found by a kernel
 *     (a page index outside the pool, a bounded wait that ran out) are recorded in a per-device
 *     status word read by wf_check_status.
 *   - Attention computes in bf16 with fp32 accumulation; FP8 appears only in the K/V transport
 *     calls (wf_kv_append_fp8, wf_kv_dequant and their chunk-range forms).  Batch 1, one layer
 *     per call.
 */
#ifndef WF_H_
#define WF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* wf_stream_t; /* a cudaStream_t */

enum {
  WF_OK = 0,
  WF_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, layer/chunk index out of range, scale <= 0 */
  WF_ERR_SHAPE = 2,        /* head_dim not 64/128, page_size not a positive multiple of 16,
                              offsets not starting at 0 or decreasing, too many chunks, no query chunk */
  WF_ERR_STAGE_ORDER = 3,  /* chunk_stage decreases along the logical (oldest-first) order */
  WF_ERR_CAPACITY = 4,     /* the layer needs more pages than max_pages_per_seq */
  WF_ERR_PAGE_OOB = 5,     /* device: a page-table entry outside [0, num_pages); that page was not
                              written (append) or was read as page 0 (attention) */
  WF_ERR_TIMEOUT = 6,      /* device: a bounded wait inside a kernel ran out; the kernel stopped */
  WF_ERR_CUDA = 7,         /* a CUDA runtime or driver call failed */
  WF_ERR_NO_DEVICE = 8     /* no sm_100 device is current */
};

/* Maximum number of chunks (context + active) in one wavefront descriptor. */
#define WF_MAX_CHUNKS 64

/* One layer-independent K/V pool.  k_pool, v_pool: device bf16 [num_pages][page_size][H][D],
 * 16-byte aligned, caller-owned. */
typedef struct {
  void* k_pool;
  void* v_pool;
  int32_t num_pages;
  int32_t page_size;   /* tokens per page: a positive multiple of 16 */
  int32_t num_heads;
  int32_t head_dim;    /* 64 or 128 */
} wf_kv_pool_t;

/* The wavefront: which chunks exist, where their tokens sit, and their diffusion stage. */
typedef struct {
  int32_t num_chunks;          /* context + active, 1..WF_MAX_CHUNKS */
  int32_t num_ctx_chunks;      /* leading KV-only chunks; queries exist for chunks >= this */
  const int32_t* chunk_offsets;/* host [num_chunks+1]: token offsets in the logical sequence,
                                  [0] = 0, non-decreasing (an empty chunk is allowed) */
  const int32_t* chunk_stage;  /* host [num_chunks]: diffusion timestep, 0 = clean; must be
                                  non-decreasing in logical order (earlier = cleaner).  Validated
                                  only; the mask follows the logical order. */
  int32_t max_pages_per_seq;   /* row length of the page table */
} wf_wavefront_t;

/*
 * wf_kv_append -- publish one chunk's K/V of one layer into its pages.
 * Defining passage: project page, "03 End-to-end KV transport", item 03 "Layout" (each producer
 * writes straight into its fixed slot of the consumer's attention buffer); KipQuest "The deep
 * dive" (each replica publishes its keys and values right after projection, at every layer).
 *
 *   pool        K/V pools (device).
 *   layer       row of page_table to use, >= 0.
 *   chunk       chunk index in [0, wf->num_chunks).
 *   k, v        device bf16 [L][H][D], contiguous, 16-byte aligned, L = chunk length.
 *   page_table  device int32 [num_layers][max_pages_per_seq]; row `layer` maps logical pages of
 *               that layer to physical pages.
 *   wf          the wavefront (host).
 * Copies token i of the chunk to logical token chunk_offsets[chunk] + i, bit for bit.  Rows of a
 * page outside the chunk are not touched.  An entry outside [0, num_pages) is skipped and
 * recorded as WF_ERR_PAGE_OOB.  An empty chunk is a no-op.
 */
int wf_kv_append(const wf_kv_pool_t* pool, int layer, int chunk, const void* k, const void* v,
                 const int32_t* page_table, const wf_wavefront_t* wf, wf_stream_t stream);

/*
 * wf_attn_forward -- one block-causal chunk attention over the whole wavefront, one launch.
 * Defining passages: KipQuest "The deep dive" (within a chunk full; across chunks the anchor,
 * the clean history and every earlier, cleaner chunk, never a later, noisier one); project page
 * "01 The design gap" panel C; "03 End-to-end KV transport" item 03 (attention reads the prefix in
 * place).
 *
 *   q               device bf16 [T_q][H][D]: the query rows of chunks num_ctx_chunks..num_chunks-1
 *                   in order, T_q = chunk_offsets[num_chunks] - chunk_offsets[num_ctx_chunks].
 *   kv_pages        the K/V pools (device); every token in [0, chunk_offsets[num_chunks]) must
 *                   have been appended.  Rows past the last token may hold anything, NaN included.
 *   page_table_row  device int32 [max_pages_per_seq]: ONE layer's row.
 *   wf              the wavefront (host).
 *   scale           softmax scale (> 0), typically 1/sqrt(head_dim).
 *   out             device bf16 [T_q][H][D]: out[t,h,:] = sum_j softmax_j(scale q.k_j) v_j over
 *                   the keys j < chunk_offsets[c+1] of the query's chunk c.  fp32 accumulation,
 *                   P rounded to bf16 before P.V, output rounded to nearest even.
 *   lse_or_null     device fp32 [H][T_q] (optional): natural-log sum of exp of the scaled logits.
 * T_q = 0 is a no-op.
 */
int wf_attn_forward(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                    const wf_wavefront_t* wf, float scale, void* out, float* lse_or_null,
                    wf_stream_t stream);

/*
 * wf_attn_forward_split -- the same attention with every unit's key range split over several CTAs
 * (split-KV), for wavefronts with too few query rows to fill the GPU -- one Wave-Parallelism
 * rank's call, a single query chunk against a long prefix (project page, "02 Interactive
 * pipeline", "Inside one diffusion tick": the critical consumer sees 8 chunks).  Each of the S
 * CTAs of a unit computes a normalised partial output and log-sum-exp over its consecutive part
 * of the unit's key tiles; a second kernel merges them (out = sum_s exp(lse_s - lse) O_s).
 * Arguments and result as wf_attn_forward, plus:
 *   splits           S >= 1 key splits per unit (capped at 16 and at the key tiles of the
 *                    smallest unit), or 0 to let the library plan them from a model of the
 *                    grid (wf_attn_split_plan): S parts per unit, the last units of the
 *                    dispatch order possibly S + 1, so that the CTAs fill whole waves.
 *   workspace        device memory, 16-byte aligned, caller-owned, at least
 *                    wf_attn_workspace_size(wf, H, D, splits) bytes; may be null when that
 *                    size is 0 (S = 1 runs exactly wf_attn_forward's single pass).
 * Errors: as wf_attn_forward; WF_ERR_CAPACITY if workspace_bytes is too small; WF_ERR_INVALID_ARG
 * for splits < 0 or a null/misaligned workspace that is needed.  Two launches on `stream`; the
 * workspace must not be shared by calls that may run concurrently.
 */
int wf_attn_forward_split(const void* q, const wf_kv_pool_t* kv_pages,
                          const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                          void* out, float* lse_or_null, int splits, void* workspace,
                          size_t workspace_bytes, wf_stream_t stream);

/*
 * wf_attn_forward_split_noalloc -- wf_attn_forward_split without a caller workspace: the partial
 * results go to a static 128 MiB (134 217 728-byte) array the library keeps in device memory, one
 * per device, so the call allocates nothing.  No counterpart on the pages: it exists for callers
 * that cannot hand over device memory.  Arguments and result as wf_attn_forward_split without
 * `workspace` / `workspace_bytes`; WF_ERR_CAPACITY when the plan needs more than the 128 MiB
 * (P * T_q * H * (D + 1) * 4 bytes, P the plan's most parts; pass a smaller `splits` or use
 * wf_attn_forward_split).
 * Sharing: every call on a device uses the same array.  Calls that may run at the same time --
 * on different streams of one device, or from several host threads without ordering -- race on
 * it and may return wrong results; order them on one stream (the array is only read by the
 * merge kernel of the same call, which runs after the attention kernel on that stream).
 */
int wf_attn_forward_split_noalloc(const void* q, const wf_kv_pool_t* kv_pages,
                                  const int32_t* page_table_row, const wf_wavefront_t* wf,
                                  float scale, void* out, float* lse_or_null, int splits,
                                  wf_stream_t stream);

/*
 * wf_attn_workspace_size -- bytes of workspace wf_attn_forward_split needs for this wavefront,
 * head count, head_dim and `splits` (0: the library's choice on the current device):
 * P * T_q * H * (D + 1) * 4 bytes (fp32 partial outputs and log-sum-exps, each rounded up to 256)
 * with P the plan's largest part count, when some unit is split, else 0.  Also 0 for invalid
 * arguments (the forward call then reports the error).
 */
size_t wf_attn_workspace_size(const wf_wavefront_t* wf, int num_heads, int head_dim, int splits);

/*
 * wf_attn_split_plan -- the split plan wf_attn_forward_split uses for this wavefront and head
 * count: every unit (256 query rows x one head) in *parts parts, the last *tail_units units of the
 * dispatch order in *parts + 1.  splits > 0 gives that uniform plan (capped as above); 0 the
 * library's choice for num_sms SMs (0: the current device's).  Host-only when num_sms > 0.
 * Errors: WF_ERR_INVALID_ARG for null pointers or splits < 0; WF_ERR_SHAPE for an invalid
 * wavefront or one without query rows; WF_ERR_NO_DEVICE if num_sms is 0 and no sm_100 device is
 * current.
 */
int wf_attn_split_plan(const wf_wavefront_t* wf, int num_heads, int splits, int num_sms,
                       int32_t* parts, int32_t* tail_units);

/* ---------------------------------------------------------------------------------------------
 * One-way K/V publication between GPUs (Wave Parallelism).  Every GPU owns one chunk of the
 * wavefront and attends to the chunks before it; each producer writes its K/V, right after
 * projection, straight into the attention buffers of every consumer, one way (project page, "03
 * End-to-end KV transport", items 01-03; KipQuest "The deep dive").  Here all GPUs keep pools of
 * the same geometry with the same page table, so a chunk lands in the same pages everywhere, and
 * each pool has a flag array uint32 [num_layers][WF_MAX_CHUNKS] whose word (layer, chunk) holds
 * the generation of the chunk's last publication.  Peer pools and flags are reached through
 * pointers mapped with wf_ipc_import (or any other peer mapping); data moves by plain stores
 * from this GPU's SMs over NVLink, never by TMA loads from a peer.
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  void* k_pool;        /* device bf16 pool of the destination GPU, same geometry as the source */
  void* v_pool;
  uint32_t* flags;     /* that GPU's flag array [num_layers][WF_MAX_CHUNKS], or NULL */
} wf_pool_dst_t;

/*
 * wf_kv_append_publish -- wf_kv_append into `pool` and, in the same kernel, into every peer pool
 * (up to 8), then a second kernel sets word (layer, chunk) of `flags` (this GPU's flag array, may
 * be NULL) and of every peer's flags to `generation` with a system-scope release, after a
 * system-wide fence.  Arguments as wf_kv_append plus `flags`, `peers[num_peers]` and
 * `generation`.  An empty chunk only sets the flags.  Errors as wf_kv_append; WF_ERR_INVALID_ARG
 * for more than 8 peers or a null/misaligned peer pool.  Asynchronous on `stream`.
 */
int wf_kv_append_publish(const wf_kv_pool_t* pool, uint32_t* flags, const wf_pool_dst_t* peers,
                         int num_peers, int layer, int chunk, const void* k, const void* v,
                         const int32_t* page_table, const wf_wavefront_t* wf, uint32_t generation,
                         wf_stream_t stream);

/*
 * wf_attn_forward_published -- wf_attn_forward_split on chunks that other GPUs publish: before
 * loading the keys of chunk c the kernel waits until flags_row[c] has reached `generation`
 * (signed 32-bit difference >= 0, so generations may wrap), read with a system-scope acquire.
 * flags_row: device uint32 [WF_MAX_CHUNKS], this layer's row of this GPU's flag array; every
 * chunk the queries see (own chunk included) must be flagged, e.g. by wf_kv_append_publish.
 * A wait that lasts longer than 2 s stops the kernel and records WF_ERR_TIMEOUT (read with
 * wf_check_status).  Other arguments and errors as wf_attn_forward_split.
 */
int wf_attn_forward_published(const void* q, const wf_kv_pool_t* kv_pages,
                              const int32_t* page_table_row, const wf_wavefront_t* wf,
                              float scale, void* out, float* lse_or_null,
                              const uint32_t* flags_row, uint32_t generation, int splits,
                              void* workspace, size_t workspace_bytes, wf_stream_t stream);

/*
 * Query segments: attention whose rows carry their own key limit.  Segment i holds query rows
 * [rows_end[i-1], rows_end[i]) (rows_end[-1] = 0) and sees logical keys [0, kv_end[i]) of the
 * paged pool; rows_end must not decrease, kv_end must not decrease over the non-empty segments
 * and lie in [1, num_keys].  The wavefront descriptor is the special case where every query
 * chunk is a segment whose limit is its own end; segments also express a query chunk that is not
 * the last of its keys -- the store pass of a copy-free rolling window, whose rows see the whole
 * history ring although their own slot sits inside it (wf_window_round_ring).
 */
typedef struct {
  int32_t num_segments;        /* 1 .. WF_MAX_CHUNKS */
  const int32_t* rows_end;     /* host, [num_segments], cumulative query rows */
  const int32_t* kv_end;       /* host, [num_segments], visible keys of each segment's rows */
  int32_t num_keys;            /* logical keys the page table maps (>= every kv_end) */
  int32_t max_pages_per_seq;   /* entries of page_table_row */
} wf_segments_t;

/*
 * wf_attn_forward_segments -- wf_attn_forward_split on query segments.  q, out: bf16
 * [rows_end[last]][H][D]; lse_or_null fp32 [H][rows]; splits, workspace as
 * wf_attn_forward_split, sized by wf_attn_segments_workspace_size.  WF_ERR_SHAPE for limits that
 * decrease or exceed num_keys, WF_ERR_CAPACITY when num_keys needs more than max_pages_per_seq
 * pages; other errors as wf_attn_forward.  Asynchronous on `stream`.
 */
int wf_attn_forward_segments(const void* q, const wf_kv_pool_t* kv_pages,
                             const int32_t* page_table_row, const wf_segments_t* segments,
                             float scale, void* out, float* lse_or_null, int splits,
                             void* workspace, size_t workspace_bytes, wf_stream_t stream);
size_t wf_attn_segments_workspace_size(const wf_segments_t* segments, int num_heads, int head_dim,
                                       int splits);

/*
 * wf_ipc_export / wf_ipc_import / wf_ipc_close -- share device memory (pools, flag arrays)
 * between processes.  export writes the 64-byte IPC handle of the allocation containing
 * device_ptr (cudaIpcGetMemHandle on its base) and device_ptr's byte offset inside it; import
 * maps such a handle from another process with peer access enabled (cudaIpcOpenMemHandle) and
 * returns base + offset; close unmaps the allocation containing an imported pointer.
 * WF_ERR_CUDA on failure (e.g. a handle imported in the process that exported it).
 */
int wf_ipc_export(const void* device_ptr, void* handle64, size_t* offset);
int wf_ipc_import(const void* handle64, size_t offset, void** device_ptr);
int wf_ipc_close(void* device_ptr);

/*
 * FP8 K/V pages for transport (project page, "03 End-to-end KV transport", item 01 "Precision":
 * K/V sent in FP8 halve the bytes the producers move and are converted back before attention).
 * An FP8 pool has the geometry of a bf16 pool and is addressed through the same page table:
 * e4m3 codes (sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinities; largest finite
 * magnitude 448) in [num_pages][page_size][num_heads][head_dim] bytes, and one fp32 scale per
 * (token, head) row in [num_pages][page_size][num_heads].  A per-page scale is not used: two
 * chunks may share a page.  All four pointers are device memory owned by the caller, 16-byte
 * aligned.
 */
typedef struct {
  void* k_codes;
  void* v_codes;
  float* k_scale;
  float* v_scale;
  int32_t num_pages;
  int32_t page_size;   /* tokens per page: a positive multiple of 16 */
  int32_t num_heads;
  int32_t head_dim;    /* 64 or 128 */
} wf_kv_pool_fp8_t;

/*
 * wf_kv_append_fp8 -- wf_kv_append into an FP8 pool.  Each (token, head) row x of head_dim values,
 * with amax its largest magnitude, is stored as scale = amax / 448 and codes
 * e4m3(x * (448 / amax)), rounded to nearest even and saturated at +-448; both divisions and
 * the product are fp32 round-to-nearest.  A row of zeros stores scale 0 and zero codes, and so
 * does a row whose 448 / amax overflows fp32 (amax below about 1.3e-36); their codes keep the
 * values' signs.
 * Arguments and errors as wf_kv_append (k, v: device bf16 [L_c][H][D], 16-byte aligned).
 */
int wf_kv_append_fp8(const wf_kv_pool_fp8_t* pool, int layer, int chunk, const void* k,
                     const void* v, const int32_t* page_table, const wf_wavefront_t* wf,
                     wf_stream_t stream);

/*
 * wf_kv_dequant -- write chunk `chunk` of layer `layer` from the FP8 pool `src` into the bf16 pool
 * `dst` (same geometry, same page table): value = bf16_rne(decode(code) * scale).  Only that
 * chunk's rows of `dst` are written.  Errors as wf_kv_append; WF_ERR_SHAPE if the two pools'
 * geometries differ.  Attention then reads `dst` as usual.
 */
int wf_kv_dequant(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer, int chunk,
                  const int32_t* page_table, const wf_wavefront_t* wf, wf_stream_t stream);

/*
 * wf_kv_append_fp8_chunks / wf_kv_dequant_chunks -- wf_kv_append_fp8 / wf_kv_dequant of the
 * consecutive chunks [chunk_begin, chunk_end) in one launch: the same per-row quantization and
 * conversion, for chunks written or read together (a round's context, a whole layer).
 * k, v: the rows of those chunks in order, device bf16 [L][H][D] with L the sum of their
 * lengths.  Errors as the one-chunk calls; WF_ERR_INVALID_ARG if the range is empty, reversed
 * or outside the wavefront.
 */
int wf_kv_append_fp8_chunks(const wf_kv_pool_fp8_t* pool, int layer, int chunk_begin,
                            int chunk_end, const void* k, const void* v,
                            const int32_t* page_table, const wf_wavefront_t* wf,
                            wf_stream_t stream);
int wf_kv_dequant_chunks(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer,
                         int chunk_begin, int chunk_end, const int32_t* page_table,
                         const wf_wavefront_t* wf, wf_stream_t stream);

/*
 * FP8 publication (project page, "03 End-to-end KV transport", items 01 "Precision" and 03
 * "Layout": the producer sends each chunk's K/V in FP8 straight into the consumers' buffers,
 * which convert them back before attention).  The transport moves head_dim + 4 bytes per
 * (token, head) row of each tensor instead of 2 head_dim (0.516 x at head_dim 128).
 */
typedef struct {
  void* k_codes;       /* the destination GPU's FP8 pool, same geometry as the source */
  void* v_codes;
  float* k_scale;
  float* v_scale;
  uint32_t* flags;     /* that GPU's flag array [num_layers][WF_MAX_CHUNKS], or NULL */
} wf_fp8_dst_t;

/*
 * wf_kv_append_publish_fp8 -- wf_kv_append_fp8 into `pool` and, in the same kernel (the bf16
 * chunk is read and quantized once), into every peer's FP8 pool (up to 8, plain stores through
 * peer pointers), then raises word (layer, chunk) of `flags` (may be NULL) and of every peer's
 * flags to `generation` as wf_kv_append_publish does: after a system-wide fence, with a
 * system-scope release, and not at all when a row of the chunk has a page outside the pool
 * (WF_ERR_PAGE_OOB is then recorded).  Errors as wf_kv_append_fp8; WF_ERR_INVALID_ARG for more
 * than 8 peers or a null/misaligned peer pointer.  Asynchronous on `stream`.
 */
int wf_kv_append_publish_fp8(const wf_kv_pool_fp8_t* pool, uint32_t* flags,
                             const wf_fp8_dst_t* peers, int num_peers, int layer, int chunk,
                             const void* k, const void* v, const int32_t* page_table,
                             const wf_wavefront_t* wf, uint32_t generation, wf_stream_t stream);

/*
 * wf_kv_dequant_published -- wf_kv_dequant of a chunk another GPU publishes into `src`: every
 * block first waits until flags_row[chunk] has reached `generation` (signed 32-bit difference
 * >= 0, system-scope acquire), then converts.  flags_row: device uint32 [WF_MAX_CHUNKS], this
 * layer's row of this GPU's flag array.  A wait longer than 2 s records WF_ERR_TIMEOUT (read with
 * wf_check_status) and writes nothing.  A plain wf_attn_forward on `dst`, later on the same
 * stream, then reads the chunk.  Other arguments and errors as wf_kv_dequant.
 */
int wf_kv_dequant_published(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer,
                            int chunk, const int32_t* page_table, const wf_wavefront_t* wf,
                            const uint32_t* flags_row, uint32_t generation, wf_stream_t stream);

/*
 * INT8 attention tier (Sage-like).  The pages name SageAttention with W8A8 as the fast attention
 * backend (GitHub README, results table, "Sage . causal . paged" rows; KipQuest abstract) and give
 * no internals; the tier built here, in two calls:
 *   wf_qk_quantize_i8  mu = mean of the layer's keys per (head, channel) over all T_kv tokens
 *                      (exact fp64 sum, fp64 division, one fp32 rounding); K' = fp32(K - mu),
 *                      which shifts every logit of a query row by one constant and so leaves the
 *                      softmax unchanged; then Q per (128 query rows, head) and K' per (128 keys,
 *                      head), counted from row / key 0, as int8 codes with scale = amax / 127:
 *                      code = clamp(round_half_even(x * (127 / amax)), -127, 127), fp32 steps
 *                      (a block of zeros, or one whose 127 / amax overflows, gets scale 0).
 *   wf_attn_forward_i8 the block-causal attention of wf_attn_forward with
 *                      S = scale * scale_q * scale_k * (Q_i8 . K_i8) -- an exact integer product
 *                      on the tensor core -- and P.V in bf16 over the unquantized V pages.
 * Head dimension 128 only (WF_ERR_SHAPE otherwise).  All buffers are caller-owned device memory,
 * sized by wf_qk_i8_sizes; codes are int8 [rows][H][D] with K' in logical key order (contiguous,
 * no page table), scales fp32 [H][ceil(rows / 128)].
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  void* q_codes;      /* int8 [T_q][H][128], 16-byte aligned */
  float* q_scale;     /* fp32 [H][ceil(T_q / 128)] */
  void* k_codes;      /* int8 [T_kv][H][128], logical key order, 16-byte aligned */
  float* k_scale;     /* fp32 [H][ceil(T_kv / 128)] */
  float* k_mean;      /* fp32 [H][128], 16-byte aligned */
  double* k_sum;      /* fp64 [H][128] scratch, 8-byte aligned */
} wf_qk_i8_t;

/* Byte sizes of the six wf_qk_i8_t buffers, in field order, for a wavefront of num_heads heads.
 * WF_ERR_SHAPE unless head_dim is 128. */
int wf_qk_i8_sizes(const wf_wavefront_t* wf, int num_heads, int head_dim, size_t sizes[6]);

/* Quantize q (bf16 [T_q][H][128], the query rows of the wavefront) and the layer's keys (the K
 * pool through page_table_row, all T_kv tokens) into `qk`.  Errors as wf_attn_forward (a page
 * outside the pool: WF_ERR_PAGE_OOB from wf_check_status).  Asynchronous on `stream`. */
int wf_qk_quantize_i8(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                      const wf_wavefront_t* wf, const wf_qk_i8_t* qk, wf_stream_t stream);

/* wf_attn_forward on quantized Q and K (filled by wf_qk_quantize_i8 for the same wavefront and
 * page table); V is read from kv_pages as in wf_attn_forward.  out, lse_or_null and errors as
 * wf_attn_forward; WF_ERR_INVALID_ARG for a null field of qk or unaligned codes.  The call reads
 * q_scale and k_scale as fp32 arrays: pass the struct the quantize call accepted (which checked
 * their 4-byte alignment) -- this call does not check it again.  Asynchronous on `stream`. */
int wf_attn_forward_i8(const wf_qk_i8_t* qk, const wf_kv_pool_t* kv_pages,
                       const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                       void* out, float* lse_or_null, wf_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * FP8 (e4m3) attention tier: the e4m3 twin of the INT8 tier, QK^T on tcgen05.mma kind::f8f6f4
 * (project page, "03 End-to-end KV transport", item 01 "Precision", measures K/V in FP8; the
 * pages give no scale granularity for attention operands, so the blocks are the INT8 tier's).
 *   wf_qk_quantize_e4m3  Q per (128 query rows, head) and K per (128 keys, head), counted from
 *                        row / key 0, as e4m3 codes with scale = amax / 448:
 *                        code = e4m3(x * (448 / amax)), fp32 steps, rounded to nearest even and
 *                        saturated at 448 (a block of zeros, or one whose 448 / amax overflows,
 *                        gets scale 0); no key smoothing.
 *   wf_attn_forward_e4m3 the block-causal attention of wf_attn_forward with
 *                        S = scale * scale_q * scale_k * (Q_e4m3 . K_e4m3), fp32 accumulation on
 *                        the tensor core, and P.V in bf16 over the unquantized V pages.
 * Head dimension 128 only (WF_ERR_SHAPE otherwise).  Buffers as the INT8 tier's first four, with
 * e4m3 codes (one byte each) in place of int8; sizes from wf_qk_e4m3_sizes.
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  void* q_codes;      /* e4m3 [T_q][H][128], 16-byte aligned */
  float* q_scale;     /* fp32 [H][ceil(T_q / 128)] */
  void* k_codes;      /* e4m3 [T_kv][H][128], logical key order, 16-byte aligned */
  float* k_scale;     /* fp32 [H][ceil(T_kv / 128)] */
} wf_qk_e4m3_t;

/* Byte sizes of the four wf_qk_e4m3_t buffers, in field order.  WF_ERR_SHAPE unless head_dim is
 * 128. */
int wf_qk_e4m3_sizes(const wf_wavefront_t* wf, int num_heads, int head_dim, size_t sizes[4]);

/* Quantize q (bf16 [T_q][H][128]) and the layer's keys (the K pool through page_table_row, all
 * T_kv tokens) into `qk`.  Errors as wf_qk_quantize_i8.  Asynchronous on `stream`. */
int wf_qk_quantize_e4m3(const void* q, const wf_kv_pool_t* kv_pages,
                        const int32_t* page_table_row, const wf_wavefront_t* wf,
                        const wf_qk_e4m3_t* qk, wf_stream_t stream);

/* wf_attn_forward on e4m3 Q and K (filled by wf_qk_quantize_e4m3 for the same wavefront and page
 * table); V is read from kv_pages.  out, lse_or_null and errors as wf_attn_forward_i8, and the
 * same rule for the scales: pass the struct the quantize call accepted. */
int wf_attn_forward_e4m3(const wf_qk_e4m3_t* qk, const wf_kv_pool_t* kv_pages,
                         const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                         void* out, float* lse_or_null, wf_stream_t stream);

/*
 * Rolling context window: the plan of one round of a stream (host only, no device work).
 *
 * The pages' rules:
 *   - Round t of a stream has its active cells on a diagonal that advances one chunk per round:
 *     chunk c enters at round c, is on denoising step t - c at round t, and gets its store pass
 *     (a forward pass at the clean timestep whose K/V become history) at round c + num_stages.
 *   - A chunk sees the anchor, the clean history, the live store and every earlier, cleaner chunk
 *     in flight, and never a later, noisier one (KipQuest summary of arXiv 2611.00859, "The deep
 *     dive").
 *
 * Readings taken here:
 *   - The anchor is the first chunk stored; it is kept for the whole stream.
 *   - The history is the `history` most recently stored chunks after the anchor.
 *   - Every chunk has chunk_len tokens.
 *
 * Layout.  Every layer uses one fixed page table over
 * slots = 1 + history + 1 + num_stages chunk slots of chunk_len tokens:
 *   [anchor][history ring][live store][in flight, cleanest first].
 *
 * Order and placement:
 *   - Anchor and history keep their slots.  Every query sees all of them, so their order does not
 *     matter, and the history is a ring: slot 1 + (c - 1) mod history for stored chunk c >= 1.
 *   - The store chunk and the chunks in flight are appended every round right after the last
 *     occupied history slot.
 *   - While the ring fills, the store chunk already sits in its own ring slot.
 *   - Once the ring is full, the store chunk's K/V must also be appended into slot `store_to` (the
 *     slot of the chunk that leaves, `evicted`) after the round's attention at that layer.
 *
 * Slot i holds logical tokens [i * chunk_len, (i + 1) * chunk_len), so a round's chunk_offsets and
 * chunk_stage can be passed straight into a wf_wavefront_t (num_chunks, num_ctx_chunks likewise).
 */
enum { WF_ROLE_ANCHOR = 0, WF_ROLE_HISTORY = 1, WF_ROLE_STORE = 2, WF_ROLE_ACTIVE = 3 };

typedef struct {
  int32_t chunk_len;        /* tokens per chunk, >= 1 */
  int32_t num_stages;       /* denoising steps = in-flight positions, >= 1 */
  const int32_t* stages;    /* host [num_stages]: timesteps, noisiest first, > 0, strictly decreasing */
  int32_t history;          /* clean-history chunks kept after the anchor, >= 0 */
} wf_window_t;

typedef struct {
  int64_t round;
  int32_t num_chunks;                          /* occupied slots, in logical order */
  int32_t num_ctx_chunks;                      /* anchor + history: K/V only this round */
  int64_t chunk_id[WF_MAX_CHUNKS];             /* stream index of the chunk in each slot */
  int32_t role[WF_MAX_CHUNKS];                 /* WF_ROLE_* */
  int32_t chunk_stage[WF_MAX_CHUNKS];          /* 0 for anchor, history, store */
  int32_t chunk_offsets[WF_MAX_CHUNKS + 1];
  int32_t store_to;                            /* slot for the store hand-over, or -1 */
  int64_t evicted;                             /* chunk leaving the history after the round, or -1 */
  int32_t store_kv_end;                        /* keys the store pass's rows see, or -1 */
} wf_round_t;

/*
 * wf_window_slots -- slots and tokens one layer of the window occupies (pages needed:
 * ceil(tokens / page_size)).  WF_ERR_INVALID_ARG for null pointers, WF_ERR_SHAPE for a window that
 * breaks the rules above, needs more than WF_MAX_CHUNKS slots or more than INT32_MAX tokens.
 */
int wf_window_slots(const wf_window_t* window, int32_t* slots, int64_t* tokens);

/*
 * wf_window_round -- the plan of round `round` (>= 0) into *out.  Errors as wf_window_slots;
 * WF_ERR_INVALID_ARG for a negative round.
 */
int wf_window_round(const wf_window_t* window, int64_t round, wf_round_t* out);

/*
 * wf_window_round_ring -- the copy-free plan of round `round`: the same stream, with the history
 * kept in a ring of history + 1 slots that also holds the store pass.
 *   [anchor][ring: history + 1 slots][in flight, cleanest first]
 * The store pass writes its chunk once, straight into the ring slot it keeps as history: the slot
 * of the chunk that left the history at the end of the previous round (chunk c >= 1 lives in ring
 * slot 1 + (c - 1) mod (history + 1)).  Nothing is handed over after attention, so no slot is
 * written in the round in which another GPU may still read it.  The chunks in flight follow the
 * last occupied ring slot.  Slots are listed in slot order; the store pass's rows see the anchor
 * and the whole occupied ring (store_kv_end), every chunk in flight sees the slots up to its own.
 * Query rows run in slot order (store pass first), so the round is one wf_attn_forward_segments
 * call.  store_to is always -1; num_ctx_chunks counts the anchor and history slots.  Errors as
 * wf_window_round.
 */
int wf_window_round_ring(const wf_window_t* window, int64_t round, wf_round_t* out);

/*
 * wf_check_status -- synchronise `stream`, then return and clear the first error any kernel of
 * this library recorded on the current device since the last call (WF_OK if none).  A pending
 * CUDA error on the stream is returned as WF_ERR_CUDA.
 */
int wf_check_status(wf_stream_t stream);

/*
 * wf_selftest_timeout -- exercise the kernels' failure path without faulting anything: one CTA
 * waits, through the same bounded mbarrier wait the attention kernels use, on a barrier that no
 * thread will ever arrive on.  After `timeout_us` microseconds (1..1000000) the wait gives up,
 * records WF_ERR_TIMEOUT in the device status word and the kernel returns normally; the CUDA
 * context stays usable.  Asynchronous on `stream`; read the result with wf_check_status.
 * (No counterpart on the reference pages: it exists so the timeout path can be tested.)
 */
int wf_selftest_timeout(unsigned timeout_us, wf_stream_t stream);

/* wf_strerror -- a static, human-readable name for an error code. */
const char* wf_strerror(int code);

/* wf_version -- library version, major * 10000 + minor * 100 + patch. */
int wf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WF_H_ */
