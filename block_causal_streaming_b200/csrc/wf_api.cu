// wf_api.cu -- the C ABI (include/wf.h): host-side validation, TMA descriptors, launches and the
// per-device status word.  One translation unit holds every kernel of the library, so the device
// status/abort words below are plain module globals.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>
#include <queue>

#include "../../include/wf.h"
#include "append_kernel.cuh"
#include "attn_kernel.cuh"
#include "combine_kernel.cuh"
#include "fp8_kernel.cuh"
#include "i8_kernel.cuh"
#include "publish_kernel.cuh"

// First error any kernel of this library recorded on this device (0 = none); cleared by
// wf_check_status.
__device__ int g_wf_status = 0;
// Launch id of the last attention launch in which a bounded wait ran out; every other CTA of
// that launch stops as soon as it sees it.
__device__ unsigned g_wf_abort = 0;

// Scratch of wf_attn_forward_split_noalloc: one static array per device, so that entry point
// needs no allocation.  128 MiB holds the partial results of the library's plan for a 4680-row,
// 12-head, head_dim-128 call -- 3 key splits, the last units 4 (4 x 4680 x 12 x 129 x 4 B =
// 115.9 MB); larger plans are rejected.
constexpr size_t kScratchBytes = size_t(128) << 20;
__device__ __align__(256) unsigned char g_wf_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<unsigned> g_launch_counter{1};

struct DeviceState {
  // Set (release) once the fields below are filled; read (acquire) without the lock.
  std::atomic<bool> ready{false};
  bool sm100 = false;
  int* status = nullptr;
  unsigned* abort_word = nullptr;
  int num_sms = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device set-up: architecture check, device addresses of the module globals, and the
// shared-memory opt-in of the attention kernels.
int device_state(DeviceState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return WF_ERR_NO_DEVICE;
  }
  DeviceState& d = g_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      cudaDeviceProp prop;
      if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
        cudaGetLastError();
        return WF_ERR_NO_DEVICE;
      }
      d.sm100 = (prop.major == 10 && prop.minor == 0);
      d.num_sms = prop.multiProcessorCount;
      if (d.sm100) {
        if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_wf_status) != cudaSuccess ||
            cudaGetSymbolAddress(reinterpret_cast<void**>(&d.abort_word), g_wf_abort) !=
                cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<128>::ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<64>::ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<128, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<128>::ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<64, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<64>::ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<128, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<128, true>::ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(wfk::wf_attn_fwd_kernel<128, false, true, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::AttnSmem<128, true>::ALLOC) != cudaSuccess) {
          cudaGetLastError();
          return WF_ERR_CUDA;
        }
      }
      d.ready.store(true, std::memory_order_release);
    }
  }
  if (!d.sm100) return WF_ERR_NO_DEVICE;
  *out = &d;
  return WF_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_pool(const wf_kv_pool_t* pool) {
  if (pool == nullptr || pool->k_pool == nullptr || pool->v_pool == nullptr) return WF_ERR_INVALID_ARG;
  if (!aligned16(pool->k_pool) || !aligned16(pool->v_pool)) return WF_ERR_INVALID_ARG;
  if (pool->num_pages < 1 || pool->num_heads < 1) return WF_ERR_SHAPE;
  if (pool->head_dim != 64 && pool->head_dim != 128) return WF_ERR_SHAPE;
  if (pool->page_size < 16 || pool->page_size % 16 != 0) return WF_ERR_SHAPE;
  // TMA coordinates and token indices are 32-bit
  if (static_cast<int64_t>(pool->num_pages) * pool->page_size > INT32_MAX) return WF_ERR_SHAPE;
  return WF_OK;
}

// Checks the descriptor against the pool; on success returns the total token count.
int validate_wavefront(const wf_wavefront_t* wf, const wf_kv_pool_t* pool, int* t_kv) {
  if (wf == nullptr || wf->chunk_offsets == nullptr || wf->chunk_stage == nullptr)
    return WF_ERR_INVALID_ARG;
  if (wf->num_chunks < 1 || wf->num_chunks > WF_MAX_CHUNKS) return WF_ERR_SHAPE;
  if (wf->num_ctx_chunks < 0 || wf->num_ctx_chunks > wf->num_chunks) return WF_ERR_SHAPE;
  const int32_t* off = wf->chunk_offsets;
  if (off[0] != 0) return WF_ERR_SHAPE;
  for (int c = 0; c < wf->num_chunks; ++c)
    if (off[c + 1] < off[c]) return WF_ERR_SHAPE;
  for (int c = 0; c + 1 < wf->num_chunks; ++c)
    if (wf->chunk_stage[c + 1] < wf->chunk_stage[c]) return WF_ERR_STAGE_ORDER;
  const int64_t total = off[wf->num_chunks];
  const int64_t pages = (total + pool->page_size - 1) / pool->page_size;
  if (wf->max_pages_per_seq < 0 || pages > wf->max_pages_per_seq) return WF_ERR_CAPACITY;
  *t_kv = static_cast<int>(total);
  return WF_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

typedef CUresult (*GetRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange from the driver, for the IPC helpers.
GetRangeFn get_range_fn() {
  static GetRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetRangeFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// bf16 tensor (D, H, rows) with row stride H*D, 128B swizzle, box (64, 1, box_rows).
bool encode_rows(CUtensorMap* map, const void* ptr, int D, int H, int64_t rows, int box_rows,
                 CUtensorMapL2promotion promo) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(H) * D * 2};
  const cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 tensor (D, H, rows) with row stride H*D bytes, 128B swizzle, box (128, 1, box_rows): the
// int8 Q and K' codes of the INT8 tier (D = 128 bytes per row).
bool encode_rows_u8(CUtensorMap* map, const void* ptr, int D, int H, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H) * D};
  const cuuint32_t box[3] = {128u, 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// ------------------------------------------------------------------------------ attention setup
// The query chunks of a wavefront: rows of query chunk i end at row_end[i] (query-row space) and
// see the first kv_end[i] keys.  Empty chunks own no rows and are skipped.
struct QueryPlan {
  int t_q = 0;
  int nqc = 0;
  int row_end[WF_MAX_CHUNKS];
  int kv_end[WF_MAX_CHUNKS];
};

int query_plan(const wf_wavefront_t* wf, QueryPlan* qp) {
  if (wf->chunk_offsets == nullptr || wf->num_chunks < 1 || wf->num_chunks > WF_MAX_CHUNKS ||
      wf->num_ctx_chunks < 0 || wf->num_ctx_chunks >= wf->num_chunks)
    return WF_ERR_SHAPE;
  const int32_t* off = wf->chunk_offsets;
  const int t_ctx = off[wf->num_ctx_chunks];
  qp->nqc = 0;
  for (int c = wf->num_ctx_chunks; c < wf->num_chunks; ++c) {
    if (off[c + 1] < off[c]) return WF_ERR_SHAPE;
    if (off[c + 1] == off[c]) continue;
    qp->row_end[qp->nqc] = off[c + 1] - t_ctx;
    qp->kv_end[qp->nqc] = off[c + 1];
    ++qp->nqc;
  }
  qp->t_q = off[wf->num_chunks] - t_ctx;
  return WF_OK;
}

constexpr int kUnitRows = wfk::kNQT * wfk::kBM;   // query rows per unit (one CTA)
constexpr int kMaxSplits = 16;

int num_pairs(const QueryPlan& qp) { return (qp.t_q + kUnitRows - 1) / kUnitRows; }

// Key tiles of the units of row block `pair` (the block's last row sees the most keys).
int unit_tiles(const QueryPlan& qp, int pair) {
  const int last = std::min((pair + 1) * kUnitRows, qp.t_q) - 1;
  int n = qp.kv_end[qp.nqc - 1];
  for (int c = 0; c < qp.nqc; ++c)
    if (last < qp.row_end[c]) { n = qp.kv_end[c]; break; }
  return (n + wfk::kBN - 1) / wfk::kBN;
}

// Heads per dispatch group: the fewest groups of at most kHeadsPerGroup heads that divide H
// evenly (one group -- plain heads-fastest order -- when none does).  Measured on a B200 (p50,
// 1.3B 5-step / 14B-shaped wavefronts): at most 1, 2, 3, 4, 6, 12 heads per group ->
// 2.85 / 21.4, 2.84 / 18.3, 2.80 / 18.1, 2.79 / 18.3-18.5, 2.79 / 18.7, 2.85 / 19.3-19.7 ms.
#ifndef WF_HEADS_PER_GROUP
#define WF_HEADS_PER_GROUP 4
#endif
constexpr int kHeadsPerGroup = WF_HEADS_PER_GROUP;
int head_group(int H) {
  for (int g = (H + kHeadsPerGroup - 1) / kHeadsPerGroup; g <= H / 2; ++g)
    if (H % g == 0 && H / g <= kHeadsPerGroup) return H / g;
  return H;
}

// Every split must own at least one key tile of every unit.
int max_splits(const QueryPlan& qp) {
  int m = kMaxSplits;
  for (int pr = 0; pr < num_pairs(qp); ++pr) m = std::min(m, unit_tiles(qp, pr));
  return std::max(m, 1);
}

size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// part_o: fp32 [S][T_q][H][D], then part_lse: fp32 [S][H][T_q] (S: the plan's most parts).
size_t split_workspace_bytes(const QueryPlan& qp, int H, int D, int S) {
  if (S <= 1) return 0;
  const size_t rows = static_cast<size_t>(S) * qp.t_q * H;
  return align256(rows * D * sizeof(float)) + align256(rows * sizeof(float));
}

// A split plan: every unit runs in S parts (CTAs over consecutive key tiles), the last `tail`
// units of the dispatch order in S + 1.
struct SplitPlan {
  int S = 1;
  int tail = 0;
  int parts() const { return tail > 0 ? S + 1 : S; }
};

// Length in tile-times of one launch under `plan`: CTAs in dispatch order go to the SM that
// frees first (the hardware's in-order block dispatch), each costing its key tiles plus a
// prologue/epilogue of kCtaOverhead tiles; a plan with parts adds the merge pass, about
// kMergePerPart tile-times per million (row, head, part) items.  (Calibrated on one
// Wave-Parallelism rank's call on a B200: ~3 us of prologue per CTA, ~1.3 us per tile, the
// merge of 3 x 4680 x 12 parts ~29 us.)
constexpr double kCtaOverhead = 2.5, kMergePerPart = 130.0;
double plan_cost(const QueryPlan& qp, int H, int num_sms, const SplitPlan& plan) {
  const int n_pairs = num_pairs(qp);
  const int hg = head_group(H);
  const int units = n_pairs * H;
  std::vector<double> sm(static_cast<size_t>(num_sms), 0.0);
  std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>,
                      std::greater<std::pair<double, int>>> free_at;
  for (int i = 0; i < num_sms; ++i) free_at.push({0.0, i});
  double makespan = 0.0, merge_items = 0.0;
  for (int u = 0; u < units; ++u) {
    const int in_group = u % (n_pairs * hg);
    const int pair = n_pairs - 1 - in_group / hg;
    const int n = unit_tiles(qp, pair);
    const int parts = u >= units - plan.tail ? plan.S + 1 : plan.S;
    const int rows = std::min((pair + 1) * kUnitRows, qp.t_q) - pair * kUnitRows;
    if (parts > 1) merge_items += static_cast<double>(rows) * parts;
    for (int s = 0; s < parts; ++s) {
      const int nk = static_cast<int>(static_cast<int64_t>(s + 1) * n / parts) -
                     static_cast<int>(static_cast<int64_t>(s) * n / parts);
      auto top = free_at.top();
      free_at.pop();
      const double end = top.first + nk + kCtaOverhead;
      makespan = std::max(makespan, end);
      free_at.push({end, top.second});
    }
  }
  return makespan + kMergePerPart * merge_items / 1e6;
}

// Key splits per unit, for grids shorter than two waves (one CTA per SM): of the plans with S
// parts per unit -- one part, or S >= 2 alone or with the last units given one part more so
// that the CTAs fill whole waves -- the one plan_cost finds shortest.  The choice is cached per query layout.
// (Measured on one Wave-Parallelism rank's call, 228 units on 148 SMs, uniform S = 1, 2, 3, 4,
// 5, 6, 16 -> 1.18, 1.22, 1.16, 1.27, 1.22, 1.32, 1.53 ms with an earlier kernel: tail waves
// cost about what this model predicts.)
SplitPlan auto_plan(const QueryPlan& qp, int H, int num_sms) {
  const int64_t units = static_cast<int64_t>(num_pairs(qp)) * H;
  SplitPlan best;
  if (units >= 2 * static_cast<int64_t>(num_sms) || units * kMaxSplits > INT32_MAX / 2)
    return best;
  struct Entry {
    QueryPlan qp;
    int H, sms;
    SplitPlan plan;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  auto same = [&](const Entry& e) {
    if (e.H != H || e.sms != num_sms || e.qp.t_q != qp.t_q || e.qp.nqc != qp.nqc) return false;
    for (int c = 0; c < qp.nqc; ++c)
      if (e.qp.row_end[c] != qp.row_end[c] || e.qp.kv_end[c] != qp.kv_end[c]) return false;
    return true;
  };
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (same(e)) return e.plan;
  }
  const int cap = max_splits(qp);
  double best_cost = plan_cost(qp, H, num_sms, best);
  for (int S = 1; S <= cap; ++S) {
    const int64_t ctas = units * S;
    const int64_t fill = (ctas + num_sms - 1) / num_sms * num_sms - ctas;
    for (const int64_t tail : {int64_t{0}, fill}) {
      // (a tail on S = 1 would mix whole and split units; every plan keeps all units split or
      // none)
      if (S == 1 || tail > units || (tail > 0 && S + 1 > cap)) continue;
      const SplitPlan cand{S, static_cast<int>(tail)};
      const double cost = plan_cost(qp, H, num_sms, cand);
      if (cost < best_cost) {
        best_cost = cost;
        best = cand;
      }
    }
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 32) cache.erase(cache.begin());
  cache.push_back({qp, H, num_sms, best});
  return best;
}

// The plan of a call: `splits` > 0 asks for that many parts in every unit (capped so that every
// part has a key tile); 0 lets the library choose.
SplitPlan plan_splits(const QueryPlan& qp, int H, int num_sms, int splits) {
  if (splits > 0) return SplitPlan{std::min(splits, max_splits(qp)), 0};
  return auto_plan(qp, H, num_sms);
}

// Device address of g_wf_scratch on the current device, looked up once per device.
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return WF_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr &&
      cudaGetSymbolAddress(&g_scratch_addr[dev], g_wf_scratch) != cudaSuccess) {
    cudaGetLastError();
    g_scratch_addr[dev] = nullptr;
    return WF_ERR_CUDA;
  }
  *out = g_scratch_addr[dev];
  return WF_OK;
}

// A validated attention launch.
struct AttnLaunch {
  alignas(64) wfk::AttnParams p;
  QueryPlan qp;
  DeviceState* d = nullptr;
  int D = 0;
  float* lse_out = nullptr;   // the caller's lse (written by the combine pass when split)
};

// The query plan of explicit segments: rows [rows_end[i-1], rows_end[i]) see keys [0, kv_end[i]).
int segments_plan(const wf_segments_t* seg, const wf_kv_pool_t* pool, QueryPlan* qp) {
  if (seg == nullptr || seg->rows_end == nullptr || seg->kv_end == nullptr)
    return WF_ERR_INVALID_ARG;
  if (seg->num_segments < 1 || seg->num_segments > WF_MAX_CHUNKS || seg->num_keys < 1)
    return WF_ERR_SHAPE;
  const int64_t pages = (static_cast<int64_t>(seg->num_keys) + pool->page_size - 1) /
                        pool->page_size;
  if (seg->max_pages_per_seq < 0 || pages > seg->max_pages_per_seq) return WF_ERR_CAPACITY;
  qp->nqc = 0;
  int prev_rows = 0, prev_kv = 1;
  for (int i = 0; i < seg->num_segments; ++i) {
    const int r = seg->rows_end[i], n = seg->kv_end[i];
    if (r < prev_rows) return WF_ERR_SHAPE;                          // rows run forward
    if (r == prev_rows) continue;                                    // an empty segment
    if (n < prev_kv || n > seg->num_keys) return WF_ERR_SHAPE;       // limits never decrease
    qp->row_end[qp->nqc] = r;
    qp->kv_end[qp->nqc] = n;
    ++qp->nqc;
    prev_rows = r;
    prev_kv = n;
  }
  qp->t_q = prev_rows;
  return WF_OK;
}

int prepare_common(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                   float scale, void* out, float* lse_or_null, AttnLaunch* L);

int prepare_attention(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                      const wf_wavefront_t* wf, float scale, void* out, float* lse_or_null,
                      AttnLaunch* L) {
  int rc = validate_pool(kv_pages);
  if (rc) return rc;
  int t_kv = 0;
  rc = validate_wavefront(wf, kv_pages, &t_kv);
  if (rc) return rc;
  if (wf->num_ctx_chunks >= wf->num_chunks) return WF_ERR_SHAPE;   // no query chunk
  rc = query_plan(wf, &L->qp);
  if (rc) return rc;
  return prepare_common(q, kv_pages, page_table_row, scale, out, lse_or_null, L);
}

// Everything after the query plan: checks of the pointers, tensor maps and kernel parameters.
int prepare_common(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                   float scale, void* out, float* lse_or_null, AttnLaunch* L) {
  int rc = WF_OK;
  if (!(scale > 0.f) || !std::isfinite(scale)) return WF_ERR_INVALID_ARG;
  wfk::AttnParams& p = L->p;
  std::memset(&p, 0, sizeof(p));
  const int t_q = L->qp.t_q;
  if (t_q == 0) return WF_OK;                                        // nothing to compute
  if (q == nullptr || out == nullptr || page_table_row == nullptr || !aligned16(q) ||
      !aligned16(out) || (lse_or_null != nullptr && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return WF_ERR_INVALID_ARG;
  rc = device_state(&L->d);
  if (rc) return rc;

  const int H = kv_pages->num_heads, D = kv_pages->head_dim, ps = kv_pages->page_size;
  static_assert(alignof(wfk::AttnParams) >= 64, "tensor maps need 64-byte alignment");
  L->D = D;
  // a box never crosses a page or a tile edge
  const int box_rows = gcd_int(ps, wfk::kBN);
  const int64_t total_rows = static_cast<int64_t>(kv_pages->num_pages) * ps;
  if (!encode_rows(&p.tm_q, q, D, H, t_q, wfk::kBM, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_rows(&p.tm_k, kv_pages->k_pool, D, H, total_rows, box_rows,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !encode_rows(&p.tm_v, kv_pages->v_pool, D, H, total_rows, box_rows,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return WF_ERR_CUDA;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse_or_null;
  L->lse_out = lse_or_null;
  p.page_table = page_table_row;
  p.status = L->d->status;
  p.grid_abort = L->d->abort_word;
  p.T_q = t_q;
  p.H = H;
  p.num_pages = kv_pages->num_pages;
  p.page_size = ps;
  p.total_rows = static_cast<int>(total_rows);
  p.box_rows = box_rows;
  p.n_pairs = num_pairs(L->qp);
  p.head_group = head_group(H);
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.nqc = L->qp.nqc;
  for (int c = 0; c < L->qp.nqc; ++c) {
    p.qc_row_end[c] = L->qp.row_end[c];
    p.qc_kv_end[c] = L->qp.kv_end[c];
  }
  p.n_splits = 1;
  if (static_cast<int64_t>(p.n_pairs) * H * kMaxSplits * 2 > INT32_MAX) return WF_ERR_SHAPE;
  return WF_OK;
}

// Point the launch at a workspace holding the plan's partial results.
void set_split_buffers(AttnLaunch* L, const SplitPlan& plan, void* workspace) {
  const size_t rows = static_cast<size_t>(plan.parts()) * L->qp.t_q * L->p.H;
  L->p.n_splits = plan.S;
  L->p.n_tail = plan.tail;
  L->p.part_o = static_cast<float*>(workspace);
  L->p.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           align256(rows * L->D * sizeof(float)));
}

int launch_attention(AttnLaunch* L, cudaStream_t s) {
  wfk::AttnParams& p = L->p;
  p.launch_id = g_launch_counter.fetch_add(1);
  if (p.launch_id == 0) p.launch_id = g_launch_counter.fetch_add(1);
  const int64_t grid = static_cast<int64_t>(p.n_pairs) * p.H * p.n_splits + p.n_tail;
  const unsigned g = static_cast<unsigned>(grid);
  const bool wait = p.flags != nullptr;
  if (L->D == 128 && !wait)
    wfk::wf_attn_fwd_kernel<128><<<g, wfk::kAttnThreads, wfk::AttnSmem<128>::ALLOC, s>>>(p);
  else if (L->D == 128)
    wfk::wf_attn_fwd_kernel<128, true><<<g, wfk::kAttnThreads, wfk::AttnSmem<128>::ALLOC, s>>>(
        p);
  else if (!wait)
    wfk::wf_attn_fwd_kernel<64><<<g, wfk::kAttnThreads, wfk::AttnSmem<64>::ALLOC, s>>>(p);
  else
    wfk::wf_attn_fwd_kernel<64, true><<<g, wfk::kAttnThreads, wfk::AttnSmem<64>::ALLOC, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return WF_ERR_CUDA;
  if (p.n_splits > 1 || p.n_tail > 0) {
    const int64_t threads = static_cast<int64_t>(p.T_q) * p.H * 32;
    const unsigned blocks =
        static_cast<unsigned>((threads + wfk::kCombineThreads - 1) / wfk::kCombineThreads);
    const wfk::CombinePlan cp{p.n_splits, p.n_tail, p.n_pairs, p.head_group, kUnitRows};
    if (L->D == 128)
      wfk::wf_combine_kernel<128><<<blocks, wfk::kCombineThreads, 0, s>>>(
          p.part_o, p.part_lse, cp, p.T_q, p.H, p.out, L->lse_out);
    else
      wfk::wf_combine_kernel<64><<<blocks, wfk::kCombineThreads, 0, s>>>(
          p.part_o, p.part_lse, cp, p.T_q, p.H, p.out, L->lse_out);
    if (cudaGetLastError() != cudaSuccess) return WF_ERR_CUDA;
  }
  return WF_OK;
}


// One CTA waits on a barrier nobody arrives on; the bounded wait must give up, record
// WF_ERR_TIMEOUT and return.
__global__ void wf_selftest_timeout_kernel(int* status, unsigned* grid_abort, unsigned launch_id,
                                           unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t never;
  __shared__ int cta_abort;
  if (threadIdx.x == 0) {
    cta_abort = 0;
    wfk::mbar_init(wfk::smem_u32(&never), 1);
    wfk::mbar_init_fence();
  }
  __syncthreads();
  const wfk::WaitCtx w{&cta_abort, grid_abort, status, launch_id, WF_ERR_TIMEOUT, timeout_ns};
  if (threadIdx.x == 0) (void)wfk::mbar_wait(wfk::smem_u32(&never), 0, w);
  __syncthreads();
}

}  // namespace

extern "C" {

int wf_version(void) { return 100; }

const char* wf_strerror(int code) {
  switch (code) {
    case WF_OK: return "WF_OK";
    case WF_ERR_INVALID_ARG: return "WF_ERR_INVALID_ARG: null/misaligned pointer or index out of range";
    case WF_ERR_SHAPE: return "WF_ERR_SHAPE: unsupported or inconsistent shape";
    case WF_ERR_STAGE_ORDER: return "WF_ERR_STAGE_ORDER: chunk stages decrease along the logical order";
    case WF_ERR_CAPACITY: return "WF_ERR_CAPACITY: more pages needed than max_pages_per_seq";
    case WF_ERR_PAGE_OOB: return "WF_ERR_PAGE_OOB: a page-table entry is outside the pool";
    case WF_ERR_TIMEOUT: return "WF_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    case WF_ERR_CUDA: return "WF_ERR_CUDA: a CUDA call failed";
    case WF_ERR_NO_DEVICE: return "WF_ERR_NO_DEVICE: no sm_100 device is current";
    default: return "unknown wf error code";
  }
}

int wf_kv_append(const wf_kv_pool_t* pool, int layer, int chunk, const void* k, const void* v,
                 const int32_t* page_table, const wf_wavefront_t* wf, wf_stream_t stream) {
  int rc = validate_pool(pool);
  if (rc) return rc;
  int t_kv = 0;
  rc = validate_wavefront(wf, pool, &t_kv);
  if (rc) return rc;
  if (layer < 0 || chunk < 0 || chunk >= wf->num_chunks || page_table == nullptr)
    return WF_ERR_INVALID_ARG;
  const int t0 = wf->chunk_offsets[chunk];
  const int rows = wf->chunk_offsets[chunk + 1] - t0;
  if (rows == 0) return WF_OK;
  if (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v)) return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  rc = device_state(&d);
  if (rc) return rc;
  const int vec_per_row = pool->num_heads * pool->head_dim * 2 / 16;
  const int32_t* row = page_table + static_cast<int64_t>(layer) * wf->max_pages_per_seq;
  const int warps_per_block = wfk::kAppendThreads / 32;
  int blocks = (rows + warps_per_block - 1) / warps_per_block;
  if (blocks > d->num_sms * 8) blocks = d->num_sms * 8;
  wfk::wf_append_kernel<<<blocks, wfk::kAppendThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(pool->k_pool),
      static_cast<uint4*>(pool->v_pool), row, t0, rows, vec_per_row, pool->page_size,
      pool->num_pages, d->status);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_attn_forward(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                    const wf_wavefront_t* wf, float scale, void* out, float* lse_or_null,
                    wf_stream_t stream) {
  AttnLaunch L;
  const int rc = prepare_attention(q, kv_pages, page_table_row, wf, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  return launch_attention(&L, reinterpret_cast<cudaStream_t>(stream));
}

size_t wf_attn_workspace_size(const wf_wavefront_t* wf, int num_heads, int head_dim, int splits) {
  QueryPlan qp;
  if (wf == nullptr || num_heads < 1 || (head_dim != 64 && head_dim != 128) || splits < 0 ||
      query_plan(wf, &qp) != WF_OK || qp.t_q == 0)
    return 0;
  int sms = 0;
  if (splits == 0) {
    DeviceState* d = nullptr;
    if (device_state(&d) != WF_OK) return 0;
    sms = d->num_sms;
  }
  const SplitPlan plan = plan_splits(qp, num_heads, sms, splits);
  return split_workspace_bytes(qp, num_heads, head_dim, plan.parts());
}

int wf_attn_split_plan(const wf_wavefront_t* wf, int num_heads, int splits, int num_sms,
                       int32_t* parts, int32_t* tail_units) {
  if (wf == nullptr || parts == nullptr || tail_units == nullptr || splits < 0 || num_heads < 1 ||
      num_sms < 0)
    return WF_ERR_INVALID_ARG;
  QueryPlan qp;
  if (query_plan(wf, &qp) != WF_OK || qp.t_q == 0) return WF_ERR_SHAPE;
  if (splits == 0 && num_sms == 0) {
    DeviceState* d = nullptr;
    const int rc = device_state(&d);
    if (rc) return rc;
    num_sms = d->num_sms;
  }
  const SplitPlan plan = plan_splits(qp, num_heads, num_sms, splits);
  *parts = plan.S;
  *tail_units = plan.tail;
  return WF_OK;
}

int wf_attn_forward_split(const void* q, const wf_kv_pool_t* kv_pages,
                          const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                          void* out, float* lse_or_null, int splits, void* workspace,
                          size_t workspace_bytes, wf_stream_t stream) {
  if (splits < 0) return WF_ERR_INVALID_ARG;
  AttnLaunch L;
  const int rc = prepare_attention(q, kv_pages, page_table_row, wf, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  const SplitPlan plan = plan_splits(L.qp, L.p.H, L.d->num_sms, splits);
  if (plan.parts() > 1) {
    const size_t need = split_workspace_bytes(L.qp, L.p.H, L.D, plan.parts());
    if (workspace == nullptr || !aligned16(workspace)) return WF_ERR_INVALID_ARG;
    if (workspace_bytes < need) return WF_ERR_CAPACITY;
    set_split_buffers(&L, plan, workspace);
  }
  return launch_attention(&L, reinterpret_cast<cudaStream_t>(stream));
}

int wf_attn_forward_segments(const void* q, const wf_kv_pool_t* kv_pages,
                             const int32_t* page_table_row, const wf_segments_t* segments,
                             float scale, void* out, float* lse_or_null, int splits,
                             void* workspace, size_t workspace_bytes, wf_stream_t stream) {
  if (splits < 0) return WF_ERR_INVALID_ARG;
  int rc = validate_pool(kv_pages);
  if (rc) return rc;
  AttnLaunch L;
  rc = segments_plan(segments, kv_pages, &L.qp);
  if (rc) return rc;
  rc = prepare_common(q, kv_pages, page_table_row, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  const SplitPlan plan = plan_splits(L.qp, L.p.H, L.d->num_sms, splits);
  if (plan.parts() > 1) {
    const size_t need = split_workspace_bytes(L.qp, L.p.H, L.D, plan.parts());
    if (workspace == nullptr || !aligned16(workspace)) return WF_ERR_INVALID_ARG;
    if (workspace_bytes < need) return WF_ERR_CAPACITY;
    set_split_buffers(&L, plan, workspace);
  }
  return launch_attention(&L, reinterpret_cast<cudaStream_t>(stream));
}

size_t wf_attn_segments_workspace_size(const wf_segments_t* segments, int num_heads, int head_dim,
                                       int splits) {
  QueryPlan qp;
  wf_kv_pool_t geo{nullptr, nullptr, 1, 16, num_heads, head_dim};
  if (segments == nullptr || num_heads < 1 || (head_dim != 64 && head_dim != 128) ||
      splits < 0)
    return 0;
  geo.page_size = 16;
  geo.num_pages = INT32_MAX / 16;
  wf_segments_t s = *segments;
  s.max_pages_per_seq = INT32_MAX;          // capacity is checked by the attention call
  if (segments_plan(&s, &geo, &qp) != WF_OK || qp.t_q == 0) return 0;
  int sms = 0;
  if (splits == 0) {
    DeviceState* d = nullptr;
    if (device_state(&d) != WF_OK) return 0;
    sms = d->num_sms;
  }
  const SplitPlan plan = plan_splits(qp, num_heads, sms, splits);
  return split_workspace_bytes(qp, num_heads, head_dim, plan.parts());
}

int wf_attn_forward_split_noalloc(const void* q, const wf_kv_pool_t* kv_pages,
                                  const int32_t* page_table_row, const wf_wavefront_t* wf,
                                  float scale, void* out, float* lse_or_null, int splits,
                                  wf_stream_t stream) {
  if (splits < 0) return WF_ERR_INVALID_ARG;
  AttnLaunch L;
  int rc = prepare_attention(q, kv_pages, page_table_row, wf, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  const SplitPlan plan = plan_splits(L.qp, L.p.H, L.d->num_sms, splits);
  if (plan.parts() > 1) {
    if (split_workspace_bytes(L.qp, L.p.H, L.D, plan.parts()) > kScratchBytes)
      return WF_ERR_CAPACITY;
    void* scratch = nullptr;
    rc = scratch_address(&scratch);
    if (rc) return rc;
    set_split_buffers(&L, plan, scratch);
  }
  return launch_attention(&L, reinterpret_cast<cudaStream_t>(stream));
}

int wf_kv_append_publish(const wf_kv_pool_t* pool, uint32_t* flags, const wf_pool_dst_t* peers,
                         int num_peers, int layer, int chunk, const void* k, const void* v,
                         const int32_t* page_table, const wf_wavefront_t* wf, uint32_t generation,
                         wf_stream_t stream) {
  int rc = validate_pool(pool);
  if (rc) return rc;
  int t_kv = 0;
  rc = validate_wavefront(wf, pool, &t_kv);
  if (rc) return rc;
  if (layer < 0 || chunk < 0 || chunk >= wf->num_chunks || page_table == nullptr ||
      num_peers < 0 || num_peers > wfk::kMaxPublishDst - 1 || (num_peers > 0 && peers == nullptr))
    return WF_ERR_INVALID_ARG;
  for (int i = 0; i < num_peers; ++i)
    if (peers[i].k_pool == nullptr || peers[i].v_pool == nullptr ||
        !aligned16(peers[i].k_pool) || !aligned16(peers[i].v_pool) ||
        (reinterpret_cast<uintptr_t>(peers[i].flags) & 3u))
      return WF_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(flags) & 3u) return WF_ERR_INVALID_ARG;
  const int t0 = wf->chunk_offsets[chunk];
  const int rows = wf->chunk_offsets[chunk + 1] - t0;
  if (rows > 0 && (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v)))
    return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  rc = device_state(&d);
  if (rc) return rc;
  wfk::PublishParams p;
  std::memset(&p, 0, sizeof(p));
  p.k = static_cast<const uint4*>(k);
  p.v = static_cast<const uint4*>(v);
  p.pt_row = page_table + static_cast<int64_t>(layer) * wf->max_pages_per_seq;
  p.status = d->status;
  p.token0 = t0;
  p.rows = rows;
  p.vec_per_row = pool->num_heads * pool->head_dim * 2 / 16;
  p.page_size = pool->page_size;
  p.num_pages = pool->num_pages;
  p.generation = generation;
  const size_t flag_at = static_cast<size_t>(layer) * WF_MAX_CHUNKS + chunk;
  p.n_dst = 1 + num_peers;
  p.dst[0] = {static_cast<uint4*>(pool->k_pool), static_cast<uint4*>(pool->v_pool),
              flags != nullptr ? flags + flag_at : nullptr};
  for (int i = 0; i < num_peers; ++i)
    p.dst[1 + i] = {static_cast<uint4*>(peers[i].k_pool), static_cast<uint4*>(peers[i].v_pool),
                    peers[i].flags != nullptr ? peers[i].flags + flag_at : nullptr};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (rows > 0) {
    const int warps_per_block = wfk::kPublishThreads / 32;
    int blocks = (rows + warps_per_block - 1) / warps_per_block;
    if (blocks > d->num_sms * 8) blocks = d->num_sms * 8;
    wfk::wf_publish_kernel<<<blocks, wfk::kPublishThreads, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return WF_ERR_CUDA;
  }
  wfk::wf_publish_flags_kernel<<<1, 32, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_attn_forward_published(const void* q, const wf_kv_pool_t* kv_pages,
                              const int32_t* page_table_row, const wf_wavefront_t* wf,
                              float scale, void* out, float* lse_or_null,
                              const uint32_t* flags_row, uint32_t generation, int splits,
                              void* workspace, size_t workspace_bytes, wf_stream_t stream) {
  if (splits < 0 || flags_row == nullptr || (reinterpret_cast<uintptr_t>(flags_row) & 3u))
    return WF_ERR_INVALID_ARG;
  AttnLaunch L;
  const int rc = prepare_attention(q, kv_pages, page_table_row, wf, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  const SplitPlan plan = plan_splits(L.qp, L.p.H, L.d->num_sms, splits);
  if (plan.parts() > 1) {
    const size_t need = split_workspace_bytes(L.qp, L.p.H, L.D, plan.parts());
    if (workspace == nullptr || !aligned16(workspace)) return WF_ERR_INVALID_ARG;
    if (workspace_bytes < need) return WF_ERR_CAPACITY;
    set_split_buffers(&L, plan, workspace);
  }
  L.p.flags = flags_row;
  L.p.flag_gen = generation;
  L.p.nchunks = wf->num_chunks;
  for (int c = 0; c < wf->num_chunks; ++c) L.p.chunk_end[c] = wf->chunk_offsets[c + 1];
  return launch_attention(&L, reinterpret_cast<cudaStream_t>(stream));
}

int wf_ipc_export(const void* device_ptr, void* handle64, size_t* offset) {
  if (device_ptr == nullptr || handle64 == nullptr || offset == nullptr) return WF_ERR_INVALID_ARG;
  // an IPC handle names a whole allocation: find its base (a pool may be a sub-range of a
  // larger block of the caller's allocator) and report where device_ptr sits inside it
  GetRangeFn range = get_range_fn();
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range == nullptr ||
      range(&base, &size, reinterpret_cast<CUdeviceptr>(device_ptr)) != CUDA_SUCCESS)
    return WF_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
  std::memcpy(handle64, &h, sizeof(h));
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(device_ptr) - base);
  return WF_OK;
}

int wf_ipc_import(const void* handle64, size_t offset, void** device_ptr) {
  if (handle64 == nullptr || device_ptr == nullptr) return WF_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle64, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  *device_ptr = static_cast<uint8_t*>(base) + offset;
  return WF_OK;
}

int wf_ipc_close(void* device_ptr) {
  if (device_ptr == nullptr) return WF_ERR_INVALID_ARG;
  GetRangeFn range = get_range_fn();
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range == nullptr ||
      range(&base, &size, reinterpret_cast<CUdeviceptr>(device_ptr)) != CUDA_SUCCESS)
    return WF_ERR_CUDA;
  if (cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  return WF_OK;
}

namespace {

int validate_pool_fp8(const wf_kv_pool_fp8_t* pool) {
  if (pool == nullptr || pool->k_codes == nullptr || pool->v_codes == nullptr ||
      pool->k_scale == nullptr || pool->v_scale == nullptr)
    return WF_ERR_INVALID_ARG;
  if (!aligned16(pool->k_codes) || !aligned16(pool->v_codes) || !aligned16(pool->k_scale) ||
      !aligned16(pool->v_scale))
    return WF_ERR_INVALID_ARG;
  // the same geometry rules as a bf16 pool
  wf_kv_pool_t g{pool->k_codes, pool->v_codes, pool->num_pages, pool->page_size, pool->num_heads,
                 pool->head_dim};
  return validate_pool(&g);
}

// Checks shared by the FP8 calls; on success *t0 / *rows are the chunk's token range and *row its
// page-table row.
int fp8_chunk_args(const wf_kv_pool_fp8_t* pool, int layer, int chunk, const int32_t* page_table,
                   const wf_wavefront_t* wf, int* t0, int* rows, const int32_t** row,
                   int chunk_end = -1) {
  int rc = validate_pool_fp8(pool);
  if (rc) return rc;
  wf_kv_pool_t g{pool->k_codes, pool->v_codes, pool->num_pages, pool->page_size, pool->num_heads,
                 pool->head_dim};
  int t_kv = 0;
  rc = validate_wavefront(wf, &g, &t_kv);
  if (rc) return rc;
  // chunks [chunk, end)
  const int end = chunk_end < 0 ? chunk + 1 : chunk_end;
  if (layer < 0 || chunk < 0 || end <= chunk || end > wf->num_chunks || page_table == nullptr)
    return WF_ERR_INVALID_ARG;
  *t0 = wf->chunk_offsets[chunk];
  *rows = wf->chunk_offsets[end] - *t0;
  *row = page_table + static_cast<int64_t>(layer) * wf->max_pages_per_seq;
  // the quantizer indexes its threads over the (token, head) rows of both tensors with 32-bit
  // integers
  if (8 * static_cast<int64_t>(*rows) * pool->num_heads >= (int64_t{1} << 30)) return WF_ERR_SHAPE;
  return WF_OK;
}

// Quantization: kQuantLanes threads per (token, head) row of each tensor.
int quant_blocks(const DeviceState* d, int rows, int heads) {
  const int64_t threads = 2 * wfk::kQuantLanes * static_cast<int64_t>(rows) * heads;
  const int64_t blocks = (threads + wfk::kFp8Threads - 1) / wfk::kFp8Threads;
  const int64_t cap = static_cast<int64_t>(d->num_sms) * 16;
  return static_cast<int>(blocks < cap ? blocks : cap);
}

// Dequantization: one warp per token.
int dequant_blocks(const DeviceState* d, int rows) {
  const int per_block = wfk::kFp8Threads / 32;
  const int64_t blocks = (static_cast<int64_t>(rows) + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(d->num_sms) * 8;   // 64 warps per SM in flight
  return static_cast<int>(blocks < cap ? blocks : cap);
}

}  // namespace

}  // extern "C"

namespace {

// Quantize one chunk into pool and the FP8 peers (shared by the append and the publication).
int launch_quant(const wf_kv_pool_fp8_t* pool, const wf_fp8_dst_t* peers, int num_peers,
                 int t0, int rows, const int32_t* row, const void* k, const void* v,
                 cudaStream_t s) {
  DeviceState* d = nullptr;
  const int rc = device_state(&d);
  if (rc) return rc;
  wfk::QuantParams p;
  std::memset(&p, 0, sizeof(p));
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.pt_row = row;
  p.status = d->status;
  p.token0 = t0;
  p.rows = rows;
  p.H = pool->num_heads;
  p.page_size = pool->page_size;
  p.num_pages = pool->num_pages;
  p.n_dst = 1 + num_peers;
  p.dst[0] = {static_cast<uint8_t*>(pool->k_codes), static_cast<uint8_t*>(pool->v_codes),
              pool->k_scale, pool->v_scale};
  for (int i = 0; i < num_peers; ++i)
    p.dst[1 + i] = {static_cast<uint8_t*>(peers[i].k_codes),
                    static_cast<uint8_t*>(peers[i].v_codes), peers[i].k_scale, peers[i].v_scale};
  const int blocks = quant_blocks(d, rows, pool->num_heads);
  if (pool->head_dim == 128)
    wfk::wf_quant_append_kernel<128><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  else
    wfk::wf_quant_append_kernel<64><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

// Dequantize one chunk; with flag != null every block first waits for it to reach `generation`.
int launch_dequant(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int t0, int rows,
                   const int32_t* row, const uint32_t* flag, uint32_t generation,
                   cudaStream_t s) {
  DeviceState* d = nullptr;
  const int rc = device_state(&d);
  if (rc) return rc;
  wfk::DequantParams p;
  std::memset(&p, 0, sizeof(p));
  p.k_codes = static_cast<const uint8_t*>(src->k_codes);
  p.v_codes = static_cast<const uint8_t*>(src->v_codes);
  p.k_scale = src->k_scale;
  p.v_scale = src->v_scale;
  p.k_pool = static_cast<__nv_bfloat16*>(dst->k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(dst->v_pool);
  p.pt_row = row;
  p.status = d->status;
  p.token0 = t0;
  p.rows = rows;
  p.H = src->num_heads;
  p.page_size = src->page_size;
  p.num_pages = src->num_pages;
  p.flag = flag;
  p.generation = generation;
  p.grid_abort = d->abort_word;
  p.launch_id = g_launch_counter.fetch_add(1);
  if (p.launch_id == 0) p.launch_id = g_launch_counter.fetch_add(1);
  const int blocks = dequant_blocks(d, rows);
  const bool wait = flag != nullptr;
  if (src->head_dim == 128 && !wait)
    wfk::wf_dequant_kernel<128, false><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  else if (src->head_dim == 128)
    wfk::wf_dequant_kernel<128, true><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  else if (!wait)
    wfk::wf_dequant_kernel<64, false><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  else
    wfk::wf_dequant_kernel<64, true><<<blocks, wfk::kFp8Threads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int same_geometry(const wf_kv_pool_fp8_t* a, const wf_kv_pool_t* b) {
  return b->num_pages == a->num_pages && b->page_size == a->page_size &&
         b->num_heads == a->num_heads && b->head_dim == a->head_dim;
}

}  // namespace

extern "C" {

int wf_kv_append_fp8(const wf_kv_pool_fp8_t* pool, int layer, int chunk, const void* k,
                     const void* v, const int32_t* page_table, const wf_wavefront_t* wf,
                     wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  const int rc = fp8_chunk_args(pool, layer, chunk, page_table, wf, &t0, &rows, &row);
  if (rc) return rc;
  if (rows == 0) return WF_OK;
  if (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v)) return WF_ERR_INVALID_ARG;
  return launch_quant(pool, nullptr, 0, t0, rows, row, k, v,
                      reinterpret_cast<cudaStream_t>(stream));
}

int wf_kv_append_publish_fp8(const wf_kv_pool_fp8_t* pool, uint32_t* flags,
                             const wf_fp8_dst_t* peers, int num_peers, int layer, int chunk,
                             const void* k, const void* v, const int32_t* page_table,
                             const wf_wavefront_t* wf, uint32_t generation, wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  int rc = fp8_chunk_args(pool, layer, chunk, page_table, wf, &t0, &rows, &row);
  if (rc) return rc;
  if (num_peers < 0 || num_peers > wfk::kMaxFp8Dst - 1 || (num_peers > 0 && peers == nullptr))
    return WF_ERR_INVALID_ARG;
  for (int i = 0; i < num_peers; ++i)
    if (peers[i].k_codes == nullptr || peers[i].v_codes == nullptr ||
        peers[i].k_scale == nullptr || peers[i].v_scale == nullptr ||
        !aligned16(peers[i].k_codes) || !aligned16(peers[i].v_codes) ||
        !aligned16(peers[i].k_scale) || !aligned16(peers[i].v_scale) ||
        (reinterpret_cast<uintptr_t>(peers[i].flags) & 3u))
      return WF_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(flags) & 3u) return WF_ERR_INVALID_ARG;
  if (rows > 0 && (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v)))
    return WF_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (rows > 0) {
    rc = launch_quant(pool, peers, num_peers, t0, rows, row, k, v, s);
    if (rc) return rc;
  }
  // the generation flags, released once every row is written (the kernel of the bf16 path)
  wfk::PublishParams fp;
  std::memset(&fp, 0, sizeof(fp));
  fp.pt_row = row;
  fp.token0 = t0;
  fp.rows = rows;
  fp.page_size = pool->page_size;
  fp.num_pages = pool->num_pages;
  fp.generation = generation;
  const size_t flag_at = static_cast<size_t>(layer) * WF_MAX_CHUNKS + chunk;
  fp.n_dst = 1 + num_peers;
  fp.dst[0].flag = flags != nullptr ? flags + flag_at : nullptr;
  for (int i = 0; i < num_peers; ++i)
    fp.dst[1 + i].flag = peers[i].flags != nullptr ? peers[i].flags + flag_at : nullptr;
  wfk::wf_publish_flags_kernel<<<1, 32, 0, s>>>(fp);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_kv_append_fp8_chunks(const wf_kv_pool_fp8_t* pool, int layer, int chunk_begin,
                            int chunk_end, const void* k, const void* v,
                            const int32_t* page_table, const wf_wavefront_t* wf,
                            wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  if (chunk_end <= chunk_begin) return WF_ERR_INVALID_ARG;
  const int rc = fp8_chunk_args(pool, layer, chunk_begin, page_table, wf, &t0, &rows, &row,
                                chunk_end);
  if (rc) return rc;
  if (rows == 0) return WF_OK;
  if (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v)) return WF_ERR_INVALID_ARG;
  return launch_quant(pool, nullptr, 0, t0, rows, row, k, v,
                      reinterpret_cast<cudaStream_t>(stream));
}

int wf_kv_dequant_chunks(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer,
                         int chunk_begin, int chunk_end, const int32_t* page_table,
                         const wf_wavefront_t* wf, wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  if (chunk_end <= chunk_begin) return WF_ERR_INVALID_ARG;
  int rc = fp8_chunk_args(src, layer, chunk_begin, page_table, wf, &t0, &rows, &row, chunk_end);
  if (rc) return rc;
  rc = validate_pool(dst);
  if (rc) return rc;
  if (!same_geometry(src, dst)) return WF_ERR_SHAPE;
  if (rows == 0) return WF_OK;
  return launch_dequant(src, dst, t0, rows, row, nullptr, 0,
                        reinterpret_cast<cudaStream_t>(stream));
}

int wf_kv_dequant(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer, int chunk,
                  const int32_t* page_table, const wf_wavefront_t* wf, wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  int rc = fp8_chunk_args(src, layer, chunk, page_table, wf, &t0, &rows, &row);
  if (rc) return rc;
  rc = validate_pool(dst);
  if (rc) return rc;
  if (!same_geometry(src, dst)) return WF_ERR_SHAPE;
  if (rows == 0) return WF_OK;
  return launch_dequant(src, dst, t0, rows, row, nullptr, 0,
                        reinterpret_cast<cudaStream_t>(stream));
}

int wf_kv_dequant_published(const wf_kv_pool_fp8_t* src, const wf_kv_pool_t* dst, int layer,
                            int chunk, const int32_t* page_table, const wf_wavefront_t* wf,
                            const uint32_t* flags_row, uint32_t generation, wf_stream_t stream) {
  int t0 = 0, rows = 0;
  const int32_t* row = nullptr;
  int rc = fp8_chunk_args(src, layer, chunk, page_table, wf, &t0, &rows, &row);
  if (rc) return rc;
  rc = validate_pool(dst);
  if (rc) return rc;
  if (!same_geometry(src, dst)) return WF_ERR_SHAPE;
  if (flags_row == nullptr || (reinterpret_cast<uintptr_t>(flags_row) & 3u))
    return WF_ERR_INVALID_ARG;
  if (rows == 0) return WF_OK;
  return launch_dequant(src, dst, t0, rows, row, flags_row + chunk, generation,
                        reinterpret_cast<cudaStream_t>(stream));
}

int wf_qk_i8_sizes(const wf_wavefront_t* wf, int num_heads, int head_dim, size_t sizes[6]) {
  if (wf == nullptr || sizes == nullptr || num_heads < 1 || head_dim != 128 ||
      wf->chunk_offsets == nullptr || wf->num_chunks < 1 || wf->num_chunks > WF_MAX_CHUNKS ||
      wf->num_ctx_chunks < 0 || wf->num_ctx_chunks >= wf->num_chunks)
    return head_dim != 128 && wf != nullptr && sizes != nullptr ? WF_ERR_SHAPE
                                                                 : WF_ERR_INVALID_ARG;
  const int64_t t_kv = wf->chunk_offsets[wf->num_chunks];
  const int64_t t_q = t_kv - wf->chunk_offsets[wf->num_ctx_chunks];
  const int64_t hd = static_cast<int64_t>(num_heads) * head_dim;
  sizes[0] = static_cast<size_t>(t_q * hd);                                       // q_codes
  sizes[1] = static_cast<size_t>(num_heads * ((t_q + 127) / 128)) * sizeof(float);  // q_scale
  sizes[2] = static_cast<size_t>(t_kv * hd);                                      // k_codes
  sizes[3] = static_cast<size_t>(num_heads * ((t_kv + 127) / 128)) * sizeof(float); // k_scale
  sizes[4] = static_cast<size_t>(hd) * sizeof(float);                             // k_mean
  sizes[5] = static_cast<size_t>(hd) * sizeof(double);                            // k_sum
  return WF_OK;
}

int wf_qk_quantize_i8(const void* q, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                      const wf_wavefront_t* wf, const wf_qk_i8_t* qk, wf_stream_t stream) {
  int rc = validate_pool(kv_pages);
  if (rc) return rc;
  if (kv_pages->head_dim != 128) return WF_ERR_SHAPE;
  int t_kv = 0;
  rc = validate_wavefront(wf, kv_pages, &t_kv);
  if (rc) return rc;
  if (wf->num_ctx_chunks >= wf->num_chunks) return WF_ERR_SHAPE;
  const int t_q = t_kv - wf->chunk_offsets[wf->num_ctx_chunks];
  if (t_q == 0) return WF_OK;
  if (q == nullptr || qk == nullptr || page_table_row == nullptr || !aligned16(q) ||
      qk->q_codes == nullptr || qk->k_codes == nullptr || qk->q_scale == nullptr ||
      qk->k_scale == nullptr || qk->k_mean == nullptr || qk->k_sum == nullptr ||
      !aligned16(qk->q_codes) || !aligned16(qk->k_codes) || !aligned16(qk->k_mean) ||
      (reinterpret_cast<uintptr_t>(qk->k_sum) & 7u) ||
      (reinterpret_cast<uintptr_t>(qk->q_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(qk->k_scale) & 3u))
    return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  rc = device_state(&d);
  if (rc) return rc;
  const int H = kv_pages->num_heads, D = 128, cols = H * D;
  wfk::QkI8Params p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pool = static_cast<const __nv_bfloat16*>(kv_pages->k_pool);
  p.pt_row = page_table_row;
  p.q_codes = static_cast<int8_t*>(qk->q_codes);
  p.q_scale = qk->q_scale;
  p.k_codes = static_cast<int8_t*>(qk->k_codes);
  p.k_scale = qk->k_scale;
  p.k_mean = qk->k_mean;
  p.k_sum = qk->k_sum;
  p.status = d->status;
  p.T_q = t_q;
  p.T_kv = t_kv;
  p.H = H;
  p.page_size = kv_pages->page_size;
  p.num_pages = kv_pages->num_pages;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(qk->k_sum, 0, static_cast<size_t>(cols) * sizeof(double), s) != cudaSuccess)
    return WF_ERR_CUDA;
  int per = (t_kv + 4 * d->num_sms - 1) / (4 * d->num_sms);
  per = std::max(1, std::min(per, wfk::kKmeanMaxPer));
  wfk::wf_kmean_kernel<128><<<(t_kv + per - 1) / per, wfk::kKmeanThreads, 0, s>>>(p, per);
  wfk::wf_kmean_finalize<<<(cols + 255) / 256, 256, 0, s>>>(p, cols);
  wfk::wf_block_quant_kernel<128, true>
      <<<dim3((t_kv + wfk::kI8Block - 1) / wfk::kI8Block, H), wfk::kQuantI8Threads, 0, s>>>(p);
  wfk::wf_block_quant_kernel<128, false>
      <<<dim3((t_q + wfk::kI8Block - 1) / wfk::kI8Block, H), wfk::kQuantI8Threads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

}  // extern "C"

namespace {

// Attention over 8-bit Q and K codes with per-128-row scales (the INT8 or the FP8 tier).
int attn_forward_8bit(void* q_codes, const float* q_scale, void* k_codes, const float* k_scale,
                      bool e4m3, const wf_kv_pool_t* kv_pages, const int32_t* page_table_row,
                      const wf_wavefront_t* wf, float scale, void* out, float* lse_or_null,
                      wf_stream_t stream) {
  if (q_codes == nullptr || k_codes == nullptr || q_scale == nullptr || k_scale == nullptr ||
      !aligned16(k_codes))
    return WF_ERR_INVALID_ARG;
  if (kv_pages != nullptr && kv_pages->head_dim != 128) return WF_ERR_SHAPE;
  AttnLaunch L;
  int rc = prepare_attention(q_codes, kv_pages, page_table_row, wf, scale, out, lse_or_null, &L);
  if (rc || L.p.T_q == 0) return rc;
  wfk::AttnParams& p = L.p;
  const int t_kv = wf->chunk_offsets[wf->num_chunks];
  if (!encode_rows_u8(&p.tm_q, q_codes, 128, p.H, p.T_q, wfk::kBM) ||
      !encode_rows_u8(&p.tm_k, k_codes, 128, p.H, t_kv, wfk::kBN))
    return WF_ERR_CUDA;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.nqt = (p.T_q + wfk::kBM - 1) / wfk::kBM;
  p.nkb = (t_kv + wfk::kBN - 1) / wfk::kBN;
  p.launch_id = g_launch_counter.fetch_add(1);
  if (p.launch_id == 0) p.launch_id = g_launch_counter.fetch_add(1);
  const unsigned g = static_cast<unsigned>(static_cast<int64_t>(p.n_pairs) * p.H);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (e4m3)
    wfk::wf_attn_fwd_kernel<128, false, true, true>
        <<<g, wfk::kAttnThreads, wfk::AttnSmem<128, true>::ALLOC, s>>>(p);
  else
    wfk::wf_attn_fwd_kernel<128, false, true>
        <<<g, wfk::kAttnThreads, wfk::AttnSmem<128, true>::ALLOC, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

}  // namespace

extern "C" {

int wf_attn_forward_i8(const wf_qk_i8_t* qk, const wf_kv_pool_t* kv_pages,
                       const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                       void* out, float* lse_or_null, wf_stream_t stream) {
  if (qk == nullptr) return WF_ERR_INVALID_ARG;
  return attn_forward_8bit(qk->q_codes, qk->q_scale, qk->k_codes, qk->k_scale, false, kv_pages,
                           page_table_row, wf, scale, out, lse_or_null, stream);
}

int wf_attn_forward_e4m3(const wf_qk_e4m3_t* qk, const wf_kv_pool_t* kv_pages,
                         const int32_t* page_table_row, const wf_wavefront_t* wf, float scale,
                         void* out, float* lse_or_null, wf_stream_t stream) {
  if (qk == nullptr) return WF_ERR_INVALID_ARG;
  return attn_forward_8bit(qk->q_codes, qk->q_scale, qk->k_codes, qk->k_scale, true, kv_pages,
                           page_table_row, wf, scale, out, lse_or_null, stream);
}

int wf_qk_e4m3_sizes(const wf_wavefront_t* wf, int num_heads, int head_dim, size_t sizes[4]) {
  size_t all[6];
  const int rc = wf_qk_i8_sizes(wf, num_heads, head_dim, all);
  if (rc) return rc;
  for (int i = 0; i < 4; ++i) sizes[i] = all[i];
  return WF_OK;
}

int wf_qk_quantize_e4m3(const void* q, const wf_kv_pool_t* kv_pages,
                        const int32_t* page_table_row, const wf_wavefront_t* wf,
                        const wf_qk_e4m3_t* qk, wf_stream_t stream) {
  int rc = validate_pool(kv_pages);
  if (rc) return rc;
  if (kv_pages->head_dim != 128) return WF_ERR_SHAPE;
  int t_kv = 0;
  rc = validate_wavefront(wf, kv_pages, &t_kv);
  if (rc) return rc;
  if (wf->num_ctx_chunks >= wf->num_chunks) return WF_ERR_SHAPE;
  const int t_q = t_kv - wf->chunk_offsets[wf->num_ctx_chunks];
  if (t_q == 0) return WF_OK;
  if (q == nullptr || qk == nullptr || page_table_row == nullptr || !aligned16(q) ||
      qk->q_codes == nullptr || qk->k_codes == nullptr || qk->q_scale == nullptr ||
      qk->k_scale == nullptr || !aligned16(qk->q_codes) || !aligned16(qk->k_codes) ||
      (reinterpret_cast<uintptr_t>(qk->q_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(qk->k_scale) & 3u))
    return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  rc = device_state(&d);
  if (rc) return rc;
  const int H = kv_pages->num_heads;
  wfk::QkI8Params p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pool = static_cast<const __nv_bfloat16*>(kv_pages->k_pool);
  p.pt_row = page_table_row;
  p.q_codes = static_cast<int8_t*>(qk->q_codes);
  p.q_scale = qk->q_scale;
  p.k_codes = static_cast<int8_t*>(qk->k_codes);
  p.k_scale = qk->k_scale;
  p.status = d->status;
  p.T_q = t_q;
  p.T_kv = t_kv;
  p.H = H;
  p.page_size = kv_pages->page_size;
  p.num_pages = kv_pages->num_pages;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wfk::wf_block_quant_kernel<128, true, true>
      <<<dim3((t_kv + wfk::kI8Block - 1) / wfk::kI8Block, H), wfk::kQuantI8Threads, 0, s>>>(p);
  wfk::wf_block_quant_kernel<128, false, true>
      <<<dim3((t_q + wfk::kI8Block - 1) / wfk::kI8Block, H), wfk::kQuantI8Threads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_selftest_timeout(unsigned timeout_us, wf_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  const int rc = device_state(&d);
  if (rc) return rc;
  unsigned id = g_launch_counter.fetch_add(1);
  if (id == 0) id = g_launch_counter.fetch_add(1);
  wf_selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      d->status, d->abort_word, id, 1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_check_status(wf_stream_t stream) {
  DeviceState* d = nullptr;
  int rc = device_state(&d);
  if (rc) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  int st = 0;
  const int zero = 0;
  if (cudaMemcpy(&st, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(d->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  return st;
}

}  // extern "C"
