// wf_api.cu -- the C ABI (include/wf.h): host-side validation, TMA descriptors, launches and the
// per-device status word.  One translation unit holds every kernel of the library, so the device
// status/abort words below are plain module globals.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/wf.h"
#include "append_kernel.cuh"
#include "attn_kernel.cuh"
#include "attn_pair_kernel.cuh"

// First error any kernel of this library recorded on this device (0 = none); cleared by
// wf_check_status.
__device__ int g_wf_status = 0;
// Launch id of the last attention launch in which a bounded wait ran out; every other CTA of
// that launch stops as soon as it sees it.
__device__ unsigned g_wf_abort = 0;

#ifndef WF_ATTN_PAIR
#define WF_ATTN_PAIR 0
#endif

namespace {

constexpr int kMaxDevices = 64;
std::atomic<unsigned> g_launch_counter{1};

struct DeviceState {
  bool ready = false;
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
  if (!d.ready) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!d.ready) {
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
            cudaFuncSetAttribute(wfk::wf_attn_pair_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 wfk::PairSmem::ALLOC) != cudaSuccess) {
          cudaGetLastError();
          return WF_ERR_CUDA;
        }
      }
      d.ready = true;
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

int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
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
  int rc = validate_pool(kv_pages);
  if (rc) return rc;
  int t_kv = 0;
  rc = validate_wavefront(wf, kv_pages, &t_kv);
  if (rc) return rc;
  if (wf->num_ctx_chunks >= wf->num_chunks) return WF_ERR_SHAPE;   // no query chunk
  if (!(scale > 0.f) || !std::isfinite(scale)) return WF_ERR_INVALID_ARG;
  const int t_ctx = wf->chunk_offsets[wf->num_ctx_chunks];
  const int t_q = t_kv - t_ctx;
  if (t_q == 0) return WF_OK;
  if (q == nullptr || out == nullptr || page_table_row == nullptr || !aligned16(q) ||
      !aligned16(out) || (lse_or_null != nullptr && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return WF_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  rc = device_state(&d);
  if (rc) return rc;

  const int H = kv_pages->num_heads, D = kv_pages->head_dim, ps = kv_pages->page_size;
  static_assert(alignof(wfk::AttnParams) >= 64, "tensor maps need 64-byte alignment");
  wfk::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  // CTA pairs run head_dim 128; a box never crosses a page or a tile edge
  const bool use_pair = (D == 128) && WF_ATTN_PAIR;
  const int box_rows = gcd_int(ps, use_pair ? 64 : wfk::kBN);
  const int box_rows_v = gcd_int(ps, use_pair ? wfk::kPairBN : wfk::kBN);
  const int64_t total_rows = static_cast<int64_t>(kv_pages->num_pages) * ps;
  if (!encode_rows(&p.tm_q, q, D, H, t_q, wfk::kBM, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_rows(&p.tm_k, kv_pages->k_pool, D, H, total_rows, box_rows,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !encode_rows(&p.tm_v, kv_pages->v_pool, D, H, total_rows, box_rows_v,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return WF_ERR_CUDA;
  p.box_rows_v = box_rows_v;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse_or_null;
  p.page_table = page_table_row;
  p.status = d->status;
  p.grid_abort = d->abort_word;
  p.T_q = t_q;
  p.H = H;
  p.num_pages = kv_pages->num_pages;
  p.page_size = ps;
  p.total_rows = static_cast<int>(total_rows);
  p.box_rows = box_rows;
  p.n_pairs = (t_q + wfk::kNQT * wfk::kBM - 1) / (wfk::kNQT * wfk::kBM);
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.launch_id = g_launch_counter.fetch_add(1);
  if (p.launch_id == 0) p.launch_id = g_launch_counter.fetch_add(1);
  int nqc = 0;
  for (int c = wf->num_ctx_chunks; c < wf->num_chunks; ++c) {
    if (wf->chunk_offsets[c + 1] == wf->chunk_offsets[c]) continue;   // empty chunk: no rows
    p.qc_row_end[nqc] = wf->chunk_offsets[c + 1] - t_ctx;
    p.qc_kv_end[nqc] = wf->chunk_offsets[c + 1];
    ++nqc;
  }
  p.nqc = nqc;

  const int64_t grid = static_cast<int64_t>(p.n_pairs) * H;
  if (2 * grid > INT32_MAX) return WF_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_pair)
    wfk::wf_attn_pair_kernel<<<static_cast<unsigned>(2 * grid), wfk::kPairThreads,
                               wfk::PairSmem::ALLOC, s>>>(p);
  else if (D == 128)
    wfk::wf_attn_fwd_kernel<128><<<static_cast<unsigned>(grid), wfk::kAttnThreads,
                                   wfk::AttnSmem<128>::ALLOC, s>>>(p);
  else
    wfk::wf_attn_fwd_kernel<64><<<static_cast<unsigned>(grid), wfk::kAttnThreads,
                                  wfk::AttnSmem<64>::ALLOC, s>>>(p);
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
