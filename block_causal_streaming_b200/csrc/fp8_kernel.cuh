// fp8_kernel.cuh -- FP8 (e4m3) K/V pages for transport (sm_100a).
//
// Wave Forcing sends K/V in FP8 to halve the bytes each producer moves, and converts them back
// before attention (project page, "03 End-to-end KV transport", item 01 "Precision": raw
// communication about 79 -> 40 ms in the 14B diagnostic).  Two HBM-bound kernels:
//
//   wf_quant_append_kernel  bf16 chunk rows [L][H][D] -> e4m3 codes in an FP8 pool
//                           [pages][page_size][H][D] plus one fp32 scale per (token, head) row
//                           in [pages][page_size][H], through the same page table as the bf16 pool;
//   wf_dequant_kernel       e4m3 codes + scales of one chunk -> the bf16 pool attention reads.
//
// Per (token, head) row of D values, with amax the largest magnitude:
//   inv = 448 / amax, scale = amax / 448 (fp32 divisions);
//   code = e4m3(x * inv) -- round to nearest even, saturating at +-448 (cvt.rn.satfinite);
//   dequantized value = bf16_rne(decode(code) * scale).
// A row of zeros, and a row so small that 448 / amax overflows fp32 (amax below about
// 1.3e-36), gets inv = scale = 0: its codes are signed zeros and it dequantizes to zeros.
// A per-page scale is not used because two chunks may share a page (their tokens are packed
// contiguously) and the page's first writer cannot know the second chunk's range.
//
// Quantization runs four threads per (token, head) row of one tensor (K rows first, then V rows):
// each holds a quarter of the row as 16-byte vectors, takes the largest magnitude with packed
// 16-bit integer maxima on the bf16 bit patterns (for values with the sign bit cleared the
// integer order is the float order), the row maximum is two shuffles, and the two divisions are
// paid once per row.  Dequantization runs one warp per token: every lane owns 8 consecutive
// values of one head row, so a warp's loads and stores are contiguous.  Page-table entries
// outside the pool are recorded as WF_ERR_PAGE_OOB and those rows are skipped.
//
// Publication: the quantizing kernel writes each token's codes and scales to up to 9 FP8 pools
// of the same geometry (this GPU's and up to 8 peers' mapped by IPC, plain stores over NVLink),
// so FP8 transport reads the bf16 chunk once and moves 0.516 x its bytes at head_dim 128.  The
// consumer's dequantization can wait (bounded) for the chunk's publication flag before it reads
// the codes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "sm100.cuh"

namespace wfk {

constexpr int kFp8Threads = 256;
constexpr int kMaxFp8Dst = 9;   // this GPU's pool + up to 8 peers
constexpr int kFp8Batch = 4;    // dequantization: warp-wide steps whose loads are in flight together

// Largest |x| of a row of bf16 values held as 32-bit words: packed 16-bit unsigned maxima of the
// bit patterns with the sign bits cleared, then the larger half, widened to fp32 (exact).
template <int W>
__device__ __forceinline__ float row_amax(const uint32_t (&w)[W]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < W; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
  const uint32_t top = max(m & 0xFFFFu, m >> 16);
  return __uint_as_float(top << 16);
}

// e4m3 codes of the 2 W bf16 values in w (value i in byte i of the result words), scaled by inv.
template <int W>
__device__ __forceinline__ void quantize_row(const uint32_t (&w)[W], float inv,
                                             uint32_t (&c)[W / 2]) {
#pragma unroll
  for (int i = 0; i < W / 2; ++i) {
    uint32_t half[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t u = w[2 * i + j];
      const float2 x = make_float2(__uint_as_float(u << 16) * inv,
                                   __uint_as_float(u & 0xFFFF0000u) * inv);
      half[j] = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);   // .x in the low byte
    }
    c[i] = (half[0] & 0xFFFFu) | (half[1] << 16);
  }
}

// 8 codes -> 8 bf16 values: decode (e4m3 -> fp16 is exact), times the scale in fp32, RNE to bf16.
__device__ __forceinline__ uint4 dequantize8(uint2 codes, float scale) {
  const uint32_t c[2] = {codes.x, codes.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_fp8x2_storage_t pair =
        static_cast<__nv_fp8x2_storage_t>((c[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
    const __half2 hv(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
    const float2 f = __half22float2(hv);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);   // .x: low half
    o[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Pool row (token slot * H + head) of row r = (t, h) of a chunk, or -1 -- recorded as
// WF_ERR_PAGE_OOB -- when the token's page is outside the pool.
__device__ __forceinline__ int64_t fp8_pool_row(const int* pt_row, int token0, int t, int h,
                                                int H, int page_size, int num_pages,
                                                int* status) {
  const int tok = token0 + t;
  const int pg = __ldg(pt_row + tok / page_size);
  if (pg < 0 || pg >= num_pages) {
    atomicCAS(status, 0, 5 /* WF_ERR_PAGE_OOB */);
    return -1;
  }
  return (static_cast<int64_t>(pg) * page_size + tok % page_size) * H + h;
}

// Pool token slot of token `tok` (lane 0 reads the page table; every lane gets the result), or -1
// (recorded as WF_ERR_PAGE_OOB) when its page is outside the pool.
__device__ __forceinline__ int64_t fp8_token_row(const int* pt_row, int tok, int page_size,
                                                 int num_pages, int lane, int* status) {
  int pg = 0;
  if (lane == 0) pg = __ldg(pt_row + tok / page_size);
  pg = __shfl_sync(0xffffffffu, pg, 0);
  if (pg < 0 || pg >= num_pages) {
    if (lane == 0) atomicCAS(status, 0, 5 /* WF_ERR_PAGE_OOB */);
    return -1;
  }
  return static_cast<int64_t>(pg) * page_size + tok % page_size;
}

struct Fp8Dst {
  uint8_t* k_codes;
  uint8_t* v_codes;
  float* k_scale;
  float* v_scale;
};

struct QuantParams {
  const __nv_bfloat16* k;          // chunk rows [rows][H][D]
  const __nv_bfloat16* v;
  const int* pt_row;               // this layer's page-table row
  int* status;
  int token0, rows, H, page_size, num_pages, n_dst;
  Fp8Dst dst[kMaxFp8Dst];          // pools of the same geometry, written identically
};

// kQuantLanes threads per (token, head) row of one tensor (K rows first, then V rows).  Thread
// `sub` of a row holds the row's 16-byte vectors kQuantLanes i + sub, so each load instruction
// reads 16 kQuantLanes contiguous bytes of every row a warp covers; the row maximum is
// log2(kQuantLanes) shuffles between adjacent lanes.
// Measured on the 1.3B 5-step layer (7 chunks, same box): 1, 2, 4 threads per row ->
// 0.155, 0.147, 0.136 ms for the quantizing leg.
constexpr int kQuantLanes = 4;

template <int D>
__global__ void __launch_bounds__(kFp8Threads)
    wf_quant_append_kernel(const __grid_constant__ QuantParams p) {
  constexpr int LPR = kQuantLanes;
  constexpr int NV = D / 8 / LPR;   // 16-byte vectors per thread
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(LPR == 1 || LPR == 2 || LPR == 4, "1, 2 or 4 threads per row");
  const int H = p.H;
  const int nrows = p.rows * H;                 // per tensor; the host keeps 2 LPR nrows < 2^31
  const int stride = gridDim.x * blockDim.x;
  // Warp-uniform loop (the shuffles below need every lane): lanes past the end, and rows whose
  // page is outside the pool, compute on zeros and store nothing.  The threads of a row are
  // adjacent lanes of one warp.
  for (int base = blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < 2 * LPR * nrows;
       base += stride) {
    const int i = base + (threadIdx.x & 31);
    const bool in = i < 2 * LPR * nrows;
    const int sub = i % LPR, rr = in ? i / LPR : 0;
    const bool is_v = rr >= nrows;
    const int r = is_v ? rr - nrows : rr;
    const uint4* src = reinterpret_cast<const uint4*>(is_v ? p.v : p.k) +
                       static_cast<int64_t>(r) * (D / 8) + sub;
    uint32_t w[4 * NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const uint4 x = in ? __ldg(src + LPR * j) : make_uint4(0, 0, 0, 0);
      w[4 * j] = x.x;
      w[4 * j + 1] = x.y;
      w[4 * j + 2] = x.z;
      w[4 * j + 3] = x.w;
    }
    const int t = r / H, h = r - t * H;
    const int64_t prow = in ? fp8_pool_row(p.pt_row, p.token0, t, h, H, p.page_size,
                                           p.num_pages, p.status)
                            : -1;
    float amax = row_amax(w);
#pragma unroll
    for (int o = 1; o < LPR; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float inv = 448.0f / amax;                        // IEEE division: these values decide codes
    const bool live = amax > 0.f && isfinite(inv);
    inv = live ? inv : 0.f;
    const float scale = live ? amax / 448.0f : 0.f;
    if (prow < 0) continue;                           // every thread of the row skips it
    uint32_t c[2 * NV];
    quantize_row(w, inv, c);
#pragma unroll 1
    for (int d = 0; d < p.n_dst; ++d) {
      uint2* dc = reinterpret_cast<uint2*>(is_v ? p.dst[d].v_codes : p.dst[d].k_codes) +
                  prow * (D / 8) + sub;
#pragma unroll
      for (int j = 0; j < NV; ++j) dc[LPR * j] = make_uint2(c[2 * j], c[2 * j + 1]);
      if (sub == 0) (is_v ? p.dst[d].v_scale : p.dst[d].k_scale)[prow] = scale;
    }
  }
}

struct DequantParams {
  const uint8_t* k_codes;          // FP8 pool
  const uint8_t* v_codes;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* k_pool;           // bf16 pool of the same geometry
  __nv_bfloat16* v_pool;
  const int* pt_row;
  int* status;
  int token0, rows, H, page_size, num_pages;
  // kWait: the chunk's publication flag, its generation, and the bounded-wait bookkeeping
  const unsigned* flag;
  unsigned generation;
  unsigned* grid_abort;
  unsigned launch_id;
};

// Loads of codes and scales: through the read-only path when the data was written before the
// launch; plain coherent loads when it was published by another GPU during it.
template <bool kNc, typename T>
__device__ __forceinline__ T fp8_load(const T* p) {
  if constexpr (kNc) return __ldg(p);
  else return *p;
}

// kWait: every block first waits (thread 0, system-scope acquire, 2 s bound) until the chunk's
// flag has reached the generation; a wait that runs out records WF_ERR_TIMEOUT, stops the other
// blocks through the grid abort word, and writes nothing.
template <int D, bool kWait>
__global__ void __launch_bounds__(kFp8Threads)
    wf_dequant_kernel(const __grid_constant__ DequantParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPS = 32 / LPR;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  if constexpr (kWait) {
    __shared__ int cta_abort;
    if (threadIdx.x == 0) {
      cta_abort = 0;
      const WaitCtx w{&cta_abort, p.grid_abort, p.status, p.launch_id, 6 /* WF_ERR_TIMEOUT */,
                      2000000000ull};
      if (!wait_flag(p.flag, p.generation, w)) cta_abort = 1;
    }
    __syncthreads();
    if (cta_abort) return;
  }
  const int H = p.H;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int steps = (H + RPS - 1) / RPS;
  const int warps = gridDim.x * (kFp8Threads / 32);
  for (int t = blockIdx.x * (kFp8Threads / 32) + (threadIdx.x >> 5); t < p.rows; t += warps) {
    const int64_t prow = fp8_token_row(p.pt_row, p.token0 + t, p.page_size, p.num_pages, lane,
                                       p.status);
    if (prow < 0) continue;
    const uint2* kc = reinterpret_cast<const uint2*>(p.k_codes + prow * H * D);
    const uint2* vc = reinterpret_cast<const uint2*>(p.v_codes + prow * H * D);
    uint4* kp = reinterpret_cast<uint4*>(p.k_pool + prow * H * D);
    uint4* vp = reinterpret_cast<uint4*>(p.v_pool + prow * H * D);
    for (int s0 = 0; s0 < steps; s0 += kFp8Batch) {
      uint2 ck[kFp8Batch], cv[kFp8Batch];
      float fk[kFp8Batch], fv[kFp8Batch];
#pragma unroll
      for (int b = 0; b < kFp8Batch; ++b) {
        const int h = (s0 + b) * RPS + rsub;
        if (h < H) {
          ck[b] = fp8_load<!kWait>(kc + h * LPR + sub);
          cv[b] = fp8_load<!kWait>(vc + h * LPR + sub);
          fk[b] = fp8_load<!kWait>(p.k_scale + prow * H + h);
          fv[b] = fp8_load<!kWait>(p.v_scale + prow * H + h);
        }
      }
#pragma unroll
      for (int b = 0; b < kFp8Batch; ++b) {
        const int h = (s0 + b) * RPS + rsub;
        if (h < H) {
          kp[h * LPR + sub] = dequantize8(ck[b], fk[b]);
          vp[h * LPR + sub] = dequantize8(cv[b], fv[b]);
        }
      }
    }
  }
}

}  // namespace wfk
