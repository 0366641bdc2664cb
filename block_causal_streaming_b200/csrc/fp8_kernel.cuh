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
// One warp per token: a token's H rows are contiguous both in the chunk and in the pool, so the
// warp walks them with 16-byte accesses -- every lane owns 8 consecutive values of one head row
// (D / 8 lanes per row, 256 / D rows per warp-wide step) -- and issues the loads of several
// steps before converting any of them.  The row maximum is log2(D / 8) shuffles within the
// row's lanes.  Page-table entries outside the pool are recorded as WF_ERR_PAGE_OOB and that
// token is skipped.
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
constexpr int kFp8Batch = 4;   // warp-wide steps whose loads are in flight together

__device__ __forceinline__ void unpack_bf16x8(const uint4& w, float (&x)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(u[i] << 16);
    x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// Largest value over the `lanes` lanes that share one head row (aligned groups of the warp).
template <int lanes>
__device__ __forceinline__ float row_max(float v) {
#pragma unroll
  for (int o = lanes / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Codes of 8 values (value i in byte i of the result) and the row's scale.  The row maximum is
// taken over all lanes of the row, so every lane derives the same inv and scale.
template <int lanes>
__device__ __forceinline__ uint2 quantize8(const float (&x)[8], float& scale) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(x[i]));
  const float amax = row_max<lanes>(a);
  float inv = 448.0f / amax;                       // IEEE division: these values decide codes
  const bool live = amax > 0.f && isfinite(inv);
  inv = live ? inv : 0.f;
  scale = live ? amax / 448.0f : 0.f;
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * h] * inv, x[4 * h + 1] * inv),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(x[4 * h + 2] * inv, x[4 * h + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    w[h] = (lo & 0xFFFFu) | (hi << 16);
  }
  return make_uint2(w[0], w[1]);
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

// Pool row of token `tok`, or -1 (recorded as WF_ERR_PAGE_OOB) when its page is outside the pool.
__device__ __forceinline__ int64_t fp8_pool_row(const int* pt_row, int tok, int page_size,
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

constexpr int kMaxFp8Dst = 9;   // this GPU's pool + up to 8 peers

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

template <int D>
__global__ void __launch_bounds__(kFp8Threads)
    wf_quant_append_kernel(const __grid_constant__ QuantParams p) {
  constexpr int LPR = D / 8;            // lanes per head row
  constexpr int RPS = 32 / LPR;         // head rows per warp-wide step
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  const int H = p.H;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int steps = (H + RPS - 1) / RPS;
  const int warps = gridDim.x * (kFp8Threads / 32);
  for (int t = blockIdx.x * (kFp8Threads / 32) + (threadIdx.x >> 5); t < p.rows; t += warps) {
    const int64_t prow =
        fp8_pool_row(p.pt_row, p.token0 + t, p.page_size, p.num_pages, lane, p.status);
    if (prow < 0) continue;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k + static_cast<int64_t>(t) * H * D);
    const uint4* vs = reinterpret_cast<const uint4*>(p.v + static_cast<int64_t>(t) * H * D);
    for (int s0 = 0; s0 < steps; s0 += kFp8Batch) {
      uint4 wk[kFp8Batch], wv[kFp8Batch];
#pragma unroll
      for (int b = 0; b < kFp8Batch; ++b) {
        const int h = (s0 + b) * RPS + rsub;
        if (h < H) {
          wk[b] = __ldg(ks + h * LPR + sub);
          wv[b] = __ldg(vs + h * LPR + sub);
        }
      }
#pragma unroll
      for (int b = 0; b < kFp8Batch; ++b) {
        const int h = (s0 + b) * RPS + rsub;
        if (s0 + b >= steps) break;                 // warp-uniform
        float xk[8], xv[8];
        unpack_bf16x8(h < H ? wk[b] : make_uint4(0, 0, 0, 0), xk);
        unpack_bf16x8(h < H ? wv[b] : make_uint4(0, 0, 0, 0), xv);
        float sk, sv;
        const uint2 ck = quantize8<LPR>(xk, sk);   // every lane shuffles, in or out of range
        const uint2 cv = quantize8<LPR>(xv, sv);
        if (h < H) {
          const int64_t e = prow * H * D / 8 + h * LPR + sub;   // 8-byte unit of the codes
#pragma unroll 1
          for (int d = 0; d < p.n_dst; ++d) {
            reinterpret_cast<uint2*>(p.dst[d].k_codes)[e] = ck;
            reinterpret_cast<uint2*>(p.dst[d].v_codes)[e] = cv;
            if (sub == 0) {
              p.dst[d].k_scale[prow * H + h] = sk;
              p.dst[d].v_scale[prow * H + h] = sv;
            }
          }
        }
      }
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
    const int64_t prow =
        fp8_pool_row(p.pt_row, p.token0 + t, p.page_size, p.num_pages, lane, p.status);
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
