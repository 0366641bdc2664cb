// i8_kernel.cuh -- quantization of Q and K for the 8-bit attention tiers (sm_100a): INT8
// (Sage-like) and FP8 (e4m3).
//
// The pages name SageAttention with W8A8 as the fast attention backend (GitHub README, results
// table, "Sage . causal . paged" rows; KipQuest abstract) and give no internals.  The tier built
// here:
//   - mu[h][d]: the mean of the keys of head h over all T_kv tokens of the layer -- an exact sum
//     (fp64 accumulation of bf16 values; for key magnitudes within 2^30 of each other every
//     partial sum is exact, so the order of the atomic adds does not matter), divided in fp64 and
//     rounded once to fp32.  K' = fp32(K - mu) shifts every logit of a query row by the same
//     constant q . mu, which the softmax does not see.
//   - one scale per (128 keys, head) of K' in logical key order and per (128 query rows, head) of
//     Q, counted from key / row 0: with a the block's largest magnitude, inv = 127 / a and
//     scale = a / 127 (fp32 divisions; both 0 for a block of zeros or when 127 / a overflows),
//     code = clamp(round_half_even(x * inv), -127, 127) with an fp32 product.
// The blocks are the attention kernel's Q tiles and K tiles, so each S tile is dequantized by one
// scalar (scale_q x scale_k) folded into the softmax's existing multiply.
// The FP8 tier (project page, "03 End-to-end KV transport", item 01 "Precision", measures K/V in
// FP8; the pages give no granularity for attention operands) uses the same blocks without the key
// mean: inv = 448 / a, scale = a / 448, code = e4m3(x * inv) rounded to nearest even and
// saturated (the FP8 K/V pages' encoder).
//
// Kernels:
//   wf_kmean_kernel     fp64 column sums of the paged bf16 keys (atomics into k_sum, zeroed first)
//   wf_kmean_finalize   k_mean = fp32(k_sum / T_kv)
//   wf_block_quant_kernel<kKeys, kE4M3>  one CTA per (block, head): K' (through the page table)
//                       or Q, largest magnitude, codes into a contiguous [rows][H][D] (int8 or
//                       e4m3) and the scale.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

namespace wfk {

constexpr int kI8Block = 128;          // rows per scale block (Q tiles and K tiles)
constexpr int kKmeanThreads = 256;
constexpr int kQuantI8Threads = 256;

struct QkI8Params {
  const __nv_bfloat16* q;       // [T_q][H][D]
  const __nv_bfloat16* k_pool;  // [num_pages * page_size][H][D]
  const int* pt_row;            // page-table row of the layer
  int8_t* q_codes;              // [T_q][H][D]
  float* q_scale;               // [H][ceil(T_q / 128)]
  int8_t* k_codes;              // [T_kv][H][D], logical key order
  float* k_scale;               // [H][ceil(T_kv / 128)]
  float* k_mean;                // [H][D]
  double* k_sum;                // [H][D], zeroed before wf_kmean_kernel
  int* status;
  int T_q, T_kv, H, page_size, num_pages;
};

// Pool row of logical token `tok` (-1, recorded as WF_ERR_PAGE_OOB, when its page is outside).
__device__ __forceinline__ int64_t i8_pool_row(const QkI8Params& p, int tok) {
  const int pg = __ldg(p.pt_row + tok / p.page_size);
  if (pg < 0 || pg >= p.num_pages) {
    atomicCAS(p.status, 0, 5 /* WF_ERR_PAGE_OOB */);
    return -1;
  }
  return static_cast<int64_t>(pg) * p.page_size + tok % p.page_size;
}

// Block b sums tokens [b * per, (b + 1) * per) (per <= kKmeanMaxPer); thread t owns columns
// t, t + 256, ... of H * D.  The block's pool rows are resolved once into shared memory, so the
// value loads of consecutive tokens are independent.
constexpr int kKmeanMaxPer = 128;

template <int D>
__global__ void __launch_bounds__(kKmeanThreads)
    wf_kmean_kernel(const __grid_constant__ QkI8Params p, int per) {
  __shared__ int64_t rows[kKmeanMaxPer];
  const int cols = p.H * D;
  const int t0 = blockIdx.x * per, n = min(p.T_kv, t0 + per) - t0;
  for (int i = threadIdx.x; i < n; i += kKmeanThreads) rows[i] = i8_pool_row(p, t0 + i);
  __syncthreads();
  for (int c = threadIdx.x; c < cols; c += kKmeanThreads) {
    double acc = 0.0;
#pragma unroll 8
    for (int i = 0; i < n; ++i) {
      const int64_t row = rows[i];
      if (row >= 0) acc += static_cast<double>(__bfloat162float(p.k_pool[row * cols + c]));
    }
    if (n > 0) atomicAdd(p.k_sum + c, acc);
  }
}

__global__ void wf_kmean_finalize(const __grid_constant__ QkI8Params p, int cols) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < cols) p.k_mean[c] = static_cast<float>(p.k_sum[c] / static_cast<double>(p.T_kv));
}

// One CTA per (block, head): 128 rows x D values, two threads per row (D / 2 values each).
// kKeys: rows are logical keys read through the page table (smoothed by k_mean for int8); else
// query rows of q.  kE4M3: the FP8 tier's codes instead -- scale = amax / 448,
// code = e4m3(x * (448 / amax)) rounded to nearest even and saturated (cvt.rn.satfinite), no
// smoothing; the same block layout.
template <int D, bool kKeys, bool kE4M3 = false>
__global__ void __launch_bounds__(kQuantI8Threads)
    wf_block_quant_kernel(const __grid_constant__ QkI8Params p) {
  constexpr int HALF = D / 2;               // values per thread
  static_assert(D == 128, "the INT8 tier runs head_dim 128");
  __shared__ float red[kQuantI8Threads / 32];
  const int b = blockIdx.x, h = blockIdx.y;
  const int rows = kKeys ? p.T_kv : p.T_q;
  const int r = b * kI8Block + (threadIdx.x >> 1), half = threadIdx.x & 1;
  const int cols = p.H * D;
  float x[HALF];
  bool live = r < rows;
  if (live) {
    const __nv_bfloat16* src;
    if (kKeys) {
      const int64_t row = i8_pool_row(p, r);
      live = row >= 0;
      src = p.k_pool + (live ? row : 0) * cols + h * D + half * HALF;
    } else {
      src = p.q + static_cast<int64_t>(r) * cols + h * D + half * HALF;
    }
    if (live) {
#pragma unroll
      for (int i = 0; i < HALF / 8; ++i) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + 8 * i);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x[8 * i + 2 * j] = __uint_as_float(u[j] << 16);
          x[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
      }
      if (kKeys && !kE4M3) {
        const float* mu = p.k_mean + h * D + half * HALF;
#pragma unroll
        for (int i = 0; i < HALF; ++i) x[i] = x[i] - __ldg(mu + i);
      }
    }
  }
  float a = 0.f;
  if (live) {
#pragma unroll
    for (int i = 0; i < HALF; ++i) a = fmaxf(a, fabsf(x[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int w = 1; w < kQuantI8Threads / 32; ++w) a = fmaxf(a, red[w]);
  constexpr float kQmax = kE4M3 ? 448.0f : 127.0f;
  float inv = kQmax / a;                      // IEEE division: these values decide codes
  const bool nz = a > 0.f && isfinite(inv);
  inv = nz ? inv : 0.f;
  if (threadIdx.x == 0) {
    const int nblocks = (rows + kI8Block - 1) / kI8Block;
    (kKeys ? p.k_scale : p.q_scale)[h * nblocks + b] = nz ? a / kQmax : 0.f;
  }
  if (!live) return;
  int8_t* dst = (kKeys ? p.k_codes : p.q_codes) + static_cast<int64_t>(r) * cols + h * D +
                half * HALF;
#pragma unroll
  for (int i = 0; i < HALF / 16; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t word = 0;
      if (kE4M3) {
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const float2 y = make_float2(x[16 * i + 4 * j + e] * inv,
                                       x[16 * i + 4 * j + e + 1] * inv);
          const uint32_t two = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
          word |= (two & 0xFFFFu) << (8 * e);                   // .x in the low byte
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int c = __float2int_rn(x[16 * i + 4 * j + e] * inv);   // round half to even
          c = max(-127, min(127, c));
          word |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * e);
        }
      }
      w[j] = word;
    }
    *reinterpret_cast<uint4*>(dst + 16 * i) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace wfk
