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
//   inv = 448 / amax, scale = amax / 448 (fp32 divisions; both 0 for a row of zeros),
//   code = e4m3(x * inv) -- round to nearest even, saturating at +-448 (cvt.rn.satfinite);
//   dequantized value = bf16_rne(decode(code) * scale).
// A per-page scale is not used because two chunks may share a page (their tokens are packed
// contiguously) and the page's first writer cannot know the second chunk's range.
//
// One warp per (token, head) row: lane i owns values [i E, (i + 1) E), E = D / 32, so a warp
// reads 2 D bytes per tensor in one coalesced transaction set and the row maximum is five
// shuffles.  Page-table entries outside the pool are recorded as WF_ERR_PAGE_OOB and that row is
// skipped.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstdint>

namespace wfk {

constexpr int kFp8Threads = 256;

template <int E>
struct Bf16Vec;   // E bf16 values loaded / stored as one word
template <>
struct Bf16Vec<4> {
  using T = uint2;
};
template <>
struct Bf16Vec<2> {
  using T = uint32_t;
};

template <int E>
__device__ __forceinline__ void unpack_bf16(typename Bf16Vec<E>::T w, float (&x)[E]) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(&w);
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    x[2 * i] = __uint_as_float(u[i] << 16);
    x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Codes of E values packed little-endian (value i in byte i), and the row scale.
template <int E>
__device__ __forceinline__ uint32_t quantize_lane(const float (&x)[E], float& scale) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) a = fmaxf(a, fabsf(x[i]));
  const float amax = warp_max(a);
  const float inv = amax > 0.f ? 448.0f / amax : 0.f;
  scale = amax > 0.f ? amax / 448.0f : 0.f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const uint32_t c = __nv_cvt_float_to_fp8(x[i] * inv, __NV_SATFINITE, __NV_E4M3);
    packed |= c << (8 * i);
  }
  return packed;
}

template <int D>
__global__ void __launch_bounds__(kFp8Threads)
    wf_quant_append_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                           uint8_t* __restrict__ k_codes, uint8_t* __restrict__ v_codes,
                           float* __restrict__ k_scale, float* __restrict__ v_scale,
                           const int* __restrict__ pt_row, int token0, int rows, int H,
                           int page_size, int num_pages, int* status) {
  constexpr int E = D / 32;
  static_assert(E == 2 || E == 4, "head_dim 64 or 128");
  using W = typename Bf16Vec<E>::T;
  const int lane = threadIdx.x & 31;
  const int64_t items = static_cast<int64_t>(rows) * H;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kFp8Threads / 32);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (kFp8Threads / 32) + (threadIdx.x >> 5);
       it < items; it += stride) {
    const int t = static_cast<int>(it / H), h = static_cast<int>(it - static_cast<int64_t>(t) * H);
    const int tok = token0 + t;
    const int pg = __ldg(pt_row + tok / page_size);
    if (pg < 0 || pg >= num_pages) {
      if (lane == 0) atomicCAS(status, 0, 5 /* WF_ERR_PAGE_OOB */);
      continue;
    }
    const size_t src = static_cast<size_t>(it) * D + lane * E;
    const size_t prow = (static_cast<size_t>(pg) * page_size + tok % page_size) * H + h;
    const W wk = *reinterpret_cast<const W*>(k + src);
    const W wv = *reinterpret_cast<const W*>(v + src);
    float xk[E], xv[E];
    unpack_bf16<E>(wk, xk);
    unpack_bf16<E>(wv, xv);
    float sk, sv;
    const uint32_t ck = quantize_lane<E>(xk, sk);
    const uint32_t cv = quantize_lane<E>(xv, sv);
    uint8_t* dk = k_codes + prow * D + lane * E;
    uint8_t* dv = v_codes + prow * D + lane * E;
    if (E == 4) {
      *reinterpret_cast<uint32_t*>(dk) = ck;
      *reinterpret_cast<uint32_t*>(dv) = cv;
    } else {
      *reinterpret_cast<uint16_t*>(dk) = static_cast<uint16_t>(ck);
      *reinterpret_cast<uint16_t*>(dv) = static_cast<uint16_t>(cv);
    }
    if (lane == 0) {
      k_scale[prow] = sk;
      v_scale[prow] = sv;
    }
  }
}

template <int E>
__device__ __forceinline__ typename Bf16Vec<E>::T dequantize_lane(uint32_t codes, float scale) {
  typename Bf16Vec<E>::T w;
  uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    float f[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __nv_fp8_storage_t c = static_cast<__nv_fp8_storage_t>(codes >> (8 * (2 * i + j)));
      const __half_raw hr = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);   // exact: e4m3 fits in fp16
      f[j] = __half2float(__half(hr)) * scale;
    }
    const __nv_bfloat162 b = __floats2bfloat162_rn(f[0], f[1]);      // .x is the low half
    u[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return w;
}

template <int D>
__global__ void __launch_bounds__(kFp8Threads)
    wf_dequant_kernel(const uint8_t* __restrict__ k_codes, const uint8_t* __restrict__ v_codes,
                      const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                      __nv_bfloat16* __restrict__ k_pool, __nv_bfloat16* __restrict__ v_pool,
                      const int* __restrict__ pt_row, int token0, int rows, int H, int page_size,
                      int num_pages, int* status) {
  constexpr int E = D / 32;
  static_assert(E == 2 || E == 4, "head_dim 64 or 128");
  using W = typename Bf16Vec<E>::T;
  const int lane = threadIdx.x & 31;
  const int64_t items = static_cast<int64_t>(rows) * H;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kFp8Threads / 32);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (kFp8Threads / 32) + (threadIdx.x >> 5);
       it < items; it += stride) {
    const int t = static_cast<int>(it / H), h = static_cast<int>(it - static_cast<int64_t>(t) * H);
    const int tok = token0 + t;
    const int pg = __ldg(pt_row + tok / page_size);
    if (pg < 0 || pg >= num_pages) {
      if (lane == 0) atomicCAS(status, 0, 5 /* WF_ERR_PAGE_OOB */);
      continue;
    }
    const size_t prow = (static_cast<size_t>(pg) * page_size + tok % page_size) * H + h;
    const uint8_t* sk = k_codes + prow * D + lane * E;
    const uint8_t* sv = v_codes + prow * D + lane * E;
    uint32_t ck, cv;
    if (E == 4) {
      ck = __ldg(reinterpret_cast<const uint32_t*>(sk));
      cv = __ldg(reinterpret_cast<const uint32_t*>(sv));
    } else {
      ck = __ldg(reinterpret_cast<const uint16_t*>(sk));
      cv = __ldg(reinterpret_cast<const uint16_t*>(sv));
    }
    const float fk = __ldg(k_scale + prow), fv = __ldg(v_scale + prow);
    *reinterpret_cast<W*>(k_pool + prow * D + lane * E) = dequantize_lane<E>(ck, fk);
    *reinterpret_cast<W*>(v_pool + prow * D + lane * E) = dequantize_lane<E>(cv, fv);
  }
}

}  // namespace wfk
