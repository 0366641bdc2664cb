// combine_kernel.cuh -- merge of the key splits of a split attention launch (sm_100a).
//
// When a unit's key range is split over S CTAs (S may differ between units: a launch can give its
// last units one part more), CTA s writes O_s = (sum over its keys of
// p_j v_j) / l_s and lse_s = log l_s (natural log, max folded in; -inf when none of its keys is
// visible to the row).  The softmax over all keys is then
//   lse = log sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) O_s,
// which this kernel evaluates with the largest lse_s subtracted first.  It is an HBM-bound pass:
// per (row, head) it reads S x (4 D + 4) bytes and writes 2 D (+ 4) bytes.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace wfk {

constexpr int kCombineThreads = 256;

// Which rows were split, and into how many parts: the unit layout of the attention launch
// (units of unit_rows query rows x one head, numbered in its dispatch order).
struct CombinePlan {
  int n_splits;      // parts of the first units
  int n_tail;        // the last n_tail units have n_splits + 1 parts
  int n_pairs;       // row blocks per head
  int head_group;    // heads per dispatch group
  int unit_rows;     // query rows per unit
};

// Parts of the unit that holds (row, head) -- the inverse of the attention kernel's unit order.
__device__ __forceinline__ int combine_parts(const CombinePlan& c, int row, int head, int H) {
  const int pair = row / c.unit_rows;
  const int group = head / c.head_group;
  const int unit = group * c.n_pairs * c.head_group + (c.n_pairs - 1 - pair) * c.head_group +
                   head % c.head_group;
  return unit >= c.n_pairs * H - c.n_tail ? c.n_splits + 1 : c.n_splits;
}

// One warp per (query row, head); lane i owns head-dim columns [i D/32, (i+1) D/32).  Rows of a
// unit that ran in one part are final already and are skipped.
template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    wf_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                      CombinePlan plan, int T_q, int H, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse) {
  constexpr int V = D / 32;   // 4 columns (one float4) at D = 128, 2 at D = 64
  static_assert(V == 2 || V == 4, "head_dim 64 or 128");
  const int64_t item = (static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (item >= static_cast<int64_t>(T_q) * H) return;
  const int row = static_cast<int>(item / H), head = static_cast<int>(item - int64_t(row) * H);
  const int n_splits = combine_parts(plan, row, head, H);
  if (n_splits < 2) return;

  float mx = -INFINITY;
  for (int s = 0; s < n_splits; ++s)
    mx = fmaxf(mx, part_lse[(static_cast<size_t>(s) * H + head) * T_q + row]);
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float ls = part_lse[(static_cast<size_t>(s) * H + head) * T_q + row];
    if (ls == -INFINITY) continue;                     // no visible key in this split
    const float w = expf(ls - mx);
    wsum += w;
    const float* src = part_o + ((static_cast<size_t>(s) * T_q + row) * H + head) * D + lane * V;
    if (V == 4) {
      const float4 x = *reinterpret_cast<const float4*>(src);
      acc[0] += w * x.x;
      acc[1] += w * x.y;
      acc[2] += w * x.z;
      acc[3] += w * x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(src);
      acc[0] += w * x.x;
      acc[1] += w * x.y;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = out + (static_cast<size_t>(row) * H + head) * D + lane * V;
#pragma unroll
  for (int i = 0; i < V; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv,
                                                                          acc[i + 1] * inv);
  if (lse != nullptr && lane == 0)
    lse[static_cast<size_t>(head) * T_q + row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace wfk
