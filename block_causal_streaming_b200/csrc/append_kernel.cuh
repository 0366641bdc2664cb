// append_kernel.cuh -- publish one chunk's K/V of one layer into its pages (sm_100a).
//
// Wave Forcing's paged exchange writes each producer's K/V straight into the consumer's fixed
// attention slots so nothing is concatenated on arrival (project page, "03 End-to-end KV
// transport", item 03 "Layout"; KipQuest "The deep dive": K/V are published right after
// projection, at every layer).  Here the slots are pages: logical token t lives in physical page
// page_table_row[t / page_size] at row t % page_size of a pool [num_pages][page_size][H][D].
//
// One token row of H*D bf16 is contiguous both in the chunk and in the pool, so the kernel is a
// row-gather copy: one warp per token row (page looked up once per row), lanes stride over the
// row in 16-byte vectors with four loads in flight before their stores.  The copy is bit-exact.
#pragma once

#include <stdint.h>

namespace wfk {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads)
    wf_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                     uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                     const int* __restrict__ pt_row, int token0, int rows, int vec_per_row,
                     int page_size, int num_pages, int* status) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kAppendThreads / 32);
  for (int t = blockIdx.x * (kAppendThreads / 32) + (threadIdx.x >> 5); t < rows; t += warps) {
    const int tok = token0 + t;
    int pg = 0;
    if (lane == 0) pg = __ldg(pt_row + tok / page_size);
    pg = __shfl_sync(0xffffffffu, pg, 0);
    if (pg < 0 || pg >= num_pages) {
      if (lane == 0) atomicCAS(status, 0, 5 /* WF_ERR_PAGE_OOB */);
      continue;
    }
    const size_t src = static_cast<size_t>(t) * vec_per_row;
    const size_t dst = (static_cast<size_t>(pg) * page_size + tok % page_size) * vec_per_row;
    for (int c0 = lane; c0 < vec_per_row; c0 += 4 * 32) {
      uint4 a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < vec_per_row) {
          a[u] = __ldg(k + src + c);
          b[u] = __ldg(v + src + c);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < vec_per_row) {
          k_pool[dst + c] = a[u];
          v_pool[dst + c] = b[u];
        }
      }
    }
  }
}

}  // namespace wfk
