// publish_kernel.cuh -- one-way publication of one chunk's K/V to every GPU that attends to it.
//
// In Wave Parallelism every GPU owns one chunk of the wavefront and attends to the chunks before
// it; each producer writes its freshly projected K/V straight into the consumers' attention
// buffers, one way, with no gather on arrival (project page, "03 End-to-end KV transport",
// items 01-03; KipQuest "The deep dive": every replica publishes its K/V right after projection,
// at every layer).  Here every GPU keeps a paged pool of the same geometry and the same page
// table, so the producer copies each token row of its chunk to the same (page, row) of its own
// pool and of every consumer's pool -- the consumer pools reached through peer pointers, plain
// 16-byte stores over NVLink, no TMA from or to peer memory.  A second, one-thread-per-pool
// kernel then raises the chunk's generation flag in every pool's flag array with a system-scope
// release; a consumer reads the flag with a system-scope acquire before loading those pages.
#pragma once

#include <stdint.h>

namespace wfk {

constexpr int kPublishThreads = 256;
constexpr int kMaxPublishDst = 9;   // this GPU + up to 8 peers

struct PublishDst {
  uint4* k_pool;
  uint4* v_pool;
  unsigned* flag;   // this layer's / chunk's word of that pool's flag array (may be null)
};

struct PublishParams {
  const uint4* k;
  const uint4* v;
  const int* pt_row;
  int* status;
  int token0, rows, vec_per_row, page_size, num_pages, n_dst;
  unsigned generation;
  PublishDst dst[kMaxPublishDst];
};

// One warp per token row, as the append kernel; every loaded 16-byte vector is stored to each
// destination pool in turn.
__global__ void __launch_bounds__(kPublishThreads)
    wf_publish_kernel(const __grid_constant__ PublishParams p) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kPublishThreads / 32);
  for (int t = blockIdx.x * (kPublishThreads / 32) + (threadIdx.x >> 5); t < p.rows; t += warps) {
    const int tok = p.token0 + t;
    int pg = 0;
    if (lane == 0) pg = __ldg(p.pt_row + tok / p.page_size);
    pg = __shfl_sync(0xffffffffu, pg, 0);
    if (pg < 0 || pg >= p.num_pages) {
      if (lane == 0) atomicCAS(p.status, 0, 5 /* WF_ERR_PAGE_OOB */);
      continue;
    }
    const size_t src = static_cast<size_t>(t) * p.vec_per_row;
    const size_t dst = (static_cast<size_t>(pg) * p.page_size + tok % p.page_size) *
                       p.vec_per_row;
    for (int c0 = lane; c0 < p.vec_per_row; c0 += 4 * 32) {
      uint4 a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < p.vec_per_row) {
          a[u] = __ldg(p.k + src + c);
          b[u] = __ldg(p.v + src + c);
        }
      }
#pragma unroll 1
      for (int d = 0; d < p.n_dst; ++d) {
        uint4* const kd = p.dst[d].k_pool;
        uint4* const vd = p.dst[d].v_pool;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          if (c < p.vec_per_row) {
            kd[dst + c] = a[u];
            vd[dst + c] = b[u];
          }
        }
      }
    }
  }
}

// Runs after wf_publish_kernel on the same stream, so every row is written; lane d makes them
// visible system-wide and then releases destination d's flag.  A row whose page-table entry is
// outside the pool was skipped by wf_publish_kernel (and recorded as WF_ERR_PAGE_OOB on this
// device), so the chunk is incomplete: its flag is then raised in no pool, and a consumer waits
// (and at worst times out) rather than reading stale pages as if they were the new chunk.
__global__ void wf_publish_flags_kernel(const __grid_constant__ PublishParams p) {
  const int lane = threadIdx.x;
  bool bad = false;
  if (p.rows > 0) {
    const int first = p.token0 / p.page_size, last = (p.token0 + p.rows - 1) / p.page_size;
    for (int i = first + lane; i <= last; i += 32) {
      const int pg = __ldg(p.pt_row + i);
      bad = bad || pg < 0 || pg >= p.num_pages;
    }
  }
  if (__any_sync(0xffffffffu, bad)) return;
  if (lane >= p.n_dst || p.dst[lane].flag == nullptr) return;
  __threadfence_system();
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p.dst[lane].flag), "r"(p.generation)
               : "memory");
}

}  // namespace wfk
