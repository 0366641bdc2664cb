// attn_kernel.cuh -- block-causal chunk attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Rule computed (Wave Forcing; KipQuest summary of arXiv 2611.00859, "The deep dive"; project
// page "01 The design gap" panel C): a query of chunk c attends fully within chunk c and to every
// earlier chunk, never to a later one.  With the K/V sequence in logical order (context first,
// then the active chunks cleanest to noisiest) the visible keys of chunk c are the prefix
// [0, kv_end_c) with kv_end_c = chunk_offsets[c+1], read in place from the paged pool (project
// page, "03 End-to-end KV transport", item 03 "Layout").
//
// One CTA = one unit of work: a head and 256 consecutive query rows (two 128-row Q tiles that
// share every K/V tile they load).  Units are numbered so that the hardware's in-order block
// dispatch runs the most expensive first (longest-processing-time order): kv_end is
// non-decreasing in the query row, so the last query rows have the most visible keys; blockIdx 0
// takes the last 256 rows, heads vary fastest.
//
// Warp roles (384 threads):
//   warps 0-3  softmax of Q tile 0: thread t owns query row t (TMEM lane t)
//   warps 4-7  softmax of Q tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j into a ring of NS shared-memory slots,
//              page by page through the page table; also allocates/frees TMEM
//   warp  9    MMA issuer: S_q = Q_q K_j^T (SS form) and O_q += P_q V_j (TS form, P in TMEM)
//   warps 10-11 idle
// TMEM (512 columns): S_q / P_q at columns [128q, 128q+128) (P, bf16x2, aliases the first 64),
// O_q at [256 + D q, 256 + D q + D).
//
// Synchronisation (all mbarriers, all waits bounded):
//   q_full        TMA -> MMA          Q tiles landed
//   kv_full[s]    TMA -> MMA          K or V tile landed in slot s
//   kv_empty[s]   MMA commit -> TMA   slot s free again (both Q tiles' MMAs on it completed)
//   s_full[q]     MMA commit -> softmax q   S_q of tile j ready (also covers PV_q of tile j-1)
//   p_full[q]     softmax q -> MMA    P_q of tile j written to TMEM (and O_q rescaled if needed)
//   o_done[q]     MMA commit -> MMA / softmax   PV_q of tile j completed
// S_q of tile j+1 overwrites the TMEM columns that PV_q of tile j reads P from, so the MMA warp
// issues it only after o_done[q] reports that PV completed.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace wfk {

constexpr int kBM = 128;        // query rows per Q tile (UMMA M)
constexpr int kBN = 128;        // keys per K/V tile (UMMA N of QK^T, K of PV)
constexpr int kNQT = 2;         // Q tiles per CTA
constexpr int kAttnThreads = 384;
constexpr int kMaxQChunks = 64;
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s per wait
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;   // 0.2 s when draining

struct AttnParams {
  CUtensorMap tm_q;  // bf16 (D, H, T_q), box (64, 1, 128), 128B swizzle
  CUtensorMap tm_k;  // bf16 (D, H, num_pages * page_size), box (64, 1, box_rows), 128B swizzle
  CUtensorMap tm_v;
  __nv_bfloat16* out;
  float* lse;
  const int* page_table;
  int* status;
  unsigned* grid_abort;
  int T_q, H, num_pages, page_size, total_rows, box_rows, n_pairs;
  float sl2;  // scale * log2(e)
  unsigned launch_id;
  int nqc;                          // non-empty query chunks
  int qc_row_end[kMaxQChunks];      // exclusive end row of query chunk i (query-row space)
  int qc_kv_end[kMaxQChunks];       // number of visible keys for rows of query chunk i
};

__device__ __forceinline__ int kv_end_of_row(const AttnParams& p, int r) {
  for (int c = 0; c < p.nqc; ++c)
    if (r < p.qc_row_end[c]) return p.qc_kv_end[c];
  return p.qc_kv_end[p.nqc - 1];
}

// Wait on a phase with only a timeout (no abort check): used to drain in-flight async work
// before shared memory or TMEM is released.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity))
    if (globaltimer_ns() - t0 > kDrainTimeoutNs) return false;
  return true;
}

template <int D>
struct AttnSmem {
  static constexpr int DH = D / 64;                      // 128-byte halves of a row
  static constexpr int NS = (D == 128) ? 4 : 8;          // K/V ring slots
  static constexpr uint32_t HALF = 128u * 128u;          // 128 rows x 128 B, 128B-swizzled
  static constexpr uint32_t TILE = DH * HALF;            // one Q, K or V tile
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = Q_OFF + kNQT * TILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NS * TILE;
  // barrier indices
  static constexpr int B_Q = 0, B_KVF = 1, B_KVE = 1 + NS, B_S = 1 + 2 * NS, B_P = B_S + 2,
                       B_O = B_P + 2, B_DRAIN = B_O + 2, NBAR = B_DRAIN + 1;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;        // slack for 1024-byte alignment
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    wf_attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = AttnSmem<D>;
  constexpr int DH = L::DH, NS = L::NS;
  constexpr uint32_t TILE = L::TILE, HALF = L::HALF;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + L::MISC_OFF);
  volatile int* const cta_abort = reinterpret_cast<volatile int*>(base_ptr + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return base + L::BAR_OFF + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x;
  const int pair = p.n_pairs - 1 - unit / p.H;
  const int head = unit % p.H;
  const int m0 = pair * (kNQT * kBM);
  const int last_row = min(m0 + kNQT * kBM, p.T_q) - 1;
  const int n_max = kv_end_of_row(p, last_row);        // keys any row of this unit may see
  const int nk = (n_max + kBN - 1) / kBN;                // K/V tiles to visit

  const WaitCtx w{cta_abort, p.grid_abort, p.status, p.launch_id, 6 /* WF_ERR_TIMEOUT */,
                  kWaitTimeoutNs};

  if (threadIdx.x == 0) {
    *cta_abort = (*reinterpret_cast<volatile unsigned*>(p.grid_abort) == p.launch_id) ? 1 : 0;
    for (int i = 0; i < L::NBAR; ++i)
      mbar_init(bar(i), (i == L::B_P || i == L::B_P + 1) ? 128u : 1u);
    mbar_init_fence();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *cta_abort != 0;

  if (!skip && warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int q = warp >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;                       // row within the Q tile == TMEM lane
    const int row_g = m0 + q * kBM + row;                 // query row
    const int n_r = kv_end_of_row(p, min(row_g, p.T_q - 1));
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + static_cast<uint32_t>(q * 128);
    const uint32_t tO = tmem + lane_off + 256u + static_cast<uint32_t>(q * D);
    const float sl2 = p.sl2;
    float m2 = -INFINITY;   // running max of the base-2 logits in use
    float l = 0.f;          // running sum of exp2(t - m2)
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_S + q), j & 1, w));
      if (!ok) break;
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + 32u * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[i]);
      }
      const int lim = n_r - j * kBN;                      // visible columns of this tile
      if (lim < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < kBN; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float tmax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      // Move the reference max only when the new one exceeds it by more than 2^8: O and l both
      // stay expressed against the same stale reference, so O / l is unchanged, and every
      // exp2(t - m2) stays <= 256.
      const bool need = tmax > m2 + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m2 - tmax);                   // 0 on the first visible tile
        m2 = tmax;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O_q holds PV of tiles < j (the s_full commit covered it); rescale this warp's rows.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32u * c, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + 32u * c, r);
        }
      }
      l *= alpha;
      const float negm = -m2;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(fmaf(s[64 * h + 2 * i], sl2, negm));
          const float p1 = ex2_approx(fmaf(s[64 * h + 2 * i + 1], sl2, negm));
          rs0 += p0;
          rs1 += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + 32u * h, pk);
      }
      l += rs0 + rs1;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::B_P + q));
    }
    // ------------------------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_O + q), (nk - 1) & 1, w));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool live = row_g < p.T_q;
      __nv_bfloat16* const orow = p.out + (static_cast<size_t>(row_g) * p.H + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + 32u * c, r);
        tmem_wait_ld();
        if (live) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                                __uint_as_float(r[2 * i + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (p.lse != nullptr && live)
        p.lse[static_cast<size_t>(head) * p.T_q + row_g] = (m2 + __log2f(l)) * 0.69314718056f;
    }
  } else if (!skip && warp == 8) {
    // ------------------------------------------------------------------------ TMA producer
    const int R = p.box_rows, nb = kBN / R;             // page boxes per K/V tile (<= 8)
    bool ok = true;
    int last_it[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) last_it[s] = -1;
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar(L::B_Q), kNQT * TILE);
#pragma unroll
      for (int qt = 0; qt < kNQT; ++qt)
#pragma unroll
        for (int h = 0; h < DH; ++h)
          tma_load_3d(base + L::Q_OFF + qt * TILE + h * HALF, &p.tm_q, 64 * h, head,
                      m0 + qt * kBM, bar(L::B_Q));
    }
    for (int j = 0; j < nk && ok; ++j) {
      // lane b resolves the physical row of box b of this tile
      int coord = p.total_rows;                          // past the pool: TMA fills zeros
      const int tok = j * kBN + lane * R;
      if (lane < nb && tok < n_max) {
        int pg = __ldg(p.page_table + tok / p.page_size);
        if (pg < 0 || pg >= p.num_pages) {
          atomicCAS(p.status, 0, 5 /* WF_ERR_PAGE_OOB */);
          pg = 0;
        }
        coord = pg * p.page_size + tok % p.page_size;
      }
      int cb[8];
#pragma unroll
      for (int b = 0; b < 8; ++b) cb[b] = __shfl_sync(0xffffffffu, coord, b);
      if (lane == 0) {
#pragma unroll
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int it = 2 * j + kv, slot = it % NS;
          ok = mbar_wait(bar(L::B_KVE + slot), ((it / NS) & 1) ^ 1, w);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::B_KVF + slot), TILE);
          const CUtensorMap* map = kv ? &p.tm_v : &p.tm_k;
          const uint32_t dst = base + L::KV_OFF + slot * TILE;
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            if (b < nb) {
#pragma unroll
              for (int h = 0; h < DH; ++h)
                tma_load_3d(dst + h * HALF + static_cast<uint32_t>(b * R * 128), map, 64 * h,
                            head, cb[b], bar(L::B_KVF + slot));
            }
          }
          last_it[slot] = it;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      // every load this warp issued must land before shared memory is released
      mbar_wait_drain(bar(L::B_Q), 0);
#pragma unroll
      for (int s = 0; s < NS; ++s)
        if (last_it[s] >= 0) mbar_wait_drain(bar(L::B_KVF + s), (last_it[s] / NS) & 1);
    }
  } else if (!skip && warp == 9) {
    // ---------------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);   // Q, K both K-major
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);     // P (TMEM), V MN-major
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar(L::B_Q), 0, w);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    int js[2] = {0, 0};   // next tile whose S is to be issued, per Q tile
    int jp[2] = {0, 0};   // next tile whose PV is to be issued, per Q tile
    bool vz_done = false;
    const int zero_from = n_max - (nk - 1) * kBN;         // rows >= this of the last V tile
    uint64_t t_last = globaltimer_ns();
    unsigned idle = 0;
    while (ok && (jp[0] < nk || jp[1] < nk)) {
      int action = -1;   // 0/1: S of Q tile 0/1;  2/3: PV of Q tile 0/1
      if (lane == 0) {
#pragma unroll
        for (int q = 0; q < 2 && action < 0; ++q) {
          const int j = js[q];
          if (j < nk && j == jp[q]) {
            const int it = 2 * j;
            if (mbar_test(bar(L::B_KVF + it % NS), (it / NS) & 1) &&
                (j == 0 || mbar_test(bar(L::B_O + q), (j - 1) & 1)))
              action = q;
          }
        }
#pragma unroll
        for (int q = 0; q < 2 && action < 0; ++q) {
          const int j = jp[q];
          if (j < js[q]) {
            const int it = 2 * j + 1;
            if (mbar_test(bar(L::B_P + q), j & 1) &&
                mbar_test(bar(L::B_KVF + it % NS), (it / NS) & 1))
              action = 2 + q;
          }
        }
        if (action < 0) {
          if ((++idle & 255u) == 0) {
            if (aborted(w)) {
              ok = false;
            } else if (globaltimer_ns() - t_last > kWaitTimeoutNs) {
              raise_abort(w);
              ok = false;
            }
          }
        } else {
          idle = 0;
          t_last = globaltimer_ns();
        }
      }
      action = __shfl_sync(0xffffffffu, action, 0);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (action < 0) continue;
      if (action < 2) {
        const int q = action, j = js[q], it = 2 * j, slot = it % NS;
        if (lane == 0) {
          tc_fence_after();
          const uint32_t qa = base + L::Q_OFF + q * TILE;
          const uint32_t kb = base + L::KV_OFF + slot * TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * HALF + (kk % 4) * 32;   // 16 bf16 = 32 B per step
            umma_ss(tmem + static_cast<uint32_t>(q * 128), smem_desc_sw128(qa + off, 16, 1024),
                    smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(L::B_S + q));
          if (js[1 - q] > j) umma_commit(bar(L::B_KVE + slot));     // both Q tiles done with K_j
        }
        js[q] = j + 1;
      } else {
        const int q = action - 2, j = jp[q], it = 2 * j + 1, slot = it % NS;
        const uint32_t vb = base + L::KV_OFF + slot * TILE;
        if (j == nk - 1 && zero_from < kBN && !vz_done) {
          // Rows past the last visible key may hold anything (even NaN, which 0 * NaN would
          // spread); zero them before any PV reads this tile.
          __syncwarp();
          const int n16 = (kBN - zero_from) * 8;                 // 16-byte pieces per half
          for (int i = lane; i < n16 * DH; i += 32) {
            const int h = i / n16, rr = i % n16;
            const uint32_t a = vb + h * HALF + static_cast<uint32_t>(zero_from * 128 + rr * 16);
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          vz_done = true;
        }
        if (lane == 0) {
          tc_fence_after();
          const uint32_t pa = tmem + static_cast<uint32_t>(q * 128);
          const uint32_t od = tmem + 256u + static_cast<uint32_t>(q * D);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ts(od, pa + 8u * kk, smem_desc_sw128(vb + kk * 2048u, HALF, 1024), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(L::B_O + q));
          if (jp[1 - q] > j) umma_commit(bar(L::B_KVE + slot));     // both Q tiles done with V_j
        }
        jp[q] = j + 1;
      }
    }
    if (lane == 0) {
      // every MMA this warp issued must complete before TMEM is released
      umma_commit(bar(L::B_DRAIN));
      mbar_wait_drain(bar(L::B_DRAIN), 0);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace wfk
