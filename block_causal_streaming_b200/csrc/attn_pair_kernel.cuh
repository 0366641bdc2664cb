// attn_pair_kernel.cuh -- block-causal chunk attention forward on CTA pairs (sm_100a, D = 128).
//
// Same rule and work order as attn_kernel.cuh (a query of chunk c sees the key prefix
// [0, kv_end_c); units of 256 query rows of one head, longest first), but each unit runs on a
// cluster of two CTAs on two SMs that share every MMA: tcgen05.mma.cta_group::2 computes
// M = 256 rows (128 per CTA, each CTA's TMEM holding its own rows) with the B operand split by N
// between the two CTAs' shared memory.  Consequences:
//   * each CTA loads only half of every K/V tile (64 of the 128 keys of K; 64 of the 128
//     head-dim columns of V), halving shared-memory and L2 traffic per SM;
//   * one Q tile per CTA leaves TMEM room for three S buffers (3 x 128 + O 128 = 512 columns),
//     so QK^T of tile j+2 is issued before P.V of tile j and the tensor pipe does not wait for
//     the softmax;
//   * the softmax of a 128 x 128 tile is split over two warpgroups (half a row per thread).
//
// Roles per CTA (384 threads): warps 0-7 softmax of this CTA's 128 rows, two warpgroups per row
// (thread t of warpgroup g = row t = TMEM lane t, keys [64 g, 64 g + 64) of each tile); warp 8
// TMA producer (+ TMEM allocation, shared by the pair) loading into CTA-local barriers; warp 10
// relay: once a local tile has landed (and, for the last V tile, its rows past the last visible
// key are zeroed) it arrives on the leader's barrier; warp 9, lane 0 of CTA rank 0 only: MMA
// issuer for both CTAs; warp 11 idle.
//
// Barriers (same layout in both CTAs; "leader" = CTA rank 0):
//   q_local, kv_local[s]  each CTA: its own TMA loads complete their bytes here
//   q_full, kv_full[s]    leader, count 2: one relay arrival per CTA
//   kv_empty[s]           both CTAs: the leader's MMA commits to each CTA's copy
//   s_full[b], o_done[b]  both CTAs: committed by the leader to each CTA's copy (b = j mod 3)
//   p_full[b]             leader, count 16: one arrival per softmax warp of both CTAs (after a
//                         __syncwarp, so one cluster-scope arrive per warp, not per thread)
//   x_max, x_sum          each CTA, count 256: the two softmax warpgroups swap row maxima / sums
// Measured on the 1.3B 5-step wavefront this kernel is correct but slower than attn_kernel.cuh
// (4.53 ms against 3.4-3.6 ms for the single-CTA kernel of the time, 2.8 ms now): the cross-CTA
// hand-offs cost more than the tensor time they save.  It is launched only when the library is
// compiled with WF_ATTN_PAIR=1.
#pragma once

#include <cuda_bf16.h>

#include "attn_kernel.cuh"
#include "sm100.cuh"

namespace wfk {

constexpr int kPairThreads = 384;
constexpr int kPairBN = 128;   // keys per K/V tile
constexpr int kPairSBuf = 3;   // S buffers per CTA

// Bounded wait with cluster-scope acquire (arrivals may come from the other CTA).
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_cluster(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*w.cta_abort != 0) return false;
      if (globaltimer_ns() - t0 > w.timeout_ns) {
        raise_abort(w);
        return false;
      }
      if ((i & 4095u) == 0 &&
          *reinterpret_cast<volatile unsigned*>(w.grid_abort) == w.launch_id) {
        *w.cta_abort = 1;
        return false;
      }
    }
  }
}

struct PairSmem {
  static constexpr uint32_t QHALF = 128u * 128u;   // 128 rows x 128 B (64 head-dim columns)
  static constexpr uint32_t QTILE = 2 * QHALF;     // this CTA's 128 query rows
  static constexpr uint32_t KHALF = 64u * 128u;    // 64 keys x 128 B
  static constexpr uint32_t SLOT = 16384u;         // K half-tile (64 keys x 256 B) or
                                                   // V half-tile (128 keys x 128 B)
  static constexpr int NS = 8;                     // ring slots: 4 tiles of K + V
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = QTILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NS * SLOT;
  static constexpr int B_Q = 0, B_KVF = 1, B_KVE = 1 + NS, B_S = 1 + 2 * NS,
                       B_P = B_S + kPairSBuf, B_O = B_P + kPairSBuf,
                       B_DRAIN = B_O + kPairSBuf, B_X = B_DRAIN + 1, B_L = B_X + 1,
                       B_KVL = B_L + 1, B_QL = B_KVL + NS, NBAR = B_QL + 1;
  static constexpr uint32_t X_OFF = BAR_OFF + NBAR * 8;          // row-max / row-sum exchange
  static constexpr uint32_t PT_OFF = X_OFF + 768 * 4;             // page-table cache
  static constexpr uint32_t MISC_OFF = PT_OFF + kPtCache * 4;
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    wf_attn_pair_kernel(const __grid_constant__ AttnParams p) {
  using L = PairSmem;
  constexpr int D = 128, BN = kPairBN, NB = kPairSBuf, NS = L::NS;
  constexpr uint32_t SLOT = L::SLOT, QHALF = L::QHALF, KHALF = L::KHALF;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + L::MISC_OFF);
  volatile int* const cta_abort = reinterpret_cast<volatile int*>(base_ptr + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return base + L::BAR_OFF + 8u * static_cast<uint32_t>(i); };

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  auto lead = [&](int i) -> uint32_t { return mapa_shared(bar(i), 0); };   // leader's copy
  auto mine = [&](int i) -> uint32_t { return mapa_shared(bar(i), rank); };
  auto other = [&](int i) -> uint32_t { return mapa_shared(bar(i), peer); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x >> 1;
  const int pair = p.n_pairs - 1 - unit / p.H;     // 256-row block, longest first
  const int head = unit % p.H;
  const int m0 = pair * 256 + 128 * static_cast<int>(rank);   // this CTA's first query row
  const int last_row = min(pair * 256 + 256, p.T_q) - 1;
  const int n_max = kv_end_of_row(p, last_row);
  const int nk = (n_max + BN - 1) / BN;

  const WaitCtx w{cta_abort, p.grid_abort, p.status, p.launch_id, 6 /* WF_ERR_TIMEOUT */,
                  kWaitTimeoutNs};

  if (threadIdx.x == 0) {
    *cta_abort = (*reinterpret_cast<volatile unsigned*>(p.grid_abort) == p.launch_id) ? 1 : 0;
    for (int i = 0; i < L::NBAR; ++i) {
      uint32_t count = 1;
      if (i == L::B_Q || (i >= L::B_KVF && i < L::B_KVF + NS)) count = 2;
      if (i >= L::B_P && i < L::B_P + NB) count = 16;   // 8 softmax warps per CTA
      if (i == L::B_X || i == L::B_L) count = 256;
      mbar_init(bar(i), count);
    }
    mbar_init_fence();
  }
  if (warp == 8) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *cta_abort != 0;

  if (!skip && warp < 8) {
    // ------------------------------------------------------------------------- softmax
    // Two warpgroups share each row: warpgroup g owns keys [64 g, 64 g + 64) of every tile and
    // head-dim columns [64 g, 64 g + 64) of O.  Per tile they swap their partial row maxima
    // through shared memory (double-buffered by tile parity) so both use the same reference.
    const int g = warp >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;
    const int row_g = m0 + row;
    const int n_r = kv_end_of_row(p, min(row_g, p.T_q - 1));
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + 384u + static_cast<uint32_t>(64 * g);
    float* const xmax = reinterpret_cast<float*>(base_ptr + L::X_OFF);   // [parity][g][row]
    float* const xsum = xmax + 512;                                      // [g][row]
    const float sl2 = p.sl2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    float m2 = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int b = j % NB;
      const uint32_t tS = tmem + lane_off + static_cast<uint32_t>(128 * b);
      ok = __all_sync(0xffffffffu, mbar_wait_cl(bar(L::B_S + b), (j / NB) & 1, w));
      if (!ok) break;
      tc_fence_after();
      float s[64];
      {
        uint32_t r[64];
        tmem_ld32(tS + 64u * g, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(tS + 64u * g + 32u, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(r[c]);
      }
      const int lim = n_r - j * BN - 64 * g;             // visible columns of this half
      const bool masked = lim < 64;
      if (masked) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < 64; c += 8) {
        mx0 = max3(mx0, s[c], s[c + 1]);
        mx1 = max3(mx1, s[c + 2], s[c + 3]);
        if (c + 4 < 64) mx2 = max3(mx2, s[c + 4], s[c + 5]);
        if (c + 6 < 64) mx3 = max3(mx3, s[c + 6], s[c + 7]);
      }
      const float mx = max3(mx0, mx1, fmaxf(mx2, mx3));
      xmax[(j & 1) * 256 + g * 128 + row] = mx;
      mbar_arrive(bar(L::B_X));
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_X), j & 1, w));
      if (!ok) break;
      const float tmax = fmaxf(mx, xmax[(j & 1) * 256 + (1 - g) * 128 + row]) * sl2;
      const bool need = tmax > m2 + 8.0f;   // move the reference max only by more than 2^8
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m2 - tmax);
        m2 = tmax;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // rescale this half of O once P.V of tile j-1 has completed
        ok = __all_sync(0xffffffffu,
                        mbar_wait_cl(bar(L::B_O + (j - 1) % NB), ((j - 1) / NB) & 1, w));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32u * c, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + 32u * c, r);
        }
      }
      l *= alpha;
      const float2 negm = make_float2(-m2, -m2);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      uint32_t pk[32];
      if (!masked) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), sl2x2, negm);
          float2 e;
          if ((i & 7) < WF_EXP2_POLY_EIGHTHS) {
            e = exp2_poly2(x);
          } else {
            e.x = ex2_approx(x.x);
            e.y = ex2_approx(x.y);
          }
          if (i & 1) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
          pk[i] = pack_bf16x2(e.x, e.y);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), sl2x2, negm);
          const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          if (i & 1) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
          pk[i] = pack_bf16x2(e.x, e.y);
        }
      }
      tmem_st32(tS + 32u * g, pk);                      // P: keys [64 g, 64 g + 64)
      const float2 acc = __fadd2_rn(acc0, acc1);
      l += acc.x + acc.y;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {   // one arrival per warp: the leader's MMA waits for all 16 warps' P
        if (rank == 0) mbar_arrive(bar(L::B_P + b));
        else mbar_arrive_cluster(lead(L::B_P + b));
      }
    }
    // ------------------------------------------------------------------------- epilogue
    xsum[g * 128 + row] = l;
    mbar_arrive(bar(L::B_L));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_L), 0, w));
    if (ok)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_cl(bar(L::B_O + (nk - 1) % NB), ((nk - 1) / NB) & 1, w));
    if (ok) {
      tc_fence_after();
      const float l_row = l + xsum[(1 - g) * 128 + row];
      const float inv_l = 1.f / l_row;
      const bool live = row_g < p.T_q;
      __nv_bfloat16* const orow = p.out + (static_cast<size_t>(row_g) * p.H + head) * D + 64 * g;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
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
      if (g == 0 && p.lse != nullptr && live)
        p.lse[static_cast<size_t>(head) * p.T_q + row_g] =
            (m2 + __log2f(l_row)) * 0.69314718056f;
    }
  } else if (!skip && warp == 8) {
    // ----------------------------------------------------------------------- TMA producer
    // K half: keys [128 j + 64 rank, +64), both head-dim halves; V half: keys [128 j, +128),
    // head-dim columns [64 rank, +64).  Boxes never cross a page.  Every load completes on a
    // barrier of this CTA; warp 10 relays each landed tile to the leader.
    const int Rk = p.box_rows, nbk = 64 / Rk;          // <= 4
    const int Rv = p.box_rows_v, nbv = 128 / Rv;       // <= 8
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar(L::B_QL), L::QTILE);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        tma_load_3d(base + L::Q_OFF + h * QHALF, &p.tm_q, 64 * h, head, m0, bar(L::B_QL));
    }
    int* const pt_s = reinterpret_cast<int*>(base_ptr + L::PT_OFF);
    const int n_cached = cache_page_table(p, pt_s, n_max, lane);
    auto page_row = [&](int tok) -> int {
      if (tok >= n_max) return p.total_rows;           // past the pool: TMA fills zeros
      return pool_row(p, pt_s, n_cached, tok);
    };
    int issued = 0;
    for (int j = 0; j < nk && ok; ++j) {
      // lanes 0..nbk-1 resolve the K boxes, lanes 8..8+nbv-1 the V boxes
      int coord = p.total_rows;
      if (lane < nbk) coord = page_row(j * BN + 64 * static_cast<int>(rank) + lane * Rk);
      else if (lane >= 8 && lane < 8 + nbv) coord = page_row(j * BN + (lane - 8) * Rv);
      int ck[4], cv[8];
#pragma unroll
      for (int b = 0; b < 4; ++b) ck[b] = __shfl_sync(0xffffffffu, coord, b);
#pragma unroll
      for (int b = 0; b < 8; ++b) cv[b] = __shfl_sync(0xffffffffu, coord, 8 + b);
      if (lane == 0) {
        const int itk = 2 * j, sk = itk % NS;
        ok = mbar_wait_cl(bar(L::B_KVE + sk), ((itk / NS) & 1) ^ 1, w);
        if (ok) {
          mbar_arrive_expect_tx(bar(L::B_KVL + sk), SLOT);
          const uint32_t dst = base + L::KV_OFF + sk * SLOT;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            if (b < nbk) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_3d(dst + h * KHALF + static_cast<uint32_t>(b * Rk * 128), &p.tm_k,
                            64 * h, head, ck[b], bar(L::B_KVL + sk));
            }
          }
          issued = itk + 1;
        }
        const int itv = 2 * j + 1, sv = itv % NS;
        if (ok) ok = mbar_wait_cl(bar(L::B_KVE + sv), ((itv / NS) & 1) ^ 1, w);
        if (ok) {
          mbar_arrive_expect_tx(bar(L::B_KVL + sv), SLOT);
          const uint32_t dst = base + L::KV_OFF + sv * SLOT;
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            if (b < nbv)
              tma_load_3d(dst + static_cast<uint32_t>(b * Rv * 128), &p.tm_v,
                          64 * static_cast<int>(rank), head, cv[b], bar(L::B_KVL + sv));
          }
          issued = itv + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      // every load of this CTA must land before its shared memory is released
      mbar_wait_drain(bar(L::B_QL), 0);
      for (int it = issued - 1; it >= 0 && it >= issued - NS; --it)
        mbar_wait_drain(bar(L::B_KVL + it % NS), (it / NS) & 1);
    }
  } else if (!skip && warp == 10) {
    // --------------------------------------------------------------------- load relay
    // Waits for each of this CTA's loads on its local barrier and arrives on the leader's
    // barrier, so the leader's MMA knows both halves have landed.  Before releasing the last
    // V tile it zeroes the rows past the last visible key (they may hold NaN, which 0 * NaN
    // would spread through P.V).
    bool ok = true;
    if (lane == 0) ok = mbar_wait_cl(bar(L::B_QL), 0, w);
    if (lane == 0 && ok) {
  if (rank == 0) mbar_arrive(bar(L::B_Q));
  else mbar_arrive_cluster(lead(L::B_Q));
}
    ok = __shfl_sync(0xffffffffu, ok, 0);
    const int zero_from = n_max - (nk - 1) * BN;
    for (int it = 0; ok && it < 2 * nk; ++it) {
      const int slot = it % NS;
      if (lane == 0) ok = mbar_wait_cl(bar(L::B_KVL + slot), (it / NS) & 1, w);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (it == 2 * nk - 1 && zero_from < BN) {
        const uint32_t vb = base + L::KV_OFF + slot * SLOT;
        for (int i = lane; i < (BN - zero_from) * 8; i += 32)
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                           vb + static_cast<uint32_t>(zero_from * 128 + i * 16)),
                       "r"(0u)
                       : "memory");
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
  if (rank == 0) mbar_arrive(bar(L::B_KVF + slot));
  else mbar_arrive_cluster(lead(L::B_KVF + slot));
}
    }
  } else if (!skip && warp == 9 && lane == 0 && rank == 0) {
    // ------------------------------------------------------------------ MMA issuer (pair)
    constexpr uint32_t idesc_qk = idesc_bf16_f32(256, BN, 0, 0);   // Q, K both K-major
    constexpr uint32_t idesc_pv = idesc_bf16_f32(256, D, 0, 1);    // P (TMEM), V MN-major
    const uint64_t dq0 = smem_desc_sw128(base + L::Q_OFF, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(base + L::KV_OFF, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(base + L::KV_OFF, KHALF, 1024);
    bool ok = mbar_wait_cl(bar(L::B_Q), 0, w);

    auto issue_s = [&](int j) -> bool {   // S(j) = Q K_j^T into S buffer j mod 3
      const int it = 2 * j, slot = it % NS, b = j % NB;
      if (!mbar_wait_cl(bar(L::B_KVF + slot), (it / NS) & 1, w)) return false;
      if (j >= NB && !mbar_wait_cl(bar(L::B_O + b), ((j - NB) / NB) & 1, w)) return false;
      tc_fence_after();
      const uint64_t dk = dk0 + ((static_cast<uint32_t>(slot) * SLOT) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_pair(tmem + static_cast<uint32_t>(128 * b),
                     dq0 + (((kk / 4) * QHALF + (kk % 4) * 32) >> 4),
                     dk + (((kk / 4) * KHALF + (kk % 4) * 32) >> 4), idesc_qk, kk > 0 ? 1u : 0u);
      umma_commit_pair(mine(L::B_S + b));
      umma_commit_pair(other(L::B_S + b));
      umma_commit_pair(mine(L::B_KVE + slot));
      umma_commit_pair(other(L::B_KVE + slot));
      return true;
    };
    auto issue_pv = [&](int j) -> bool {  // O += P(j) V_j
      const int it = 2 * j + 1, slot = it % NS, b = j % NB;
      if (!mbar_wait_cl(bar(L::B_KVF + slot), (it / NS) & 1, w)) return false;
      if (!mbar_wait_cl(bar(L::B_P + b), (j / NB) & 1, w)) return false;
      tc_fence_after();
      const uint64_t dv = dv0 + ((static_cast<uint32_t>(slot) * SLOT) >> 4);
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk)
        umma_ts_pair(tmem + 384u, tmem + static_cast<uint32_t>(128 * b + 8 * kk),
                     dv + ((kk * 2048u) >> 4), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      umma_commit_pair(mine(L::B_O + b));
      umma_commit_pair(other(L::B_O + b));
      umma_commit_pair(mine(L::B_KVE + slot));
      umma_commit_pair(other(L::B_KVE + slot));
      return true;
    };
    // S runs two tiles ahead of P.V: the tensor pipe holds S(j+1) and S(j+2) while the
    // softmax works on tile j+1.
    for (int j = 0; ok && j < 2 && j < nk; ++j) ok = issue_s(j);
    for (int j = 0; ok && j < nk; ++j) {
      ok = issue_pv(j);
      if (ok && j + 2 < nk) ok = issue_s(j + 2);
    }
    umma_commit_pair(mine(L::B_DRAIN));
    mbar_wait_drain(bar(L::B_DRAIN), 0);
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // no CTA leaves while the pair's MMAs or remote arrivals may touch it
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace wfk
