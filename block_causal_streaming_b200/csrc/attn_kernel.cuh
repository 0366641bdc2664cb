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
// non-decreasing in the query row, so blockIdx 0 takes the last 256 rows.  Heads vary fastest
// within groups of a few heads (the host picks the group size), so the CTAs of a group stream
// the same key range at about the same time and share it in L2.
//
// Warp roles (384 threads):
//   warps 0-3  softmax of Q tile 0: thread t owns query row t (TMEM lane t)
//   warps 4-7  softmax of Q tile 1
//   warp  8    TMA producer of Q (once) and of K_j (128 keys each) into the K ring, page by page
//              through the page table; allocates/frees TMEM
//   warp  9    QK^T issuer (one thread): S_q = Q_q K_j^T (SS form)
//   warp 10    P.V issuer (one thread): O_q += P_q V_j (TS form, P in TMEM)
//   warp 11    TMA producer of V_j into the V ring; zeroes the rows of the last V tile past
//              the last visible key
// Two issuing threads because one thread's chain of MMAs into one accumulator runs well below
// the tensor core's rate, and two independent chains in flight reach it; two producers because
// the P.V thread trails the QK^T thread by the softmax, so V slots are held longer than K slots.
// With key splits a unit runs as several CTAs, each over a consecutive part of its key tiles
// (AttnParams::n_splits, n_tail).
// TMEM (512 columns): one S buffer at [0, 128) that the two Q tiles take turns in (128 fp32
// columns), P_q at [128 + 64 q, 192 + 64 q) (bf16 pairs) and O_q at [256 + D q, 256 + D q + D).
//
// Why P has its own columns.  With P written over its own S, QK^T of tile j+1 for a Q tile can
// only start once P.V of tile j has read P, so every Q tile runs the chain softmax -> P.V ->
// QK^T -> softmax and the tensor pipe waits on the softmax's whole latency.  TMEM cannot hold two
// S buffers, two P buffers and two O accumulators at head_dim 128, so the two Q tiles share one
// S buffer instead: the softmax of a tile hands the buffer back as soon as it has read S into
// registers, and the next QK^T -- of the other Q tile -- starts then, while the softmax is still
// computing P.  A QK^T never waits for a P.V.
//
// Issue order: the QK^T thread issues S_0(0), S_1(0), S_0(1), S_1(1), ...; S_1(j) waits until
// softmax 0 has read S_0(j), S_0(j+1) until softmax 1 has read S_1(j).  The P.V thread issues
// P.V_0(0), P.V_1(0), P.V_0(1), ...; P.V_q(j) waits for P_q(j).  The softmax of tile j writes
// P_q(j) only after P.V_q(j-1) -- which reads P_q(j-1) from the same columns -- has completed;
// it was issued a tile earlier, so that wait is short.
//
// Synchronisation (all mbarriers, all waits bounded):
//   q_full          TMA -> MMA          Q tiles landed
//   kv_full[s]      TMA -> MMA          K or V tile landed in slot s
//   kv_empty[s]     MMA commit -> TMA   slot s free again (both Q tiles' MMAs on it completed;
//                                       K slots freed by the QK^T thread, V slots by the P.V one)
//   s_full[q]       MMA commit -> softmax q   S_q of the current tile ready in the S buffer
//   s_free          softmax -> MMA      the S buffer has been read (one phase per S tile, the
//                                       two Q tiles alternating; one arrival per warp)
//   p_full[q]       softmax q -> MMA    P_q written to TMEM (and O_q rescaled if needed)
//   o_done[q]       MMA commit -> softmax q   P.V_q of the previous tile completed (P_q free,
//                                             O rescale, epilogue)
//   v_zeroed        TMA warp -> MMA     tail rows of the last V tile zeroed
#pragma once

#include <cuda_bf16.h>

#include <cfloat>

#include "sm100.cuh"

namespace wfk {

constexpr int kBM = 128;        // query rows per Q tile (UMMA M)
#ifndef WF_KV_RING_KB
#define WF_KV_RING_KB 160   // K/V ring: 5 tiles of 32 KB at head_dim 128
#endif
constexpr int kBN = 128;        // keys per K/V tile (UMMA N of QK^T, K of P.V)
constexpr int kNQT = 2;         // Q tiles per CTA
constexpr int kAttnThreads = 384;
#ifndef WF_K_SLOTS
#define WF_K_SLOTS 0      // K slots of the K/V ring; 0: half of the slots, rounded down
#endif
#ifndef WF_REG_SOFTMAX
#define WF_REG_SOFTMAX 200
#endif
// Register split: the kernel launches with 168 per thread (384 x 168 = 64512); the two softmax
// warpgroups take kRegSoftmax each and the producer/MMA warpgroup keeps the rest.
constexpr int kRegSoftmax = WF_REG_SOFTMAX;
constexpr int kRegOther = 3 * 168 - 2 * kRegSoftmax;
static_assert(kRegSoftmax % 8 == 0 && kRegOther % 8 == 0 && kRegOther >= 24,
              "setmaxnreg counts are multiples of 8");
static_assert(2 * 128 * kRegSoftmax + 128 * kRegOther <= 384 * 168, "split exceeds the launch");
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
  int head_group;     // heads per group of the dispatch order (divides H)
  float sl2;  // scale * log2(e)
  unsigned launch_id;
  int nqc;                          // non-empty query chunks
  int qc_row_end[kMaxQChunks];      // exclusive end row of query chunk i (query-row space)
  int qc_kv_end[kMaxQChunks];       // number of visible keys for rows of query chunk i
  // Key splits: every unit runs as n_splits CTAs over consecutive parts of its key tiles -- the
  // last n_tail units (in dispatch order) as n_splits + 1 -- and a unit with more than one part
  // writes, per part, its normalised partial output and log-sum-exp instead of `out`.
  int n_splits;
  int n_tail;
  float* part_o;                    // fp32 [parts][T_q][H][D], parts = n_splits (+1 with a tail)
  float* part_lse;                  // fp32 [parts][H][T_q], natural log; -inf: no key seen
  // Published chunks (one-way K/V publication between GPUs): with flags != null the keys of
  // chunk c are loaded only after flags[c] has reached flag_gen.  chunk_end[c]: exclusive end
  // token of chunk c in the logical key order.
  const unsigned* flags;
  unsigned flag_gen;
  int nchunks;
  int chunk_end[kMaxQChunks];
  // 8-bit tiers (kI8; kE4M3 for e4m3): tm_q / tm_k describe the 8-bit Q and K codes
  // ([rows][H][D], K contiguous in logical key order), with one scale per (128 rows, head):
  // q_scale [H][nqt], k_scale [H][nkb].
  const float* q_scale;
  const float* k_scale;
  int nqt, nkb;
};

__device__ __forceinline__ int kv_end_of_row(const AttnParams& p, int r) {
  for (int c = 0; c < p.nqc; ++c)
    if (r < p.qc_row_end[c]) return p.qc_kv_end[c];
  return p.qc_kv_end[p.nqc - 1];
}

// Physical pool row of logical token `tok` (< n_max); entries outside the pool are recorded
// as WF_ERR_PAGE_OOB and read as page 0.
__device__ __forceinline__ int pool_row(const AttnParams& p, int tok) {
  const int idx = tok / p.page_size;
  int pg = __ldg(p.page_table + idx);
  if (pg < 0 || pg >= p.num_pages) {
    atomicCAS(p.status, 0, 5 /* WF_ERR_PAGE_OOB */);
    pg = 0;
  }
  return pg * p.page_size + (tok - idx * p.page_size);
}

// Wait on a phase with only a timeout (no abort check): used to drain in-flight async work
// before shared memory or TMEM is released.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity))
    if (globaltimer_ns() - t0 > kDrainTimeoutNs) return false;
  return true;
}

// kI8: Q and K tiles hold 8-bit codes (int8 or e4m3; one 128-byte row per query / key at
// head_dim 128), V stays bf16; the 32 KB Q saves go to a sixth ring slot.
template <int D, bool kI8 = false>
struct AttnSmem {
  static constexpr int BN = kBN;
  static constexpr int DH = D / 64;                      // 128-byte halves of a bf16 row
  static constexpr int NS = (WF_KV_RING_KB + (kI8 ? 32 : 0)) * 1024 / (int)(DH * BN * 128);
  // Slots [0, NSK) hold K tiles, [NSK, NS) V tiles: two rings, each filled by its own producer
  // warp, so K loads never wait behind V tiles that the later P.V still holds.
  static constexpr int NSK = WF_K_SLOTS > 0 ? WF_K_SLOTS : NS / 2, NSV = NS - NSK;
  static_assert(NSK >= 1 && NSV >= 1, "each ring needs a slot");
  static constexpr uint32_t QHALF = kBM * 128u;          // 128 rows x 128 B, 128B-swizzled
  static constexpr uint32_t QTILE = kI8 ? QHALF : DH * QHALF;
  static constexpr uint32_t KBYTES = kI8 ? BN * 128u : DH * BN * 128u;   // bytes a K tile loads
  static constexpr uint32_t KHALF = BN * 128u;           // BN rows x 128 B
  static constexpr uint32_t KTILE = DH * KHALF;          // one K or V tile
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = Q_OFF + kNQT * QTILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NS * KTILE;
  // barrier indices; per-Q-tile barriers at base + q
  static constexpr int B_Q = 0, B_KVF = 1, B_KVE = 1 + NS, B_S = 1 + 2 * NS,
                       B_P = B_S + kNQT, B_O = B_P + kNQT, B_DRAIN = B_O + kNQT,
                       B_VZ = B_DRAIN + 2, B_SF = B_VZ + 1, NBAR = B_SF + 1;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;        // slack for 1024-byte alignment
  static_assert(ALLOC <= 227u * 1024u, "shared memory per CTA exceeds 227 KB");
};

// kWaitPublished: wait for the publication flags of the chunks (AttnParams::flags) before
// loading their keys; a separate instantiation so the plain kernel carries none of that code.
// kI8: the INT8 tier -- S = Q_i8 K_i8^T on the tensor core (kind::i8, s32 in TMEM), each S tile
// scaled by scale_q x scale_k in the softmax; P and P.V as in the bf16 kernel.
// kE4M3 (with kI8): the FP8 tier -- the 8-bit Q and K codes are e4m3, S = Q K^T by kind::f8f6f4
// with fp32 accumulation; scales, P and P.V as in the INT8 tier.
template <int D, bool kWaitPublished = false, bool kI8 = false, bool kE4M3 = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    wf_attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  static_assert(!kI8 || (D == 128 && !kWaitPublished), "the INT8 tier runs head_dim 128");
  static_assert(!kE4M3 || kI8, "the FP8 tier is an 8-bit tier");
  using L = AttnSmem<D, kI8>;
  constexpr int BN = L::BN, DH = L::DH, NS = L::NS;
  constexpr uint32_t QTILE = L::QTILE, QHALF = L::QHALF, KTILE = L::KTILE, KHALF = L::KHALF;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + L::MISC_OFF);
  volatile int* const cta_abort = reinterpret_cast<volatile int*>(base_ptr + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return base + L::BAR_OFF + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // unit, part and parts of this CTA: (U - n_tail) units of n_splits parts, then n_tail units
  // of n_splits + 1
  const int n_plain = p.n_pairs * p.H - p.n_tail;
  const int b_id = static_cast<int>(blockIdx.x);
  int unit, split, n_parts;
  if (b_id < n_plain * p.n_splits) {
    n_parts = p.n_splits;
    unit = b_id / n_parts;
    split = b_id - unit * n_parts;
  } else {
    n_parts = p.n_splits + 1;
    const int t = b_id - n_plain * p.n_splits;
    unit = n_plain + t / n_parts;
    split = t - (unit - n_plain) * n_parts;
  }
  // Heads are dispatched in groups of head_group: every row block of one group, longest first,
  // heads fastest, before the next group -- so many CTAs read one head's keys at about the same
  // time, whatever H is.
  const int group_units = p.n_pairs * p.head_group;
  const int group = unit / group_units, in_group = unit - group * group_units;
  const int pair = p.n_pairs - 1 - in_group / p.head_group;
  const int head = group * p.head_group + in_group % p.head_group;
  const int m0 = pair * (kNQT * kBM);
  const int last_row = min(m0 + kNQT * kBM, p.T_q) - 1;
  const int n_max = kv_end_of_row(p, last_row);        // keys any row of this unit may see
  const int n_tiles = (n_max + BN - 1) / BN;           // key tiles of the unit
  // This CTA's part of them: tiles [kb, kb + nk).  The host keeps n_parts <= n_tiles of every
  // unit, so nk >= 1.  Tile j below is local; its keys start at (kb + j) * BN.
  const int kb = static_cast<int>(static_cast<int64_t>(split) * n_tiles / n_parts);
  const int nk = static_cast<int>(static_cast<int64_t>(split + 1) * n_tiles / n_parts) - kb;

  const WaitCtx w{cta_abort, p.grid_abort, p.status, p.launch_id, 6 /* WF_ERR_TIMEOUT */,
                  kWaitTimeoutNs};

  if (threadIdx.x == 0) {
    *cta_abort = (*reinterpret_cast<volatile unsigned*>(p.grid_abort) == p.launch_id) ? 1 : 0;
    for (int i = 0; i < L::NBAR; ++i)
      mbar_init(bar(i), (i >= L::B_P && i < L::B_O) ? 128u : i == L::B_SF ? 4u : 1u);
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
  // Registers: see kRegSoftmax; the build checks the 168 the split relies on.

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax) : "memory");
    if (!skip) {
      // ------------------------------------------------------------------ softmax warpgroups
      const int q = warp >> 2, wq = warp & 3;
      const int row = wq * 32 + lane;                       // row within the Q tile == TMEM lane
      const int row_g = m0 + q * kBM + row;                 // query row
      const int n_r = kv_end_of_row(p, min(row_g, p.T_q - 1));
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tS = tmem + lane_off;                               // the shared S buffer
      const uint32_t tP = tmem + lane_off + 128u + static_cast<uint32_t>(q * 64);
      const uint32_t tO = tmem + lane_off + 256u + static_cast<uint32_t>(q * D);
      const float sl2 = kI8 ? p.sl2 * __ldg(p.q_scale + head * p.nqt + (m0 + q * kBM) / kBM)
                            : p.sl2;
      float m2 = -INFINITY;   // running max of the base-2 logits in use
      float l = 0.f;          // running sum of exp2(t - m2)
      bool ok = true;
      float2 sl2x2 = make_float2(sl2, sl2);
      for (int j = 0; j < nk; ++j) {
        // INT8 tier: the tile's K scale is loaded before the wait for S, which hides its latency
        const float dk = kI8 ? __ldg(p.k_scale + head * p.nkb + kb + j) : 0.f;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_S + q), j & 1, w));
        if (!ok) break;
        tc_fence_after();
        float s[BN];
        {
          uint32_t r[BN];
  #pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            tmem_ld32(tS + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
          tmem_wait_ld();
          // S is in registers: the buffer goes to the other Q tile's QK^T (one arrival per warp)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::B_SF));
          if (kI8 && !kE4M3) {
            // s32 -> fp32, exact: |S| <= 128 x 127^2 < 2^24.  (Reading the bits of
            // 1.5 x 2^23 + S as a float and subtracting 1.5 x 2^23 measured 3 % slower.)
  #pragma unroll
            for (int c = 0; c < BN; ++c) s[c] = static_cast<float>(static_cast<int>(r[c]));
          } else {
  #pragma unroll
            for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(r[c]);
          }
        }
        float tsl2 = sl2;     // logit scale of this tile
        if (kI8) {
          // scale_q x scale_k x scale x log2 e; a zero scale (a block of zeros) is kept
          // positive so masked columns stay -inf rather than 0 x inf
          tsl2 = fmaxf(sl2 * dk, FLT_MIN);
          sl2x2 = make_float2(tsl2, tsl2);
        }
        const int lim = n_r - (kb + j) * BN;                // visible columns of this tile
        const bool masked = lim < BN;
        if (masked) {
  #pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
  #pragma unroll
        for (int c = 4; c < BN; c += 8) {
          mx0 = max3(mx0, s[c], s[c + 1]);
          mx1 = max3(mx1, s[c + 2], s[c + 3]);
          if (c + 4 < BN) mx2 = max3(mx2, s[c + 4], s[c + 5]);
          if (c + 6 < BN) mx3 = max3(mx3, s[c + 6], s[c + 7]);
        }
        const float tmax = max3(mx0, mx1, fmaxf(mx2, mx3)) * tsl2;
        // Move the reference max only when the new one exceeds it by more than 2^8: O and l both
        // stay expressed against the same stale reference, so O / l is unchanged, and every
        // exp2(t - m2) stays <= 256.
        const bool need = tmax > m2 + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m2 - tmax);                   // 0 on the first visible tile
          m2 = tmax;
        }
        // p = exp2(s * scale * log2 e - m2) two columns at a time, every exponential on the
        // MUFU unit (moving 1/8 or 2/8 of them to an FMA-pipe polynomial measured 3-10 % slower).
        // no visible key yet (possible in a later key split): every p is exactly 0
        const float mref = m2 == -INFINITY ? 0.f : m2;
        const float2 negm = make_float2(-mref, -mref);
        // The row sum l adds the weights as P.V uses them -- rounded to bf16 -- so O / l is a
        // convex combination of the visible values (V = 1 gives exactly 1).
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[BN / 2];
  #pragma unroll
        for (int i = 0; i < BN / 2; ++i) {
          const float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), sl2x2, negm);
          pk[i] = pack_bf16x2(ex2_approx(x.x), ex2_approx(x.y));
          acc[i & 3] = add_bf16x2(acc[i & 3], pk[i]);
        }
        if (j > 0) {
          // P.V_q(j-1) reads P_q(j-1) from the columns P_q(j) goes to, and O_q holds P.V of the
          // tiles < j once it has completed (it was issued a tile ago, so this rarely waits).
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_O + q), (j - 1) & 1, w));
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
            // rescale this warp's rows of O_q (threads whose max did not move multiply by 1)
  #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(tO + 32u * c, r);
              tmem_wait_ld();
  #pragma unroll
              for (int i = 0; i < 32; ++i)
                r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_st32(tO + 32u * c, r);
            }
          }
        }
        // P_q into its own 64 TMEM columns (bf16 pairs).
  #pragma unroll
        for (int h = 0; h < BN / 64; ++h)
          tmem_st32(tP + 32u * h, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * h]));
        l = l * alpha + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::B_P + q));
      }
      // ------------------------------------------------------------------------- epilogue
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_O + q), (nk - 1) & 1, w));
      if (ok) {
        // O / l: bf16 into `out`, or -- for one key split of a unit -- fp32 into the partials,
        // with O = 0 and lse = -inf when no key of the split is visible to the row.
        tc_fence_after();
        const bool part = n_parts > 1;
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const bool live = row_g < p.T_q;
        const size_t orow = static_cast<size_t>(row_g) * p.H + head;
        const size_t prow = static_cast<size_t>(split) * p.T_q * p.H + orow;
  #pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32u * c, r);
          tmem_wait_ld();
          if (live && part) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + 32 * c);
  #pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv_l,
                                   __uint_as_float(r[4 * i + 1]) * inv_l,
                                   __uint_as_float(r[4 * i + 2]) * inv_l,
                                   __uint_as_float(r[4 * i + 3]) * inv_l);
          } else if (live) {
            uint32_t pk[16];
  #pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                                  __uint_as_float(r[2 * i + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(p.out + orow * D + 32 * c);
  #pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        const float lse = l > 0.f ? (m2 + __log2f(l)) * 0.69314718056f : -INFINITY;
        if (live && part)
          p.part_lse[(static_cast<size_t>(split) * p.H + head) * p.T_q + row_g] = lse;
        else if (live && p.lse != nullptr)
          p.lse[static_cast<size_t>(head) * p.T_q + row_g] = lse;
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegOther) : "memory");
    if (!skip && (warp == 8 || warp == 11)) {
      // ------------------------------------------------------------------------ TMA producers
      // Warp 8 loads the Q tiles, then K_0, K_1, ... into the K ring; warp 11 loads V_0, V_1,
      // ... into the V ring and zeroes the rows of the last V tile past the last visible key.
      const int kv = warp == 8 ? 0 : 1;
      const int ns = kv ? L::NSV : L::NSK, s0 = kv ? L::NSK : 0;
      const int R = p.box_rows, nb = BN / R;             // page boxes per K/V tile (<= BN/16)
      bool ok = true;
      if (kv == 0 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        mbar_arrive_expect_tx(bar(L::B_Q), kNQT * QTILE);
  #pragma unroll
        for (int qt = 0; qt < kNQT; ++qt)
  #pragma unroll
          for (int h = 0; h < (kI8 ? 1 : DH); ++h)     // int8: one 128-byte box per row
            tma_load_3d(base + L::Q_OFF + qt * QTILE + h * QHALF, &p.tm_q, 64 * h, head,
                        m0 + qt * kBM, bar(L::B_Q));
      }
      if (kv == 1 && lane == 0) tma_prefetch_desc(&p.tm_v);
      const CUtensorMap* map = kv ? &p.tm_v : &p.tm_k;
      // Physical row of box b of tile t (past the pool -- TMA fills zeros -- beyond n_max).
      auto box_row = [&](int t, int b) -> int {
        const int tok = (kb + t) * BN + b * R;
        if (b >= nb || t >= nk || tok >= n_max) return p.total_rows;
        return pool_row(p, tok);
      };
      int ready = 0;                                        // chunks known to be published
      int issued = 0;                                       // tiles whose loads were issued
      // Lane b holds the pool row of box b of a tile, read from the page table one tile ahead
      // so that the read's latency overlaps the load before it.
      int coord_next = box_row(0, lane);
      for (int j = 0; j < nk && ok; ++j) {
        const int coord = coord_next;
        if (j + 1 < nk) coord_next = box_row(j + 1, lane);
        int cb[BN / 16];
  #pragma unroll
        for (int b = 0; b < BN / 16; ++b) cb[b] = __shfl_sync(0xffffffffu, coord, b);
        if (kWaitPublished && lane == 0) {
          // every chunk with a key in this tile must have been published
          const int last_key = min((kb + j + 1) * BN, n_max) - 1;
          const int ready0 = ready;
          while (ok && ready < p.nchunks && (ready == 0 ? 0 : p.chunk_end[ready - 1]) <= last_key) {
            ok = wait_flag(p.flags + ready, p.flag_gen, w);
            ++ready;
          }
          if (ready != ready0) fence_proxy_async_global();
        }
        if (lane == 0 && ok) {
          const int slot = s0 + j % ns;
          ok = mbar_wait(bar(L::B_KVE + slot), ((j / ns) & 1) ^ 1, w);
          if (ok) {
            const uint32_t dst = base + L::KV_OFF + slot * KTILE;
            if (kI8 && kv == 0) {
              // int8 K' codes are contiguous in logical key order: one box of BN keys
              mbar_arrive_expect_tx(bar(L::B_KVF + slot), L::KBYTES);
              tma_load_3d(dst, map, 0, head, (kb + j) * BN, bar(L::B_KVF + slot));
            } else {
              mbar_arrive_expect_tx(bar(L::B_KVF + slot), KTILE);
  #pragma unroll
              for (int b = 0; b < BN / 16; ++b) {
                if (b < nb) {
  #pragma unroll
                  for (int h = 0; h < DH; ++h)
                    tma_load_3d(dst + h * KHALF + static_cast<uint32_t>(b * R * 128), map,
                                64 * h, head, cb[b], bar(L::B_KVF + slot));
                }
              }
            }
            issued = j + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      const int zero_from = n_max - (kb + nk - 1) * BN;    // rows >= this of the last V tile
      if (kv == 1 && ok && zero_from < BN) {
        // Rows past the last visible key may hold anything (even NaN, which 0 * NaN would spread
        // through P.V); once the last V tile has landed, zero them and release the P.V thread.
        const int slot = s0 + (nk - 1) % ns;
        if (lane == 0) ok = mbar_wait(bar(L::B_KVF + slot), ((nk - 1) / ns) & 1, w);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
          const uint32_t vb = base + L::KV_OFF + slot * KTILE;
          const int n16 = (BN - zero_from) * 8;            // 16-byte pieces per 128-byte half
          for (int i = lane; i < n16 * DH; i += 32) {
            const int h = i / n16, rr = i % n16;
            const uint32_t a = vb + h * KHALF + static_cast<uint32_t>(zero_from * 128 + rr * 16);
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::B_VZ));
        }
      }
      if (lane == 0) {
        // every load this warp issued must land before shared memory is released: the last
        // issued tile of each slot (tiles were loaded in order)
        if (kv == 0) mbar_wait_drain(bar(L::B_Q), 0);
        for (int r = 0; r < ns && r < issued; ++r) {
          const int jl = issued - 1 - ((issued - 1 - r) % ns);   // last tile in slot s0 + r
          mbar_wait_drain(bar(L::B_KVF + s0 + jl % ns), (jl / ns) & 1);
        }
      }
    } else if (!skip && (warp == 9 || warp == 10) && lane == 0) {
      // ---------------------------------------------------------------------- MMA issuers
      // Two threads: warp 9 issues every QK^T, warp 10 every P.V.  A chain of MMAs into one
      // accumulator issued by one thread runs at about 88 cycles per 128 x 128 x 16 step for
      // QK^T (operands in SMEM) and 128 for P.V (P from TMEM), against 64 at the tensor core's
      // rate; two independent chains in flight together run at the full rate.  Descriptors are
      // built once; per instruction only a compile-time offset (16-byte units) is added to the
      // start-address field, so the issue loop stays a few instructions per MMA.
      constexpr uint32_t idesc_qk = kE4M3 ? idesc_e4m3_f32(kBM, BN)   // Q, K both K-major
                                    : kI8 ? idesc_s8_s32(kBM, BN)
                                          : idesc_bf16_f32(kBM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);     // P (TMEM), V MN-major
      const uint64_t dq0 = smem_desc_sw128(base + L::Q_OFF, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(base + L::KV_OFF, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(base + L::KV_OFF, KHALF, 1024);
      bool ok = true;
      constexpr int NSK = L::NSK, NSV = L::NSV;
      if (warp == 9) {
        // S(j, q) = Q_q K_j^T into the shared S columns: D/16 K-steps of 16 columns (4 per
        // 128-byte half of a row; INT8: D/32 steps of 32).  S(j, 0) waits for K_j and, after
        // the first tile, for softmax 1 to have read S_1(j-1); S(j, 1) for softmax 0 to have
        // read S_0(j).
        constexpr int kSteps = kI8 ? D / 32 : D / 16;
        auto issue_s = [&](int j, int q) {
          const int slot = j % NSK;
          const uint64_t dk = dk0 + ((static_cast<uint32_t>(slot) * KTILE) >> 4);
          const uint64_t dq = dq0 + ((static_cast<uint32_t>(q) * QTILE) >> 4);
  #pragma unroll
          for (int kk = 0; kk < kSteps; ++kk) {
            if (kE4M3)
              umma_ss_f8(tmem, dq + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), idesc_qk,
                         kk > 0 ? 1u : 0u);
            else if (kI8)
              umma_ss_i8(tmem, dq + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), idesc_qk,
                         kk > 0 ? 1u : 0u);
            else
              umma_ss(tmem, dq + (((kk / 4) * QHALF + (kk % 4) * 32) >> 4),
                      dk + (((kk / 4) * KHALF + (kk % 4) * 32) >> 4), idesc_qk,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(L::B_S + q));
        };
        int sf = 0;           // S-free phases consumed: one per S tile read by a softmax
        ok = mbar_wait(bar(L::B_Q), 0, w);
        for (int j = 0; ok && j < nk; ++j) {
          ok = mbar_wait(bar(L::B_KVF + j % NSK), (j / NSK) & 1, w);
          if (ok && j > 0) ok = mbar_wait(bar(L::B_SF), (sf++) & 1, w);
          if (!ok) break;
          tc_fence_after();
          issue_s(j, 0);
          ok = mbar_wait(bar(L::B_SF), (sf++) & 1, w);
          if (!ok) break;
          tc_fence_after();
          issue_s(j, 1);
          umma_commit(bar(L::B_KVE + j % NSK));                  // K_j free
        }
      } else {
        // PV(j, q): O_q += P_q(j) V_j (BN/16 K-steps, P_q in its own TMEM columns), once V_j
        // has landed (tail rows zeroed for the last tile) and P_q(j) is written.
        const bool zero_tail = (n_max - (kb + nk - 1) * BN) < BN;   // the loader zeroes V's tail
        auto issue_pv = [&](int j, int q) {
          const int slotv = NSK + j % NSV;
          const uint64_t dv = dv0 + ((static_cast<uint32_t>(slotv) * KTILE) >> 4);
          const uint32_t pa = tmem + 128u + static_cast<uint32_t>(q * 64);
          const uint32_t od = tmem + 256u + static_cast<uint32_t>(q * D);
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ts(od, pa + 8u * kk, dv + ((kk * 2048u) >> 4), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(L::B_O + q));
        };
        for (int j = 0; ok && j < nk; ++j) {
          ok = mbar_wait(bar(L::B_KVF + NSK + j % NSV), (j / NSV) & 1, w);
          if (ok && j == nk - 1 && zero_tail) ok = mbar_wait(bar(L::B_VZ), 0, w);
          if (ok) ok = mbar_wait(bar(L::B_P + 0), j & 1, w);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j, 0);
          ok = mbar_wait(bar(L::B_P + 1), j & 1, w);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j, 1);
          umma_commit(bar(L::B_KVE + NSK + j % NSV));            // V_j free
        }
      }
      // every MMA this thread issued must complete before TMEM is released
      umma_commit(bar(L::B_DRAIN + (warp - 9)));
      mbar_wait_drain(bar(L::B_DRAIN + (warp - 9)), 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace wfk
