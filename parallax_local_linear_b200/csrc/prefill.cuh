// Parallax causal prefill on sm_100a: TMA, tcgen05.mma, tensor memory.
//
// Every position t of a sequence is a query with probe rho_t over keys 0..t
// (causal, diagonal included) or over all keys.  Per query row the kernel
// keeps the running max m and l = sum e, c = sum e*a, O1 = sum e v,
// O2 = sum e*a v with e = exp(scale q.k - m), a = rho.k - a_ref, and writes
// out = (O1/l)(1 + c/l) - O2/l, which equals vbar - S_KV^T rho (the
// covariance correction of the wispaper.ai blog "Parallax: Breaking the
// Boundary Bias with Parameterized Local Linear Attention", section "The Core
// Insight: Covariance Correction"; computed in a single pass, as in its
// "Hardware Efficiency" section).  a_ref = rho_t.k_0, read from the first key
// tile (key 0 is visible to every row).
//
// The four products are dense contractions and run on the tensor cores:
//     S  = Q K^T,    A  = R K^T            (128 x 64 per key tile, fp32 in TMEM)
//     O1 += P V,     O2 += (P o A') V      (128 x 128, fp32 in TMEM)
// with P = exp2(S * scale * log2(e) - m) and A' = A - a_ref.
//
// CTA = one 128-row query tile of one (sequence, head); key tiles of 64.
// Warp roles (320 threads):
//   warp 0       TMA producer: Q and R once, then separate K and V rings.
//   warp 1       TMEM allocator; lane 0 issues every tcgen05.mma.
//   warps 2..9   softmax, two warpgroups.  Thread = query row = TMEM lane;
//                warpgroup g takes the key tiles j = g, g+2, ... (all 64
//                columns), forms P and P o A' in bf16 and writes them back
//                over its S and A buffer (the A operand of the value
//                products comes straight from TMEM).  The two warpgroups
//                work on consecutive tiles at once, so one's exponentials
//                overlap the other's loads, reductions and waits.  The
//                reference max of P passes from tile j-1's warpgroup to
//                tile j's through shared memory and an mbarrier; when it
//                grows by more than 2^8, that warpgroup rescales O1 and O2.
//                At the end warpgroup g writes output columns 64g..64g+63.
//
// TMEM columns (512 x 128 lanes x 32 bit): O1 [0,128), O2 [128,256), and two
// buffers of S / A: S_b at 256 + 128 b, A_b at 320 + 128 b (buffer b holds
// the tiles of warpgroup b).  While a warpgroup works on tile j, the tensor
// cores run the value products of tile j-1 and the score products of tile
// j+1, which the other warpgroup takes up as soon as they land.
//
// Two forms of the same kernel:
//   dense   q, rho [B, H, T, d]; k, v [B, Hkv, T, d]; every position a query.
//   paged   chunked (append) prefill: sequence b holds L_b = seq_lens[b] keys
//           in 64-token pages of a pool [P, Hkv, 64, d]; its q_len_b queries
//           are packed at rows cu_q[b] .. cu_q[b+1]-1 of q, rho, out
//           [total_q, H, d] and sit at the LAST positions L_b - q_len_b ..
//           L_b - 1 of the sequence (their keys are already in the cache).
//           A key tile is one page.  The unused tail of a sequence's last
//           page may hold anything, NaN included: masked columns get s = -inf
//           and a = 0 (a select, since 0 * NaN is NaN), and the softmax warps
//           zero those V rows in shared memory before the value products.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace plx {

constexpr int kPfBM = 128;        // query rows per CTA (= TMEM lanes)
constexpr int kPfBN = 64;         // keys per tile
constexpr int kPfD = 128;         // head dim
#ifndef PLX_PREFILL_STAGES
#define PLX_PREFILL_STAGES 4
#endif
// Depth of each of the K and V rings.  A key tile must be in flight for the
// L2 latency (~1.5 us) while the tensor cores work through the tiles ahead
// of it, and K and V are released separately (K after the score products,
// V after the value products), so each ring keeps several tiles in flight.
constexpr int kPfStages = PLX_PREFILL_STAGES;
constexpr int kPfThreads = 320;   // producer warp, MMA warp, two softmax warpgroups
constexpr int kPfSoftmax = 256;   // softmax threads
constexpr float kPfRescaleLog2 = 8.f;   // lazy rescale threshold (factor 256)
// Key tiles whose P and P o A' also enter the value products as bf16 lo parts
// (x = bf16(x) + lo), in query tiles whose rows see fewer than 128 keys.  A
// row with few keys has nothing to average the bf16 rounding of P o A' (|a|
// reaches ~10 for unit-scale probes) over; such rows' keys all lie in tiles
// 0 and 1.  Rows with 128 keys or more average it out.
#ifndef PLX_PREFILL_SPLIT_TILES
#define PLX_PREFILL_SPLIT_TILES 2
#endif
constexpr int kPfSplitTiles = PLX_PREFILL_SPLIT_TILES;

struct PrefillArgs {
  int B, H, Hkv, T, group;
  int n_mblk;                     // ceil(T / 128) (dense), ceil(max q_len / 128) (paged)
  int causal, out_bf16;
  float scale_log2;               // scale * log2(e), > 0
  void* out;                      // [B, H, T, D] (dense), [total_q, H, D] (paged)
  // paged form only
  const int32_t* cu_q;            // [B + 1] first packed query row of each sequence
  const int32_t* seq_lens;        // [B] keys of each sequence, its queries included
  const int32_t* page_table;      // [B, max_pages] physical page of each 64-key tile
  int max_pages, num_pages, total_q, max_q;
  // dense form, training: per-row quantities the backward pass reads (null: not written)
  float* vbar;                    // [B, H, T, D]: vbar = O1 / l
  float2* stats;                  // [B, H, T]: (m + log2 l, abar = c / l), weights w = 2^(s*scale*log2(e) - x)
  unsigned long long wait_ns;     // limit of one pipeline wait (0: give up unless complete)
};

// Four MMAs under one elect.sync: the issuing warp spends fewer instructions
// per MMA, which matters when it shares its sub-partition with busy warps
// (the tensor pipe's queue is short, so a late issue leaves it idle).
// MMAs 0 and 1 take accumulate flag acc01, MMAs 2 and 3 acc23.
__device__ __forceinline__ void tc_mma_ss4(uint32_t d0, uint64_t a0, uint64_t b0, uint32_t d1, uint64_t a1,
                                           uint64_t b1, uint32_t d2, uint64_t a2, uint64_t b2, uint32_t d3,
                                           uint64_t a3, uint64_t b3, uint32_t idesc, uint32_t acc01,
                                           uint32_t acc23) {
  asm volatile(
      "{\n\t.reg .pred p01, p23, e;\n\tsetp.ne.b32 p01, %13, 0;\n\tsetp.ne.b32 p23, %14, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], %4, %5, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%6], %7, %8, %12, p23;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%9], %10, %11, %12, p23;\n\t}" ::"r"(d0),
      "l"(a0), "l"(b0), "r"(d1), "l"(a1), "l"(b1), "r"(d2), "l"(a2), "l"(b2), "r"(d3), "l"(a3), "l"(b3),
      "r"(idesc), "r"(acc01), "r"(acc23)
      : "memory");
}

__device__ __forceinline__ void tc_mma_ts4(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t d1, uint32_t a1,
                                           uint64_t b1, uint32_t d2, uint32_t a2, uint64_t b2, uint32_t d3,
                                           uint32_t a3, uint64_t b3, uint32_t idesc, uint32_t acc01,
                                           uint32_t acc23) {
  asm volatile(
      "{\n\t.reg .pred p01, p23, e;\n\tsetp.ne.b32 p01, %13, 0;\n\tsetp.ne.b32 p23, %14, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], [%4], %5, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%6], [%7], %8, %12, p23;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%9], [%10], %11, %12, p23;\n\t}" ::"r"(d0),
      "r"(a0), "l"(b0), "r"(d1), "r"(a1), "l"(b1), "r"(d2), "r"(a2), "l"(b2), "r"(d3), "r"(a3), "l"(b3),
      "r"(idesc), "r"(acc01), "r"(acc23)
      : "memory");
}

struct PfLayout {
  static constexpr int kQBytes = kPfBM * kPfD * 2;       // 32 KB: two 64-column boxes of 128 rows
  static constexpr int kKVBytes = kPfBN * kPfD * 2;      // 16 KB: two 64-column boxes of 64 rows
  static constexpr int kQ = 0;
  static constexpr int kR = kQ + kQBytes;
  static constexpr int kK = kR + kQBytes;
  static constexpr int kV = kK + kPfStages * kKVBytes;
  static constexpr int kBar = kV + kPfStages * kKVBytes;
  // barriers: q_full, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_full[2], o_done,
  // drain, hand[2] (hand[g]: the reference max for warpgroup g's next tile is in m_ref)
  static constexpr int kNumBars = 1 + 4 * kPfStages + 2 + 2 + 1 + 1 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;       // tmem base, abort flag
  static constexpr int kMref = kMisc + 16;                // float [128 rows]: reference max after the last tile
  static constexpr int kAref = kMref + 128 * 4;           // float [128]
  static constexpr int kLC = kAref + 128 * 4;             // float [2 warpgroups][128 rows][l, c, m]
  static constexpr int kBytes = kLC + 2 * 128 * 3 * 4 + 1024;   // + alignment slack
};

constexpr uint32_t kColO1 = 0, kColO2 = 128;
__device__ __forceinline__ uint32_t col_s(int b) { return 256u + 128u * b; }
__device__ __forceinline__ uint32_t col_a(int b) { return 320u + 128u * b; }

template <bool kPaged>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillArgs a) {
  using Ly = PfLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kPfStages;
  uint64_t* k_empty = v_full + kPfStages;
  uint64_t* v_empty = k_empty + kPfStages;
  uint64_t* s_full = v_empty + kPfStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 1;
  uint64_t* hand = drain + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::kMisc + 4);
  float* mref_s = reinterpret_cast<float*>(sm + Ly::kMref);
  float* aref_s = reinterpret_cast<float*>(sm + Ly::kAref);
  float* lc_s = reinterpret_cast<float*>(sm + Ly::kLC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest query tiles first: the last tile of every head, then the one before...
  const int BH = a.B * a.H;
  const int mblk = a.n_mblk - 1 - (int)(blockIdx.x / BH);
  const int bh = blockIdx.x % BH;
  const int b = bh / a.H, h = bh % a.H, kvh = h / a.group;
  const int m0 = mblk * kPfBM;
  // The sequence: q_len queries (first packed row q_first) at the last
  // positions pos0 .. pos0 + q_len - 1 of its L keys.  Dense: q_len = L = T.
  int q_len = a.T, L = a.T, q_first = 0;
  const int32_t* pt = nullptr;
  if constexpr (kPaged) {
    q_first = a.cu_q[b];
    q_len = a.cu_q[b + 1] - q_first;
    L = a.seq_lens[b];
    const bool bad = q_first < 0 || q_len < 0 || q_len > a.max_q ||
                     (long long)q_first + q_len > (long long)a.total_q || L < q_len ||
                     (long long)L > (long long)a.max_pages * kPfBN;
    if (bad) {   // uniform over the CTA: nothing below has run yet
      if (threadIdx.x == 0) report_error(4 /* PLX_DEVERR_BAD_LENGTH */);
      return;
    }
    if (m0 >= q_len) return;
    pt = a.page_table + (size_t)b * a.max_pages;
  }
  const int pos0 = L - q_len;
  const int kv_end = a.causal ? min(L, pos0 + m0 + kPfBM) : L;
  const int n = (kv_end + kPfBN - 1) / kPfBN;
  // Rows of this tile see at least min_keys keys; below 128 the bf16
  // rounding of P o A' is not averaged away, so the first tiles are split.
  const int min_keys = a.causal ? min(pos0 + m0 + 1, L) : L;
  const bool few_keys = min_keys < 2 * kPfBN;
  const int q_row = kPaged ? q_first + m0 : (b * a.H + h) * a.T + m0;
  const int kv_row = (b * a.Hkv + kvh) * a.T;   // dense form only
  if constexpr (kPaged) {
    // Every page this tile reads must lie in the pool.
    bool badp = false;
    for (int i = threadIdx.x; i < n; i += kPfThreads) {
      const int pg = pt[i];
      badp |= pg < 0 || pg >= a.num_pages;
    }
    if (__syncthreads_or(badp)) {
      if (threadIdx.x == 0) report_error(1 /* PLX_DEVERR_BAD_PAGE */);
      return;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kPfSoftmax / 2);
      mbar_init(&hand[i], kPfSoftmax / 2);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_r);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t keep = l2_policy_evict_last();   // K/V tiles are re-read by other query tiles
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, 2 * Ly::kQBytes);
      for (int bx = 0; bx < 2; ++bx) {
        if constexpr (kPaged) {   // [total_q, H, D]: box of 128 rows of one head
          tma_load_3d(sm + Ly::kQ + bx * (Ly::kQBytes / 2), &tm_q, bx * 64, h, q_row, q_full, once);
          tma_load_3d(sm + Ly::kR + bx * (Ly::kQBytes / 2), &tm_r, bx * 64, h, q_row, q_full, once);
        } else {
          tma_load_2d(sm + Ly::kQ + bx * (Ly::kQBytes / 2), &tm_q, bx * 64, q_row, q_full, once);
          tma_load_2d(sm + Ly::kR + bx * (Ly::kQBytes / 2), &tm_r, bx * 64, q_row, q_full, once);
        }
      }
      int issued = 0, issued_k = 0;   // V and K tiles issued
      for (int j = 0; j < n; ++j) {
        const int s = j % kPfStages;
        const uint32_t par = ((j / kPfStages) - 1) & 1;
        // pool rows [P * Hkv * 64] (paged; page ids checked above) or [B * Hkv * T]
        const int row = kPaged ? (pt[j] * a.Hkv + kvh) * kPfBN : kv_row + j * kPfBN;
        if (j >= kPfStages && !mbar_wait_bounded(a.wait_ns, &k_empty[s], par)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&k_full[s], Ly::kKVBytes);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_2d(sm + Ly::kK + s * Ly::kKVBytes + bx * (Ly::kKVBytes / 2), &tm_k, bx * 64, row, &k_full[s], keep);
        if (j >= kPfStages && !mbar_wait_bounded(a.wait_ns, &v_empty[s], par)) {
          *abort_flag = 1;
          ++issued_k;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], Ly::kKVBytes);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_2d(sm + Ly::kV + s * Ly::kKVBytes + bx * (Ly::kKVBytes / 2), &tm_v, bx * 64, row, &v_full[s], keep);
        ++issued;
        ++issued_k;
      }
      // Every issued load must land before the CTA exits.
      mbar_wait_drain(q_full, 0);
      for (int s = 0; s < kPfStages && s < issued_k; ++s) {
        const int last = s + ((issued_k - 1 - s) / kPfStages) * kPfStages;
        mbar_wait_drain(&k_full[s], (last / kPfStages) & 1);
      }
      for (int s = 0; s < kPfStages && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kPfStages) * kPfStages;
        mbar_wait_drain(&v_full[s], (last / kPfStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lockstep (every branch is warp-uniform);
    // one elected lane issues each tcgen05.mma / commit.
    constexpr uint32_t kIdS = idesc_bf16(kPfBM, kPfBN, false);   // 128 x 64, K-major B
    constexpr uint32_t kIdPV = idesc_bf16(kPfBM, kPfD, true);    // 128 x 128, MN-major B (V)
    // Descriptors of every operand base; a k-step adds its byte offset / 16.
    const uint64_t dq = smem_desc_sw128(smem_u32(sm + Ly::kQ), 16, 1024);
    const uint64_t dr = smem_desc_sw128(smem_u32(sm + Ly::kR), 16, 1024);
    const uint64_t dk = smem_desc_sw128(smem_u32(sm + Ly::kK), 16, 1024);
    const uint64_t dv = smem_desc_sw128(smem_u32(sm + Ly::kV), Ly::kKVBytes / 2, 1024);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, bar, parity));
    };
    bool ok = wait_warp(q_full, 0);
    tc_fence_after();
    for (int j = 0; ok && j <= n; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (j < n) {
        const int s = j % kPfStages, b2 = j & 1;
        if (!(ok = wait_warp(&k_full[s], (j / kPfStages) & 1))) break;
        tc_fence_after();
        const uint64_t dks = dk + (uint64_t)((s * Ly::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; kk += 2) {
          // 16 columns of d per step: box kk / 4, 32 bytes into the 128-byte row per
          // step; S and A of two steps per issue
          const uint64_t oq0 = (uint64_t)((kk >> 2) * (Ly::kQBytes / 2 / 16) + (kk & 3) * 2);
          const uint64_t ok0 = (uint64_t)((kk >> 2) * (Ly::kKVBytes / 2 / 16) + (kk & 3) * 2);
          const uint64_t oq1 = oq0 + 2, ok1 = ok0 + 2;   // kk + 1 stays in the same box
          tc_mma_ss4(tmem + col_s(b2), dq + oq0, dks + ok0, tmem + col_a(b2), dr + oq0, dks + ok0,
                     tmem + col_s(b2), dq + oq1, dks + ok1, tmem + col_a(b2), dr + oq1, dks + ok1, kIdS,
                     kk > 0 ? 1u : 0u, 1u);
        }
        tc_commit(&s_full[b2]);
        tc_commit(&k_empty[s]);   // K(j) is free once the score products are done
      }
      if (j >= 1) {
        const int jp = j - 1, bp = jp & 1, sp = jp % kPfStages;
        // V(j-1) landed long ago; waiting on it first keeps it off the path
        // from the softmax's arrival to the value products.
        if (!(ok = wait_warp(&v_full[sp], (jp / kPfStages) & 1))) break;
        if (!(ok = wait_warp(&p_full[bp], (jp >> 1) & 1))) break;
        tc_fence_after();
        const uint64_t dvs = dv + (uint64_t)((sp * Ly::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; kk += 2) {
          // 16 keys per step: 8 TMEM columns of packed bf16 pairs (keys 32q..32q+31
          // sit in columns 32q..32q+15), 16 rows of V; O1 and O2 of two steps per issue
          const uint64_t vd0 = dvs + (uint64_t)(kk * 16 * 128 / 16), vd1 = vd0 + 16 * 128 / 16;
          const uint32_t pc0 = 32u * (kk >> 1), pc1 = pc0 + 8u;   // kk even: (kk & 1) = 0, kk + 1 odd
          tc_mma_ts4(tmem + kColO1, tmem + col_s(bp) + pc0, vd0, tmem + kColO2, tmem + col_a(bp) + pc0, vd0,
                     tmem + kColO1, tmem + col_s(bp) + pc1, vd1, tmem + kColO2, tmem + col_a(bp) + pc1, vd1, kIdPV,
                     (jp > 0 || kk > 0) ? 1u : 0u, 1u);
        }
        if (few_keys && jp < kPfSplitTiles) {   // lo parts: 16 columns after their hi parts
#pragma unroll
          for (int kk = 0; kk < kPfBN / 16; kk += 2) {
            const uint64_t vd0 = dvs + (uint64_t)(kk * 16 * 128 / 16), vd1 = vd0 + 16 * 128 / 16;
            const uint32_t pc0 = 32u * (kk >> 1) + 16u, pc1 = pc0 + 8u;
            tc_mma_ts4(tmem + kColO1, tmem + col_s(bp) + pc0, vd0, tmem + kColO2, tmem + col_a(bp) + pc0, vd0,
                       tmem + kColO1, tmem + col_s(bp) + pc1, vd1, tmem + kColO2, tmem + col_a(bp) + pc1, vd1,
                       kIdPV, 1u, 1u);
          }
        }
        tc_commit(&v_empty[sp]);
        tc_commit(o_done);
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // Every issued MMA must complete before TMEM is released.
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int g = (warp - 2) >> 2;           // warpgroup: tiles j = g, g+2, ...; S / A buffer g
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;            // query row within the tile
    const int t = m0 + r;                    // query index within the sequence's queries
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int key_lim = a.causal ? min(pos0 + t + 1, L) : L;   // keys [0, key_lim) visible
    const int split_tiles = few_keys ? kPfSplitTiles : 0;
    const uint32_t cS = tmem + lane_off + col_s(g), cA = tmem + lane_off + col_a(g);
    // m_ref: reference max of P after the latest tile (both warpgroups' P
    // enter the same O, so they share it).  m_mine: the reference this
    // warpgroup's partial l and c are relative to.
    float m_ref = -INFINITY, m_mine = -INFINITY, aref = 0.f;
    float2 l2 = make_float2(0.f, 0.f), c2 = make_float2(0.f, 0.f);
    // Each decision that gates a warp-collective tcgen05 op is reduced over
    // the warpgroup (bar_and), so its four warps always run the same tiles.
    bool fine = true;
    int j = g;
    for (; j < n; j += 2) {
      const bool w = !*abort_flag && mbar_wait_bounded(a.wait_ns, &s_full[g], (j >> 1) & 1);
      tc_fence_after();
      uint32_t sr[64], ar[32];
      tmem_ld32p(cS, sr);
      tmem_ld32p(cS + 32, sr + 32);
      tmem_wait_ld();
      // Tiles that reach the diagonal or the sequence end need the mask.
      const int key0 = j * kPfBN;
      const bool masked = (a.causal && key0 + kPfBN - 1 > pos0 + m0) || (key0 + kPfBN > L);
      if (masked) {
#pragma unroll
        for (int cc = 0; cc < 64; ++cc)
          if (key0 + cc >= key_lim) sr[cc] = __float_as_uint(-INFINITY);
      }
      float mt[8];   // eight independent running maxima: a short dependency chain, few registers
#pragma unroll
      for (int i = 0; i < 8; ++i) mt[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[i + 8]));
#pragma unroll
      for (int i = 16; i < 64; ++i) mt[i & 7] = fmaxf(mt[i & 7], __uint_as_float(sr[i]));
      mt[0] = fmaxf(fmaxf(fmaxf(mt[0], mt[4]), fmaxf(mt[1], mt[5])), fmaxf(fmaxf(mt[2], mt[6]), fmaxf(mt[3], mt[7])));
      tmem_ld32(cA, ar);   // probe values of keys 0..31, loaded while the reference is handed over
      // The reference after tile j-1 comes from the other warpgroup.
      const bool wh = j == 0 || mbar_wait_bounded(a.wait_ns, &hand[g], ((j - 1) >> 1) & 1);
      const bool go = bar_and(1 + g, kPfSoftmax / 2, w && wh && fine);
      tmem_wait_ld();
      if (!go) {
        fine = false;
        break;
      }
      if (j == 0) {
        aref = __uint_as_float(ar[0]);   // a_ref = rho . k_0: key 0 is visible to every row
      } else {
        m_ref = mref_s[r];
        if (j == 1) aref = aref_s[r];
      }
      // scale > 0, so the max of the scaled scores is the scaled max
      const float m_new = fmaxf(m_ref, mt[0] * a.scale_log2);
      const bool need = m_new > m_ref + kPfRescaleLog2;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m_ref - m_new);
        m_ref = m_new;
      }
      mref_s[r] = m_ref;
      if (j == 0) aref_s[r] = aref;
      mbar_arrive(&hand[1 - g]);
      if (m_mine != m_ref) {   // bring this warpgroup's partial sums to the current reference
        const float f = ex2(m_mine - m_ref);
        l2 = mul2(l2, make_float2(f, f));
        c2 = mul2(c2, make_float2(f, f));
        m_mine = m_ref;
      }
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nm2 = make_float2(-m_ref, -m_ref);
      const float2 na2 = make_float2(-aref, -aref);
      // S of this tile is in registers and A is read half by half, so P and
      // P o A' overwrite them in TMEM as they go: the bf16 pairs of keys
      // 32q..32q+31 go to columns 32q..32q+15 of the S / A buffer, their lo
      // parts (split tiles only) to 32q+16..32q+31 -- columns this half has
      // already consumed.  The split is a separate instantiation so that
      // ordinary tiles run a loop without it.
      auto form_p = [&](auto split_tag) {
        constexpr bool kSplit = decltype(split_tag)::value;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1) {
            tmem_ld32(cA + 32, ar);
            tmem_wait_ld();
          }
          if constexpr (kPaged) {   // a page tail may hold NaN keys: select, not multiply
            if (masked) {
#pragma unroll
              for (int cc = 0; cc < 32; ++cc)
                if (key0 + 32 * q + cc >= key_lim) ar[cc] = 0u;
            }
          }
          uint32_t pp[16], pa[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = 32 * q + 2 * i;
            const float2 x2 = fma2(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sc2, nm2);
            const float2 p2 = make_float2(ex2(x2.x), ex2(x2.y));
            l2 = add2(l2, p2);
            const float2 q2 =
                mul2(p2, add2(make_float2(__uint_as_float(ar[2 * i]), __uint_as_float(ar[2 * i + 1])), na2));
            c2 = add2(c2, q2);
            pp[i] = pack_bf16(p2.x, p2.y);
            pa[i] = pack_bf16(q2.x, q2.y);
            if constexpr (kSplit) {   // lo parts reuse entries already consumed: sr[32q+i] (<= e), ar[i] (<= 2i)
              sr[32 * q + i] = pack_bf16(p2.x - bf16_lo_f(pp[i]), p2.y - bf16_hi_f(pp[i]));
              ar[i] = pack_bf16(q2.x - bf16_lo_f(pa[i]), q2.y - bf16_hi_f(pa[i]));
            }
          }
          tmem_st16(cS + 32 * q, pp);
          tmem_st16(cA + 32 * q, pa);
          if constexpr (kSplit) {
            tmem_st16(cS + 32 * q + 16, sr + 32 * q);
            tmem_st16(cA + 32 * q + 16, ar);
          }
        }
      };
      if (j < split_tiles)
        form_p(std::true_type{});
      else
        form_p(std::false_type{});
      // O may be touched only once the value products of tile j-1 are done.
      // Waiting on that one phase is exact without waiting on the earlier
      // ones: s_full(j) was committed after the value products of tile j-2,
      // so o_done has completed phase j-2, and tile j's value products cannot
      // start before this warpgroup arrives on p_full below; the phase is
      // j-1 or j.  The wait is skipped unless O is rescaled, except at the
      // last tile, which pins the phase for the epilogue's wait to n-1 or n.
      const bool rescale = __any_sync(0xffffffffu, need) && j >= 1;
      if (j >= 1 && (j == n - 1 || rescale)) {
        const bool wo = __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, o_done, (j - 1) & 1));
        fine = fine && wo;
        if (wo && rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int part = 0; part < 8; ++part) {   // O1 then O2, 32 columns at a time
            uint32_t ov[32];
            const uint32_t addr = tmem + lane_off + kColO1 + part * 32;
            tmem_ld32(addr, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(addr, ov);
          }
        }
      }
      if constexpr (kPaged) {
        // The sequence ends inside this page: zero the V rows past its end
        // (their weights are 0, but 0 * NaN is not) before the value
        // products, which wait on this warpgroup's arrival below.
        if (key0 + kPfBN > L) {
          const int s = j % kPfStages, nv = L - key0;
          const bool wv = mbar_wait_bounded(a.wait_ns, &v_full[s], (j / kPfStages) & 1);
          fine = fine && wv;
          if (wv) {
            uint8_t* vt = sm + Ly::kV + s * Ly::kKVBytes;
            for (int i = (int)threadIdx.x - 64 - 128 * g; i < (kPfBN - nv) * 16; i += kPfSoftmax / 2) {
              const int row = nv + (i >> 4), c = i & 15;   // c: box (c >> 3), 16-byte chunk (c & 7)
              *reinterpret_cast<uint4*>(vt + (c >> 3) * (Ly::kKVBytes / 2) + row * 128 + (c & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[g]);
    }
    // ---- epilogue: the last tile's warpgroup waits for the last value
    // products (its j == n-1 wait above made the phase exact), the barrier
    // below releases the other; then the rows are written.
    bool wl = fine && j >= n && !*abort_flag;
    if (wl && ((n - 1) & 1) == g) wl = mbar_wait_bounded(a.wait_ns, o_done, (n - 1) & 1);
    lc_s[(g * 128 + r) * 3 + 0] = l2.x + l2.y;
    lc_s[(g * 128 + r) * 3 + 1] = c2.x + c2.y;
    lc_s[(g * 128 + r) * 3 + 2] = m_mine;
    if (bar_and(3, kPfSoftmax, wl)) {
      tc_fence_after();
      // O is relative to the last reference, the larger of the two (references only grow).
      const float ma = lc_s[r * 3 + 2], mb = lc_s[(128 + r) * 3 + 2];
      const float mm = fmaxf(ma, mb);
      const float fa = ex2(ma - mm), fb = ex2(mb - mm);   // a warpgroup with no tiles has l = c = 0
      // explicit fmaf throughout, so that both instantiations round alike
      const float lt = fmaf(lc_s[r * 3], fa, lc_s[(128 + r) * 3] * fb);
      const float ct = fmaf(lc_s[r * 3 + 1], fa, lc_s[(128 + r) * 3 + 1] * fb);
      const float inv = 1.f / lt;
      const float corr = fmaf(ct, inv, 1.f);
      if constexpr (!kPaged) {
        if (a.stats != nullptr && g == 0 && t < q_len)
          // c accumulates e * (a - a_ref), so abar = c / l + a_ref
          a.stats[(size_t)(b * a.H + h) * a.T + t] = make_float2(mm + __log2f(lt), ct * inv + aref);
      }
      const size_t orow = (kPaged ? (size_t)(q_first + t) * a.H + h : (size_t)(b * a.H + h) * a.T + t) * kPfD + 64 * g;
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        uint32_t o1[32], o2[32];
        tmem_ld32(tmem + lane_off + kColO1 + 64 * g + part * 32, o1);
        tmem_ld32(tmem + lane_off + kColO2 + 64 * g + part * 32, o2);
        tmem_wait_ld();
        if (t < q_len) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float vb = __uint_as_float(o1[i]) * inv;   // vbar
            v[i] = fmaf(vb, corr, -(__uint_as_float(o2[i]) * inv));
            if constexpr (!kPaged) o1[i] = __float_as_uint(vb);
          }
          if constexpr (!kPaged) {
            if (a.vbar != nullptr) {
              float4* vbp = reinterpret_cast<float4*>(a.vbar + orow + part * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                vbp[i] = make_float4(__uint_as_float(o1[4 * i]), __uint_as_float(o1[4 * i + 1]),
                                     __uint_as_float(o1[4 * i + 2]), __uint_as_float(o1[4 * i + 3]));
            }
          }
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + orow + part * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                                  pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + orow + part * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
    } else {
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace plx
