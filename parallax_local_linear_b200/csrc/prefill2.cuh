// Parallax causal prefill on a pair of SMs: tcgen05.mma with cta_group::2.
//
// The same computation as prefill_tc_kernel (dense form; see prefill.cuh for
// the method, the softmax and the epilogue), with M = 256 query rows per
// tensor-core instruction spread over the two CTAs of a cluster:
//
//   S  = Q K^T, A = R K^T    256 x 64 per key tile: CTA r holds query rows
//                            128r..128r+127 (its A operand, and its 128 TMEM
//                            lanes of S and A) and keys 32r..32r+31 of the
//                            tile (its half of the B operand).
//   O1 += P V, O2 += (P o A') V   256 x 128: P from each CTA's own TMEM,
//                            CTA r holds head-dimension columns 64r..64r+63
//                            of the V tile (its half of B).
//
// Each SM therefore loads half of every K and V tile, reads half of each B
// operand from its shared memory, and issues no MMA at all on the second
// CTA: the first CTA's MMA warp issues one instruction for both.  Compared
// with one CTA per 128 rows this halves the TMA writes and B-operand reads
// per SM and the MMA instructions per tile, the two costs the single-CTA
// kernel's tile period is measured to be bound by besides the tensor pipe.
//
// Cross-CTA protocol (every wait bounded):
//   * each CTA's TMA loads complete on its own barriers (so a CTA can always
//     wait for its own copies before it exits); the second CTA's MMA warp
//     forwards "my half of Q/R, K(j), V(j) has landed" to the first CTA by a
//     remote mbarrier arrive (release.cluster);
//   * the first CTA's MMA warp waits on its own and the forwarded barriers
//     (acquire.cluster), issues the MMAs, and commits their completion to the
//     barriers of both CTAs at once (tcgen05.commit multicast): s_full (S/A
//     ready), k_empty / v_empty (the stage may be refilled), o_done, drain;
//   * each softmax warp of either CTA arrives once on the first CTA's p_full
//     when its lanes' P is in their TMEM (a remote arrive from the second).
// Barriers that only tcgen05.commit arrives on are waited with CTA scope;
// those that threads of the other CTA arrive on, with cluster scope.
// Tensor memory is allocated and freed for the pair (cta_group::2); a
// cluster barrier precedes the release.
#pragma once

#include "prefill.cuh"

namespace plx {

#ifndef PLX_PREFILL2_STAGES
#define PLX_PREFILL2_STAGES 6
#endif
constexpr int kP2Stages = PLX_PREFILL2_STAGES;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {   // whole warp, both CTAs
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Arrives once on `bar` (same shared-memory offset) in every CTA of `mask`
// when the tensor-core operations issued so far have completed.
__device__ __forceinline__ void tc2_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::
          "r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tc2_mma_ss4(uint32_t d0, uint64_t a0, uint64_t b0, uint32_t d1, uint64_t a1,
                                            uint64_t b1, uint32_t d2, uint64_t a2, uint64_t b2, uint32_t d3,
                                            uint64_t a3, uint64_t b3, uint32_t idesc, uint32_t acc01,
                                            uint32_t acc23) {
  asm volatile(
      "{\n\t.reg .pred p01, p23, e;\n\tsetp.ne.b32 p01, %13, 0;\n\tsetp.ne.b32 p23, %14, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%3], %4, %5, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%6], %7, %8, %12, p23;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%9], %10, %11, %12, p23;\n\t}" ::"r"(d0),
      "l"(a0), "l"(b0), "r"(d1), "l"(a1), "l"(b1), "r"(d2), "l"(a2), "l"(b2), "r"(d3), "l"(a3), "l"(b3),
      "r"(idesc), "r"(acc01), "r"(acc23)
      : "memory");
}

__device__ __forceinline__ void tc2_mma_ts4(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t d1, uint32_t a1,
                                            uint64_t b1, uint32_t d2, uint32_t a2, uint64_t b2, uint32_t d3,
                                            uint32_t a3, uint64_t b3, uint32_t idesc, uint32_t acc01,
                                            uint32_t acc23) {
  asm volatile(
      "{\n\t.reg .pred p01, p23, e;\n\tsetp.ne.b32 p01, %13, 0;\n\tsetp.ne.b32 p23, %14, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%3], [%4], %5, %12, p01;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%6], [%7], %8, %12, p23;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%9], [%10], %11, %12, p23;\n\t}" ::"r"(d0),
      "r"(a0), "l"(b0), "r"(d1), "r"(a1), "l"(b1), "r"(d2), "r"(a2), "l"(b2), "r"(d3), "r"(a3), "l"(b3),
      "r"(idesc), "r"(acc01), "r"(acc23)
      : "memory");
}

// Arrive on a barrier of another CTA of the cluster (a shared::cluster address).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait_bounded with cluster-scope acquire: for barriers that other CTAs
// of the cluster arrive on (remote arrives, multicast commits).
__device__ __forceinline__ bool mbar_wait_cl(uint64_t limit_ns, uint64_t* bar, uint32_t parity) {
  if (limit_ns == 0) {
    if (mbar_test_wait_cl(bar, parity)) return true;
    report_error(2 /* PLX_DEVERR_TIMEOUT */);
    return false;
  }
  if (mbar_try_wait_cl(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t it = 0;
  while (!mbar_try_wait_cl(bar, parity)) {
    if ((++it & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) {
      report_error(2 /* PLX_DEVERR_TIMEOUT */);
      return false;
    }
  }
  return true;
}

struct P2Layout {
  static constexpr int kQBytes = kPfBM * kPfD * 2;        // 32 KB: two 64-column boxes of 128 rows
  static constexpr int kKBytes = (kPfBN / 2) * kPfD * 2;  // 8 KB: this CTA's 32 keys, two 64-column boxes
  static constexpr int kVBytes = kPfBN * 64 * 2;          // 8 KB: this CTA's 64 columns of 64 keys
  static constexpr int kQ = 0;
  static constexpr int kR = kQ + kQBytes;
  static constexpr int kK = kR + kQBytes;
  static constexpr int kV = kK + kP2Stages * kKBytes;
  static constexpr int kBar = kV + kP2Stages * kVBytes;
  // q_full, pq_full, k_full[S], v_full[S], pk_full[S], pv_full[S], k_empty[S], v_empty[S],
  // s_full[2], p_full[2], o_done, drain, hand[2]
  static constexpr int kNumBars = 2 + 6 * kP2Stages + 2 + 2 + 1 + 1 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;        // tmem base, abort flag
  static constexpr int kMref = kMisc + 16;
  static constexpr int kAref = kMref + 128 * 4;
  static constexpr int kLC = kAref + 128 * 4;
  static constexpr int kBytes = kLC + 2 * 128 * 3 * 4 + 1024;
};

// Grid: 2 CTAs per 256 query rows of a (sequence, head), clusters of 2,
// longest pairs first.  a.n_mblk = ceil(T / 256).
// Launched with a cluster dimension of 2 (cudaLaunchKernelEx).  320 threads
// are 10 warps, so three share an SM sub-partition's 16K registers: at most
// 168 registers a thread.
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const PrefillArgs a) {
  using Ly = P2Layout;
  constexpr int S = kP2Stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* q_full = bars;
  uint64_t* pq_full = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = k_full + S;
  uint64_t* pk_full = v_full + S;
  uint64_t* pv_full = pk_full + S;
  uint64_t* k_empty = pv_full + S;
  uint64_t* v_empty = k_empty + S;
  uint64_t* s_full = v_empty + S;
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
  const uint32_t rank = cluster_ctarank();   // 0: issues the MMAs; 1: its partner
  const int BH = a.B * a.H;
  const int pair = blockIdx.x >> 1;
  const int pblk = a.n_mblk - 1 - pair / BH;   // longest pairs first
  const int bh = pair % BH;
  const int b = bh / a.H, h = bh % a.H, kvh = h / a.group;
  const int m0p = pblk * 2 * kPfBM;            // the pair's first query row
  const int m0 = m0p + kPfBM * (int)rank;      // this CTA's first query row
  const int T = a.T;
  const int kv_end = a.causal ? min(T, m0p + 2 * kPfBM) : T;
  const int n = (kv_end + kPfBN - 1) / kPfBN;  // key tiles of the pair
  // The lo-part split is decided per pair (the MMAs are shared): rows of its
  // first CTA see the fewest keys.
  const int min_keys = a.causal ? min(m0p + 1, T) : T;
  const bool few_keys = min_keys < 2 * kPfBN;
  const int q_row = (b * a.H + h) * T + m0;
  const int kv_row = (b * a.Hkv + kvh) * T;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(pq_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&pk_full[s], 1);
      mbar_init(&pv_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);   // the 4 warps of this buffer's warpgroup in each CTA (first CTA's barrier)
      mbar_init(&hand[i], kPfSoftmax / 2);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc2(tmem_base_s, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // both CTAs' barriers exist before any remote arrive or multicast commit
  const uint32_t tmem = *tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_r);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, 2 * Ly::kQBytes);
      for (int bx = 0; bx < 2; ++bx) {
        tma_load_2d(sm + Ly::kQ + bx * (Ly::kQBytes / 2), &tm_q, bx * 64, q_row, q_full, once);
        tma_load_2d(sm + Ly::kR + bx * (Ly::kQBytes / 2), &tm_r, bx * 64, q_row, q_full, once);
      }
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % S;
        const uint32_t par = ((j / S) - 1) & 1;
        const int row = kv_row + j * kPfBN;
        if (j >= S && !mbar_wait_bounded(a.wait_ns, &k_empty[s], par)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&k_full[s], Ly::kKBytes);
        for (int bx = 0; bx < 2; ++bx)   // keys 32 rank .. 32 rank + 31 of the tile
          tma_load_2d(sm + Ly::kK + s * Ly::kKBytes + bx * (Ly::kKBytes / 2), &tm_k, bx * 64,
                      row + (kPfBN / 2) * (int)rank, &k_full[s], keep);
        ++issued_k;
        if (j >= S && !mbar_wait_bounded(a.wait_ns, &v_empty[s], par)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], Ly::kVBytes);   // columns 64 rank .. 64 rank + 63
        tma_load_2d(sm + Ly::kV + s * Ly::kVBytes, &tm_v, 64 * (int)rank, row, &v_full[s], keep);
        ++issued_v;
      }
      // Every issued load must land before the CTA exits.
      mbar_wait_drain(q_full, 0);
      for (int s = 0; s < S && s < issued_k; ++s) {
        const int last = s + ((issued_k - 1 - s) / S) * S;
        mbar_wait_drain(&k_full[s], (last / S) & 1);
      }
      for (int s = 0; s < S && s < issued_v; ++s) {
        const int last = s + ((issued_v - 1 - s) / S) * S;
        mbar_wait_drain(&v_full[s], (last / S) & 1);
      }
    }
  } else if (warp == 1 && rank == 1) {
    // ------------------------------------------------ forwarder (second CTA)
    // Tells the first CTA that this CTA's halves of Q/R, K(j) and V(j) have
    // landed, in the order the MMAs need them.
    if (lane == 0) {
      const uint32_t r_pq = dsmem_map(smem_u32(pq_full), 0);
      bool ok = mbar_wait_bounded(a.wait_ns, q_full, 0);
      if (ok) mbar_arrive_remote(r_pq);
      for (int j = 0; ok && j < n; ++j) {
        const int s = j % S;
        const uint32_t par = (j / S) & 1;
        if (*abort_flag) break;
        if (!(ok = mbar_wait_bounded(a.wait_ns, &k_full[s], par))) break;
        mbar_arrive_remote(dsmem_map(smem_u32(&pk_full[s]), 0));
        if (!(ok = mbar_wait_bounded(a.wait_ns, &v_full[s], par))) break;
        mbar_arrive_remote(dsmem_map(smem_u32(&pv_full[s]), 0));
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
    // The first CTA's MMAs write this CTA's TMEM: wait for all of them.
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (first CTA)
    constexpr uint32_t kIdS = idesc_bf16(2 * kPfBM, kPfBN, false);   // 256 x 64, K-major B
    constexpr uint32_t kIdPV = idesc_bf16(2 * kPfBM, kPfD, true);    // 256 x 128, MN-major B (V)
    constexpr uint16_t kBoth = 0x3;
    const uint64_t dq = smem_desc_sw128(smem_u32(sm + Ly::kQ), 16, 1024);
    const uint64_t dr = smem_desc_sw128(smem_u32(sm + Ly::kR), 16, 1024);
    const uint64_t dk = smem_desc_sw128(smem_u32(sm + Ly::kK), 16, 1024);
    const uint64_t dv = smem_desc_sw128(smem_u32(sm + Ly::kV), Ly::kVBytes, 1024);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_cl(a.wait_ns, bar, parity));
    };
    bool ok = wait_warp(q_full, 0) && wait_warp(pq_full, 0);
    tc_fence_after();
    for (int j = 0; ok && j <= n; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (j < n) {
        const int s = j % S, b2 = j & 1;
        const uint32_t par = (j / S) & 1;
        if (!(ok = wait_warp(&k_full[s], par) && wait_warp(&pk_full[s], par))) break;
        tc_fence_after();
        const uint64_t dks = dk + (uint64_t)((s * Ly::kKBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; kk += 2) {
          // 16 columns of d per step: box kk / 4, 32 bytes into the 128-byte row
          const uint64_t oq0 = (uint64_t)((kk >> 2) * (Ly::kQBytes / 2 / 16) + (kk & 3) * 2);
          const uint64_t ok0 = (uint64_t)((kk >> 2) * (Ly::kKBytes / 2 / 16) + (kk & 3) * 2);
          const uint64_t oq1 = oq0 + 2, ok1 = ok0 + 2;
          tc2_mma_ss4(tmem + col_s(b2), dq + oq0, dks + ok0, tmem + col_a(b2), dr + oq0, dks + ok0,
                      tmem + col_s(b2), dq + oq1, dks + ok1, tmem + col_a(b2), dr + oq1, dks + ok1, kIdS,
                      kk > 0 ? 1u : 0u, 1u);
        }
        tc2_commit_mc(&s_full[b2], kBoth);
        tc2_commit_mc(&k_empty[s], kBoth);   // K(j) is free in both CTAs once the score products are done
      }
      if (j >= 1) {
        const int jp = j - 1, bp = jp & 1, sp = jp % S;
        const uint32_t par = (jp / S) & 1;
        if (!(ok = wait_warp(&v_full[sp], par) && wait_warp(&pv_full[sp], par))) break;
        if (!(ok = wait_warp(&p_full[bp], (jp >> 1) & 1))) break;
        tc_fence_after();
        const uint64_t dvs = dv + (uint64_t)((sp * Ly::kVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; kk += 2) {
          const uint64_t vd0 = dvs + (uint64_t)(kk * 16 * 128 / 16), vd1 = vd0 + 16 * 128 / 16;
          const uint32_t pc0 = 32u * (kk >> 1), pc1 = pc0 + 8u;
          tc2_mma_ts4(tmem + kColO1, tmem + col_s(bp) + pc0, vd0, tmem + kColO2, tmem + col_a(bp) + pc0, vd0,
                      tmem + kColO1, tmem + col_s(bp) + pc1, vd1, tmem + kColO2, tmem + col_a(bp) + pc1, vd1, kIdPV,
                      (jp > 0 || kk > 0) ? 1u : 0u, 1u);
        }
        if (few_keys && jp < kPfSplitTiles) {   // lo parts: 16 columns after their hi parts
#pragma unroll
          for (int kk = 0; kk < kPfBN / 16; kk += 2) {
            const uint64_t vd0 = dvs + (uint64_t)(kk * 16 * 128 / 16), vd1 = vd0 + 16 * 128 / 16;
            const uint32_t pc0 = 32u * (kk >> 1) + 16u, pc1 = pc0 + 8u;
            tc2_mma_ts4(tmem + kColO1, tmem + col_s(bp) + pc0, vd0, tmem + kColO2, tmem + col_a(bp) + pc0, vd0,
                        tmem + kColO1, tmem + col_s(bp) + pc1, vd1, tmem + kColO2, tmem + col_a(bp) + pc1, vd1,
                        kIdPV, 1u, 1u);
          }
        }
        tc2_commit_mc(&v_empty[sp], kBoth);
        tc2_commit_mc(o_done, kBoth);
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // Every issued MMA must complete before either CTA releases tensor memory.
    tc2_commit_mc(drain, kBoth);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (both CTAs)
    // As in prefill_tc_kernel (dense form), on this CTA's 128 rows; P is
    // announced to the first CTA's p_full.
    const int g = (warp - 2) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int t = m0 + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int key_lim = a.causal ? min(t + 1, T) : T;
    const int split_tiles = few_keys ? kPfSplitTiles : 0;
    const uint32_t cS = tmem + lane_off + col_s(g), cA = tmem + lane_off + col_a(g);
    float m_ref = -INFINITY, m_mine = -INFINITY, aref = 0.f;
    float2 l2 = make_float2(0.f, 0.f), c2 = make_float2(0.f, 0.f);
    bool fine = true;
    int j = g;
    for (; j < n; j += 2) {
      const bool w = !*abort_flag && mbar_wait_bounded(a.wait_ns, &s_full[g], (j >> 1) & 1);
      tc_fence_after();
      uint32_t sr[64], ar[32];
      tmem_ld32p(cS, sr);
      tmem_ld32p(cS + 32, sr + 32);
      tmem_wait_ld();
      const int key0 = j * kPfBN;
      const bool masked = (a.causal && key0 + kPfBN - 1 > m0) || (key0 + kPfBN > T);
      if (masked) {
#pragma unroll
        for (int cc = 0; cc < 64; ++cc)
          if (key0 + cc >= key_lim) sr[cc] = __float_as_uint(-INFINITY);
      }
      float mt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mt[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[i + 8]));
#pragma unroll
      for (int i = 16; i < 64; ++i) mt[i & 7] = fmaxf(mt[i & 7], __uint_as_float(sr[i]));
      mt[0] = fmaxf(fmaxf(fmaxf(mt[0], mt[4]), fmaxf(mt[1], mt[5])), fmaxf(fmaxf(mt[2], mt[6]), fmaxf(mt[3], mt[7])));
      tmem_ld32(cA, ar);
      const bool wh = j == 0 || mbar_wait_bounded(a.wait_ns, &hand[g], ((j - 1) >> 1) & 1);
      const bool go = bar_and(1 + g, kPfSoftmax / 2, w && wh && fine);
      tmem_wait_ld();
      if (!go) {
        fine = false;
        break;
      }
      if (j == 0) {
        aref = __uint_as_float(ar[0]);   // a_ref = rho . k_0
      } else {
        m_ref = mref_s[r];
        if (j == 1) aref = aref_s[r];
      }
      // A row that sees no key of this tile (the first CTA's rows on the
      // pair's last tiles) has mt = -inf: its reference stays.
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
      if (m_mine != m_ref) {
        const float f = ex2(m_mine - m_ref);
        l2 = mul2(l2, make_float2(f, f));
        c2 = mul2(c2, make_float2(f, f));
        m_mine = m_ref;
      }
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nm2 = make_float2(-m_ref, -m_ref);
      const float2 na2 = make_float2(-aref, -aref);
      auto form_p = [&](auto split_tag) {
        constexpr bool kSplit = decltype(split_tag)::value;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1) {
            tmem_ld32(cA + 32, ar);
            tmem_wait_ld();
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
            if constexpr (kSplit) {
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
      const bool rescale = __any_sync(0xffffffffu, need) && j >= 1;
      if (j >= 1 && (j == n - 1 || rescale)) {
        const bool wo = __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, o_done, (j - 1) & 1));
        fine = fine && wo;
        if (wo && rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int part = 0; part < 8; ++part) {
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
      // One arrive per warp, after every lane's TMEM stores have completed.
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (cluster_ctarank() == 0)
          mbar_arrive(&p_full[g]);
        else
          mbar_arrive_remote(dsmem_map(smem_u32(&p_full[g]), 0));
      }
    }
    bool wl = fine && j >= n && !*abort_flag;
    if (wl && ((n - 1) & 1) == g) wl = mbar_wait_bounded(a.wait_ns, o_done, (n - 1) & 1);
    lc_s[(g * 128 + r) * 3 + 0] = l2.x + l2.y;
    lc_s[(g * 128 + r) * 3 + 1] = c2.x + c2.y;
    lc_s[(g * 128 + r) * 3 + 2] = m_mine;
    if (bar_and(3, kPfSoftmax, wl)) {
      tc_fence_after();
      const float ma = lc_s[r * 3 + 2], mb = lc_s[(128 + r) * 3 + 2];
      const float mm = fmaxf(ma, mb);
      const float fa = ex2(ma - mm), fb = ex2(mb - mm);
      const float lt = fmaf(lc_s[r * 3], fa, lc_s[(128 + r) * 3] * fb);
      const float ct = fmaf(lc_s[r * 3 + 1], fa, lc_s[(128 + r) * 3 + 1] * fb);
      const float inv = 1.f / lt;
      const float corr = fmaf(ct, inv, 1.f);
      if (a.stats != nullptr && g == 0 && t < T)
        a.stats[(size_t)(b * a.H + h) * T + t] = make_float2(mm + __log2f(lt), ct * inv + aref);
      const size_t orow = ((size_t)(b * a.H + h) * T + t) * kPfD + 64 * g;
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        uint32_t o1[32], o2[32];
        tmem_ld32(tmem + lane_off + kColO1 + 64 * g + part * 32, o1);
        tmem_ld32(tmem + lane_off + kColO2 + 64 * g + part * 32, o2);
        tmem_wait_ld();
        if (t < T) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float vb = __uint_as_float(o1[i]) * inv;
            v[i] = fmaf(vb, corr, -(__uint_as_float(o2[i]) * inv));
            o1[i] = __float_as_uint(vb);
          }
          if (a.vbar != nullptr) {
            float4* vbp = reinterpret_cast<float4*>(a.vbar + orow + part * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              vbp[i] = make_float4(__uint_as_float(o1[4 * i]), __uint_as_float(o1[4 * i + 1]),
                                   __uint_as_float(o1[4 * i + 2]), __uint_as_float(o1[4 * i + 3]));
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
  // Neither CTA releases tensor memory or exits while the other may still
  // read its shared memory or arrive on its barriers.
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc2(tmem, 512);
}

}  // namespace plx
