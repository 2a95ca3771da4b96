// Parallax causal prefill on sm_100a: TMA, tcgen05.mma, tensor memory.
//
// Every position t of a sequence is a query with probe rho_t over keys 0..t
// (causal, diagonal included) or over all keys.  Per query row the kernel
// keeps the running max m and l = sum e, c = sum e*a, O1 = sum e v,
// O2 = sum e*a v with e = exp(scale q.k - m), a = rho.k - a_ref, and writes
// out = (O1/l)(1 + c/l) - O2/l, which equals vbar - S_KV^T rho (the
// covariance correction of the wispaper.ai blog "Parallax: Breaking the
// Boundary Bias with Parameterized Local Linear Attention", section "The Core
// Insight: Covariance Correction"; computed "in a single pass" as in its
// "Hardware Efficiency" section).  a_ref = rho_t.k_0, read from the first key
// tile (key 0 is visible to every row).
//
// The four products are dense contractions and run on the tensor cores:
//     S  = Q K^T,    A  = R K^T            (128 x 64 per key tile, fp32 in TMEM)
//     O1 += P V,     O2 += (P o A') V      (128 x 128, fp32 in TMEM)
// with P = exp2(S * scale * log2(e) - m) and A' = A - a_ref.
//
// CTA = one 128-row query tile of one (sequence, head); key tiles of 64.
// Warp roles (192 threads):
//   warp 0       TMA producer: Q and R once, then a STAGES-deep K/V ring.
//   warp 1       TMEM allocator; lane 0 issues every tcgen05.mma.
//   warps 2..5   softmax: thread = query row = TMEM lane.  Reads S and A
//                from TMEM, forms P and P o A' in bf16, writes them back over
//                the S and A columns (the A operand of the value products
//                comes straight from TMEM), rescales O when the running max
//                grows by more than 2^8, and finally writes the output.
//
// TMEM columns (512 x 128 lanes x 32 bit): O1 [0,128), O2 [128,256), and two
// buffers of S / A: S_b at 256 + 128 b, A_b at 320 + 128 b.  While the
// softmax warps work on tile j, the tensor cores run the value products of
// tile j-1 and the score products of tile j+1.
#pragma once

#include "ptx.cuh"

namespace plx {

constexpr int kPfBM = 128;        // query rows per CTA (= TMEM lanes)
constexpr int kPfBN = 64;         // keys per tile
constexpr int kPfD = 128;         // head dim
constexpr int kPfStages = 3;      // K/V ring depth
constexpr float kPfRescaleLog2 = 8.f;   // lazy rescale threshold (factor 256)
// Key tiles whose P and P o A' also enter the value products as bf16 lo parts
// (x = bf16(x) + lo).  A row with few keys has nothing to average the bf16
// rounding of P o A' (|a| reaches ~10 for unit-scale probes) over; every
// row's first 128 keys lie in tiles 0 and 1, so splitting those tiles keeps
// short rows at fp32-level weights for ~1% more tensor work at T = 8192.
constexpr int kPfSplitTiles = 2;

struct PrefillArgs {
  int B, H, Hkv, T, group;
  int n_mblk;                     // ceil(T / 128)
  int causal, out_bf16;
  float scale_log2;
  void* out;                      // [B, H, T, D]
};

struct PfLayout {
  static constexpr int kQBytes = kPfBM * kPfD * 2;       // 32 KB: two 64-column boxes of 128 rows
  static constexpr int kKVBytes = kPfBN * kPfD * 2;      // 16 KB: two 64-column boxes of 64 rows
  static constexpr int kQ = 0;
  static constexpr int kR = kQ + kQBytes;
  static constexpr int kK = kR + kQBytes;
  static constexpr int kV = kK + kPfStages * kKVBytes;
  static constexpr int kBar = kV + kPfStages * kKVBytes;
  // barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr int kNumBars = 1 + 3 * kPfStages + 2 + 2 + 1 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;       // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16 + 1024;        // + alignment slack
};

constexpr uint32_t kColO1 = 0, kColO2 = 128;
__device__ __forceinline__ uint32_t col_s(int b) { return 256u + 128u * b; }
__device__ __forceinline__ uint32_t col_a(int b) { return 320u + 128u * b; }

__global__ void __launch_bounds__(192, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillArgs a) {
  using L = PfLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kPfStages;
  uint64_t* kv_empty = v_full + kPfStages;
  uint64_t* s_full = kv_empty + kPfStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest query tiles first: the last tile of every head, then the one before...
  const int BH = a.B * a.H;
  const int mblk = a.n_mblk - 1 - (int)(blockIdx.x / BH);
  const int bh = blockIdx.x % BH;
  const int b = bh / a.H, h = bh % a.H, kvh = h / a.group;
  const int m0 = mblk * kPfBM;
  const int kv_end = a.causal ? min(a.T, m0 + kPfBM) : a.T;
  const int n = (kv_end + kPfBN - 1) / kPfBN;
  const int q_row = (b * a.H + h) * a.T + m0;
  const int kv_row = (b * a.Hkv + kvh) * a.T;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
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
      mbar_arrive_expect_tx(q_full, 2 * L::kQBytes);
      for (int bx = 0; bx < 2; ++bx) {
        tma_load_2d(sm + L::kQ + bx * (L::kQBytes / 2), &tm_q, bx * 64, q_row, q_full, once);
        tma_load_2d(sm + L::kR + bx * (L::kQBytes / 2), &tm_r, bx * 64, q_row, q_full, once);
      }
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % kPfStages;
        if (j >= kPfStages && !mbar_wait_bounded(&kv_empty[s], ((j / kPfStages) - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int row = kv_row + j * kPfBN;
        mbar_arrive_expect_tx(&k_full[s], L::kKVBytes);
        mbar_arrive_expect_tx(&v_full[s], L::kKVBytes);
        for (int bx = 0; bx < 2; ++bx) {
          tma_load_2d(sm + L::kK + s * L::kKVBytes + bx * (L::kKVBytes / 2), &tm_k, bx * 64, row, &k_full[s], keep);
          tma_load_2d(sm + L::kV + s * L::kKVBytes + bx * (L::kKVBytes / 2), &tm_v, bx * 64, row, &v_full[s], keep);
        }
        ++issued;
      }
      // Every issued load must land before the CTA exits.
      mbar_wait_bounded(q_full, 0);
      for (int s = 0; s < kPfStages && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kPfStages) * kPfStages;
        mbar_wait_bounded(&k_full[s], (last / kPfStages) & 1);
        mbar_wait_bounded(&v_full[s], (last / kPfStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(kPfBM, kPfBN, false);   // 128 x 64, K-major B
      constexpr uint32_t kIdPV = idesc_bf16(kPfBM, kPfD, true);    // 128 x 128, MN-major B (V)
      const uint32_t q_base = smem_u32(sm + L::kQ), r_base = smem_u32(sm + L::kR);
      const uint32_t k_base = smem_u32(sm + L::kK), v_base = smem_u32(sm + L::kV);
      bool ok = mbar_wait_bounded(q_full, 0);
      tc_fence_after();
      for (int j = 0; ok && j <= n; ++j) {
        if (*abort_flag) break;
        if (j < n) {
          const int s = j % kPfStages, b2 = j & 1;
          if (!(ok = mbar_wait_bounded(&k_full[s], (j / kPfStages) & 1))) break;
          tc_fence_after();
          const uint32_t kb = k_base + s * L::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kPfD / 16; ++kk) {
            // 16 columns of d per step: box kk / 4, 32 bytes into the 128-byte row per step
            const uint32_t off_q = (kk >> 2) * (L::kQBytes / 2) + (kk & 3) * 32;
            const uint32_t off_k = (kk >> 2) * (L::kKVBytes / 2) + (kk & 3) * 32;
            tc_mma_ss(tmem + col_s(b2), smem_desc_sw128(q_base + off_q, 16, 1024),
                      smem_desc_sw128(kb + off_k, 16, 1024), kIdS, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < kPfD / 16; ++kk) {
            const uint32_t off_q = (kk >> 2) * (L::kQBytes / 2) + (kk & 3) * 32;
            const uint32_t off_k = (kk >> 2) * (L::kKVBytes / 2) + (kk & 3) * 32;
            tc_mma_ss(tmem + col_a(b2), smem_desc_sw128(r_base + off_q, 16, 1024),
                      smem_desc_sw128(kb + off_k, 16, 1024), kIdS, kk > 0);
          }
          tc_commit(&s_full[b2]);
        }
        if (j >= 1) {
          const int jp = j - 1, bp = jp & 1, sp = jp % kPfStages;
          if (!(ok = mbar_wait_bounded(&p_full[bp], (jp >> 1) & 1))) break;
          if (!(ok = mbar_wait_bounded(&v_full[sp], (jp / kPfStages) & 1))) break;
          tc_fence_after();
          const uint32_t vb = v_base + sp * L::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kPfBN / 16; ++kk) {
            // 16 keys per step (8 TMEM columns of packed bf16 pairs; 16 rows of V)
            const uint64_t vd = smem_desc_sw128(vb + kk * 16 * 128, L::kKVBytes / 2, 1024);
            tc_mma_ts(tmem + kColO1, tmem + col_s(bp) + kk * 8, vd, kIdPV, (jp > 0 || kk > 0) ? 1u : 0u);
            tc_mma_ts(tmem + kColO2, tmem + col_a(bp) + kk * 8, vd, kIdPV, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          if (jp < kPfSplitTiles) {   // lo parts sit in columns 32..63 of the S / A buffers
#pragma unroll
            for (int kk = 0; kk < kPfBN / 16; ++kk) {
              const uint64_t vd = smem_desc_sw128(vb + kk * 16 * 128, L::kKVBytes / 2, 1024);
              tc_mma_ts(tmem + kColO1, tmem + col_s(bp) + 32 + kk * 8, vd, kIdPV, 1u);
              tc_mma_ts(tmem + kColO2, tmem + col_a(bp) + 32 + kk * 8, vd, kIdPV, 1u);
            }
          }
          tc_commit(&kv_empty[sp]);
          tc_commit(o_done);
        }
      }
      if (!ok) *abort_flag = 1;
      // Every issued MMA must complete before TMEM is released.
      tc_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;            // query row within the tile
    const int t = m0 + r;                    // query position
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int key_lim = a.causal ? min(t + 1, a.T) : a.T;   // keys [0, key_lim) visible
    float m_used = -INFINITY, l = 0.f, c = 0.f, aref = 0.f;
    // tcgen05.ld / st are warp-collective: every wait outcome and abort
    // decision is made uniform across the warp before acting on it.
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool w = !*abort_flag && mbar_wait_bounded(bar, parity);
      return __all_sync(0xffffffffu, w);
    };
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int b2 = j & 1;
      if (!(ok = wait_warp(&s_full[b2], (j >> 1) & 1))) break;
      tc_fence_after();
      uint32_t sr[64], ar[64];
      tmem_ld32(tmem + lane_off + col_s(b2), *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(tmem + lane_off + col_s(b2) + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld32(tmem + lane_off + col_a(b2), *reinterpret_cast<uint32_t(*)[32]>(ar));
      tmem_ld32(tmem + lane_off + col_a(b2) + 32, *reinterpret_cast<uint32_t(*)[32]>(ar + 32));
      tmem_wait_ld();
      const int key0 = j * kPfBN;
      float mt = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) {
        const float x = (key0 + cc < key_lim) ? __uint_as_float(sr[cc]) * a.scale_log2 : -INFINITY;
        sr[cc] = __float_as_uint(x);
        mt = fmaxf(mt, x);
      }
      if (j == 0) aref = __uint_as_float(ar[0]);
      const float m_new = fmaxf(m_used, mt);
      const bool need = m_new > m_used + kPfRescaleLog2;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m_used - m_new);
        m_used = m_new;
      }
      l *= alpha;
      c *= alpha;
      uint32_t pp[32], pa[32];
      const bool split = j < kPfSplitTiles;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) {
        const float p0 = ex2(__uint_as_float(sr[2 * cc]) - m_used);
        const float p1 = ex2(__uint_as_float(sr[2 * cc + 1]) - m_used);
        const float q0 = p0 * (__uint_as_float(ar[2 * cc]) - aref);
        const float q1 = p1 * (__uint_as_float(ar[2 * cc + 1]) - aref);
        l += p0 + p1;
        c += q0 + q1;
        pp[cc] = pack_bf16(p0, p1);
        pa[cc] = pack_bf16(q0, q1);
        if (split) {   // the lo parts reuse sr / ar, already consumed
          sr[cc] = pack_bf16(p0 - bf16_lo_f(pp[cc]), p1 - bf16_hi_f(pp[cc]));
          ar[cc] = pack_bf16(q0 - bf16_lo_f(pa[cc]), q1 - bf16_hi_f(pa[cc]));
        }
      }
      tmem_st32(tmem + lane_off + col_s(b2), pp);
      tmem_st32(tmem + lane_off + col_a(b2), pa);
      if (split) {
        tmem_st32(tmem + lane_off + col_s(b2) + 32, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_st32(tmem + lane_off + col_a(b2) + 32, *reinterpret_cast<uint32_t(*)[32]>(ar));
      }
      if (j >= 1) {
        // O may be touched only once the value products of tile j-1 are done.
        if (!(ok = wait_warp(o_done, (j - 1) & 1))) break;
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
#pragma unroll 1
          for (int part = 0; part < 8; ++part) {
            uint32_t ov[32];
            const uint32_t addr = tmem + lane_off + kColO1 + part * 32;   // O1 and O2 are contiguous
            tmem_ld32(addr, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(addr, ov);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[b2]);
    }
    if (!ok) *abort_flag = 1;
    // ---- epilogue: wait for the last value products, then write the rows
    if (ok && wait_warp(o_done, (n - 1) & 1)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const float corr = 1.f + c * inv;
      const size_t orow = ((size_t)(b * a.H + h) * a.T + t) * kPfD;
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {
        uint32_t o1[32], o2[32];
        tmem_ld32(tmem + lane_off + kColO1 + part * 32, o1);
        tmem_ld32(tmem + lane_off + kColO2 + part * 32, o2);
        tmem_wait_ld();
        if (t < a.T) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o1[i]) * inv * corr - __uint_as_float(o2[i]) * inv;
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
