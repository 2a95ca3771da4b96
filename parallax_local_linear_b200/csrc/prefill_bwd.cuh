// Parallax prefill backward on sm_100a: TMA, tcgen05.mma, tensor memory.
//
// For one query row t with visible keys i, softmax weights w_i, probe values
// a_i = rho.k_i, abar = sum w_i a_i and vbar = sum w_i v_i, the forward output
// (the covariance correction of the wispaper.ai blog "Parallax: Breaking the
// Boundary Bias with Parameterized Local Linear Attention", section "The Core
// Insight: Covariance Correction") can be written
//     out = sum_i w_i (1 + abar - a_i) v_i.
// With g = dL/dout, D_i = g.v_i, Gbar = g.vbar, Delta = g.out and
// x_i = D_i - Gbar, differentiating gives (derived here, not printed on the
// pages):
//     dv_i   += w_i (1 + abar - a_i) g                     (u_i = w_i (1 + abar - a_i))
//     dA_i    = -w_i x_i                                   (dL/da_i)
//     dS_i    = w_i ((1 + abar - a_i) x_i + Gbar - Delta)  (dL/ds_i, s_i = scale q.k_i)
//     dq      = scale sum_i dS_i k_i,      drho = sum_i dA_i k_i,
//     dk_i   += scale dS_i q + dA_i rho.
// w_i = 2^(s_i scale log2(e) - lse2) comes back from the forward's per-row
// lse2 = m + log2(l); abar and vbar come from the forward too.
//
// Three launches:
//   prefill_bwd_rows_kernel  per row: Gbar = g.vbar, Delta = g.out, packed
//                            with (lse2, abar) into one float4.
//   prefill_bwd_dq_kernel    query-stationary: one CTA per 128-row query tile
//                            streams the key tiles it sees; S = QK^T,
//                            A = RK^T, D = GV^T (tcgen05, fp32 in TMEM), the
//                            elementwise warps form dS and dA in bf16, and
//                            dQ += dS K, dR += dA K accumulate in TMEM.
//   prefill_bwd_dkv_kernel   key-stationary: one CTA per 128-key tile of one
//                            KV head streams the 64-row query tiles (of every
//                            query head of its group) that see it;
//                            S^T = KQ^T, A^T = KR^T, D^T = VG^T, and
//                            dV += U^T G, dK += dS^T Q + dA^T R.  Its
//                            elementwise warps take 16 query columns at a
//                            time; the queries' row records come with their
//                            Q, R, G tiles.
// No atomics: every output element is written once, by one CTA.
#pragma once

#include "ptx.cuh"
#include "prefill.cuh"

namespace plx {

struct BwdArgs {
  int B, H, Hkv, T, group;
  int n_blk;                      // dq: ceil(T / 128) query tiles; dkv: ceil(T / 128) key tiles
  int causal, out_bf16;
  float scale, scale_log2;
  const float4* rows;             // [B, H, T]: (lse2, 1 + abar, Gbar, Gbar - Delta)
  void* dq;                       // [B, H, T, D]
  void* drho;                     // [B, H, T, D]
  void* dk;                       // [B, Hkv, T, D]
  void* dv;                       // [B, Hkv, T, D]
  unsigned long long wait_ns;     // limit of one pipeline wait (0: give up unless complete)
};

// ------------------------------------------------------------- MMA issue
// Several MMAs under one elect.sync, issued in argument order, each with its
// own accumulate flag: the issuing warp pays tens of cycles per elect.sync
// block, so the backward's many small products go out four at a time.
__device__ __forceinline__ void bwd_mma_ss4(uint32_t d0, uint64_t a0, uint64_t b0, uint32_t c0, uint32_t d1,
                                            uint64_t a1, uint64_t b1, uint32_t c1, uint32_t d2, uint64_t a2,
                                            uint64_t b2, uint32_t c2, uint32_t d3, uint64_t a3, uint64_t b3,
                                            uint32_t c3, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1, p2, p3, e;\n\t"
      "setp.ne.b32 p0, %12, 0;\n\tsetp.ne.b32 p1, %13, 0;\n\tsetp.ne.b32 p2, %14, 0;\n\tsetp.ne.b32 p3, %15, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %16, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], %4, %5, %16, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%6], %7, %8, %16, p2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%9], %10, %11, %16, p3;\n\t}" ::"r"(d0),
      "l"(a0), "l"(b0), "r"(d1), "l"(a1), "l"(b1), "r"(d2), "l"(a2), "l"(b2), "r"(d3), "l"(a3), "l"(b3), "r"(c0),
      "r"(c1), "r"(c2), "r"(c3), "r"(idesc)
      : "memory");
}

// The same with A in tensor memory.
__device__ __forceinline__ void bwd_mma_ts4(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t c0, uint32_t d1,
                                            uint32_t a1, uint64_t b1, uint32_t c1, uint32_t d2, uint32_t a2,
                                            uint64_t b2, uint32_t c2, uint32_t d3, uint32_t a3, uint64_t b3,
                                            uint32_t c3, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1, p2, p3, e;\n\t"
      "setp.ne.b32 p0, %12, 0;\n\tsetp.ne.b32 p1, %13, 0;\n\tsetp.ne.b32 p2, %14, 0;\n\tsetp.ne.b32 p3, %15, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %16, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], [%4], %5, %16, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%6], [%7], %8, %16, p2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%9], [%10], %11, %16, p3;\n\t}" ::"r"(d0),
      "r"(a0), "l"(b0), "r"(d1), "r"(a1), "l"(b1), "r"(d2), "r"(a2), "l"(b2), "r"(d3), "r"(a3), "l"(b3), "r"(c0),
      "r"(c1), "r"(c2), "r"(c3), "r"(idesc)
      : "memory");
}

__device__ __forceinline__ void bwd_mma_ts2(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t c0, uint32_t d1,
                                            uint32_t a1, uint64_t b1, uint32_t c1, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1, e;\n\t"
      "setp.ne.b32 p0, %6, 0;\n\tsetp.ne.b32 p1, %7, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %8, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], [%4], %5, %8, p1;\n\t}" ::"r"(d0),
      "r"(a0), "l"(b0), "r"(d1), "r"(a1), "l"(b1), "r"(c0), "r"(c1), "r"(idesc)
      : "memory");
}

// ---------------------------------------------------------------- per row
// One warp per row: Gbar = g.vbar, Delta = g.out.  out is the forward output
// in its own dtype (the loss saw those values).  The record holds the
// row's constants in the form the elementwise warps use:
// (lse2, 1 + abar, Gbar, Gbar - Delta).
//
// It also writes the row's offsets for the key-stationary kernel's products,
// as bf16 hi / lo pairs in a 64-column row: columns 0, 1 hold -lse2 / c
// (c = scale * log2(e)), 16, 17 hold -(1 + abar), 32, 33 hold -Gbar, the rest
// 0.  A product's extra k-step against a block of ones adds them, so that
// kernel reads S - lse2 / c, A - (1 + abar) and D - Gbar straight from TMEM.
template <bool kOutBf16>
__global__ void __launch_bounds__(256) prefill_bwd_rows_kernel(const __nv_bfloat16* __restrict__ dout,
                                                               const void* __restrict__ out,
                                                               const float* __restrict__ vbar,
                                                               const float2* __restrict__ stats,
                                                               float4* __restrict__ rows,
                                                               uint32_t* __restrict__ slab, float scale_log2,
                                                               long long n_rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const size_t base = (size_t)row * kPfD + lane * 4;
  const uint2 gr = *reinterpret_cast<const uint2*>(dout + base);
  const float g0 = bf16_lo_f(gr.x), g1 = bf16_hi_f(gr.x), g2 = bf16_lo_f(gr.y), g3 = bf16_hi_f(gr.y);
  float o0, o1, o2, o3;
  if constexpr (kOutBf16) {
    const uint2 orw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(out) + base);
    o0 = bf16_lo_f(orw.x), o1 = bf16_hi_f(orw.x), o2 = bf16_lo_f(orw.y), o3 = bf16_hi_f(orw.y);
  } else {
    const float4 ov = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(out) + base);
    o0 = ov.x, o1 = ov.y, o2 = ov.z, o3 = ov.w;
  }
  const float4 vb = *reinterpret_cast<const float4*>(vbar + base);
  float delta = g0 * o0 + g1 * o1 + g2 * o2 + g3 * o3;
  float gbar = g0 * vb.x + g1 * vb.y + g2 * vb.z + g3 * vb.w;
  delta = warp_sum(delta);
  gbar = warp_sum(gbar);
  const float2 st = stats[row];
  if (lane == 0) rows[row] = make_float4(st.x, 1.f + st.y, gbar, gbar - delta);
  // lane j writes bf16 columns 2j, 2j+1 of the slab row
  float off = 0.f;
  if (lane == 0) off = -st.x / scale_log2;
  if (lane == 8) off = -(1.f + st.y);
  if (lane == 16) off = -gbar;
  const uint32_t hi = pack_bf16(off, 0.f) & 0xffffu;
  const float lo = off - bf16_lo_f(hi);
  slab[(size_t)row * 32 + lane] = (lane == 0 || lane == 8 || lane == 16) ? (hi | (pack_bf16(lo, 0.f) << 16)) : 0u;
}

// One element of the backward: u, scale * dS and dA of one (query, key)
// pair.  A pair that is not visible gives zeros by selection: its inputs may
// be anything (unloaded row records, keys past the end), NaN included.
struct BwdElem {
  float u, ds, da;
};
__device__ __forceinline__ BwdElem bwd_elem(float s, float a, float dv, float lse2, float c1a, float gbar,
                                            float gmd, float scale_log2, float scale, bool visible) {
  const float w = ex2(s * scale_log2 - lse2);
  const float e1 = c1a - a;   // c1a = 1 + abar
  const float x = dv - gbar;
  BwdElem r;
  r.u = visible ? w * e1 : 0.f;
  r.da = visible ? -w * x : 0.f;
  r.ds = visible ? (w * scale) * fmaf(e1, x, gmd) : 0.f;   // gmd = Gbar - Delta
  return r;
}

// The same for two pairs at once, on packed f32x2 arithmetic, every pair
// visible.  s2, a2, d2: the two columns' S, A, D; r0, r1: the two queries'
// records.  Returns packed bf16 (u, scale*dS, dA) pairs.
__device__ __forceinline__ uint3 bwd_pair_visible(float2 s2, float2 a2, float2 d2, float4 r0, float4 r1,
                                                  float scale_log2, float scale) {
  const float2 x2 = fma2(s2, make_float2(scale_log2, scale_log2), make_float2(-r0.x, -r1.x));
  const float2 w2 = make_float2(ex2(x2.x), ex2(x2.y));
  const float2 e1 = add2(make_float2(r0.y, r1.y), make_float2(-a2.x, -a2.y));      // 1 + abar - a
  const float2 nx = add2(make_float2(r0.z, r1.z), make_float2(-d2.x, -d2.y));      // Gbar - D = -x
  const float2 u = mul2(w2, e1);
  const float2 da = mul2(w2, nx);
  const float2 t = fma2(e1, make_float2(-nx.x, -nx.y), make_float2(r0.w, r1.w));   // e1 x + Gbar - Delta
  const float2 ds = mul2(mul2(w2, make_float2(scale, scale)), t);
  return make_uint3(pack_bf16(u.x, u.y), pack_bf16(ds.x, ds.y), pack_bf16(da.x, da.y));
}

// The key-stationary kernel's version, on products whose offsets are folded
// in: sp = S - lse2 / c, ap = A - (1 + abar) = -(1 + abar - a),
// dp = D - Gbar = x; gmd = Gbar - Delta.  Then u = -w ap, dA = -w dp and
// scale * dS = -w scale (ap dp - gmd).
__device__ __forceinline__ uint3 bwd_pair_folded(float2 sp, float2 ap, float2 dp, float2 gmd, float scale_log2,
                                                 float scale) {
  const float2 x2 = mul2(sp, make_float2(scale_log2, scale_log2));
  const float2 nw = make_float2(-ex2(x2.x), -ex2(x2.y));
  const float2 u = mul2(nw, ap);
  const float2 da = mul2(nw, dp);
  const float2 t = fma2(ap, dp, make_float2(-gmd.x, -gmd.y));
  const float2 ds = mul2(mul2(nw, make_float2(scale, scale)), t);
  return make_uint3(pack_bf16(u.x, u.y), pack_bf16(ds.x, ds.y), pack_bf16(da.x, da.y));
}
__device__ __forceinline__ BwdElem bwd_elem_folded(float sp, float ap, float dp, float gmd, float scale_log2,
                                                   float scale, bool visible) {
  const float nw = -ex2(sp * scale_log2);
  BwdElem r;
  r.u = visible ? nw * ap : 0.f;
  r.da = visible ? nw * dp : 0.f;
  r.ds = visible ? (nw * scale) * fmaf(ap, dp, -gmd) : 0.f;
  return r;
}

// TMEM columns shared by both kernels.
constexpr uint32_t kBwAcc0 = 0, kBwAcc1 = 128;                 // dQ, dR  |  dK, dV
constexpr uint32_t kBwS = 256, kBwA = 320, kBwD = 384;         // fp32 products of the current tile
constexpr uint32_t kBwDS = 448, kBwDA = 480;                   // bf16 dS, dA of the current tile

// ------------------------------------------------------------- dq kernel
constexpr int kBqStages = 3;
struct BqLayout {
  static constexpr int kTile128 = 128 * kPfD * 2;   // 32 KB: two 64-column boxes of 128 rows
  static constexpr int kTile64 = 64 * kPfD * 2;     // 16 KB: two 64-column boxes of 64 rows
  static constexpr int kQ = 0, kR = kQ + kTile128, kG = kR + kTile128;
  static constexpr int kK = kG + kTile128;
  static constexpr int kV = kK + kBqStages * kTile64;
  static constexpr int kBar = kV + kBqStages * kTile64;
  // q_full, k_full[S], v_full[S], k_empty[S], v_empty[S], sad_full, sad_free, dd_full, dd_free, drain
  static constexpr int kNumBars = 1 + 4 * kBqStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;
};

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                          const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const BwdArgs a) {
  using Ly = BqLayout;
  constexpr int S = kBqStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + S;
  uint64_t* k_empty = v_full + S;
  uint64_t* v_empty = k_empty + S;
  uint64_t* sad_full = v_empty + S;   // S, A, D of the current tile are in TMEM
  uint64_t* sad_free = sad_full + 1;  // the elementwise warps have read them
  uint64_t* dd_full = sad_free + 1;   // dS, dA are in TMEM
  uint64_t* dd_free = dd_full + 1;    // the products reading dS, dA are done
  uint64_t* drain = dd_free + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kMisc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = a.B * a.H;
  const int mblk = a.n_blk - 1 - (int)(blockIdx.x / BH);   // longest first
  const int bh = blockIdx.x % BH;
  const int b = bh / a.H, h = bh % a.H, kvh = h / a.group;
  const int m0 = mblk * kPfBM;
  const int kv_end = a.causal ? min(a.T, m0 + kPfBM) : a.T;
  const int n = (kv_end + kPfBN - 1) / kPfBN;
  const int q_row = (b * a.H + h) * a.T + m0;
  const int kv_row = (b * a.Hkv + kvh) * a.T;
  // Rows with fewer than 128 keys do not average out the bf16 rounding of
  // dS and dA (dA is ~16/n per key and sums to zero): their key tiles (the
  // first two) also enter the products as bf16 lo parts, kept in the D
  // columns this half has already read.
  const int split_tiles = (a.causal ? min(m0 + 1, a.T) : a.T) < 2 * kPfBN ? kPfSplitTiles : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(sad_full, 1);
    mbar_init(sad_free, kPfSoftmax);
    mbar_init(dd_full, kPfSoftmax);
    mbar_init(dd_free, 1);
    mbar_init(drain, 1);
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
      prefetch_tmap(&tm_g);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, 3 * Ly::kTile128);
      for (int bx = 0; bx < 2; ++bx) {
        tma_load_2d(sm + Ly::kQ + bx * (Ly::kTile128 / 2), &tm_q, bx * 64, q_row, q_full, once);
        tma_load_2d(sm + Ly::kR + bx * (Ly::kTile128 / 2), &tm_r, bx * 64, q_row, q_full, once);
        tma_load_2d(sm + Ly::kG + bx * (Ly::kTile128 / 2), &tm_g, bx * 64, q_row, q_full, once);
      }
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % S;
        const uint32_t par = ((j / S) - 1) & 1;
        const int row = kv_row + j * kPfBN;
        if (j >= S && !(ok = mbar_wait_bounded(a.wait_ns, &k_empty[s], par))) break;
        mbar_arrive_expect_tx(&k_full[s], Ly::kTile64);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_2d(sm + Ly::kK + s * Ly::kTile64 + bx * (Ly::kTile64 / 2), &tm_k, bx * 64, row, &k_full[s], keep);
        ++issued_k;
        if (j >= S && !(ok = mbar_wait_bounded(a.wait_ns, &v_empty[s], par))) break;
        mbar_arrive_expect_tx(&v_full[s], Ly::kTile64);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_2d(sm + Ly::kV + s * Ly::kTile64 + bx * (Ly::kTile64 / 2), &tm_v, bx * 64, row, &v_full[s], keep);
        ++issued_v;
      }
      // Every issued load must land before the CTA exits.
      mbar_wait_drain(q_full, 0);
      for (int s = 0; s < S && s < issued_k; ++s)
        mbar_wait_drain(&k_full[s], ((s + ((issued_k - 1 - s) / S) * S) / S) & 1);
      for (int s = 0; s < S && s < issued_v; ++s)
        mbar_wait_drain(&v_full[s], ((s + ((issued_v - 1 - s) / S) * S) / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_bf16(kPfBM, kPfBN, false);   // 128 x 64, K-major B
    constexpr uint32_t kIdT = idesc_bf16(kPfBM, kPfD, true);     // 128 x 128, MN-major B
    const uint64_t dq = smem_desc_sw128(smem_u32(sm + Ly::kQ), 16, 1024);
    const uint64_t dr = smem_desc_sw128(smem_u32(sm + Ly::kR), 16, 1024);
    const uint64_t dg = smem_desc_sw128(smem_u32(sm + Ly::kG), 16, 1024);
    const uint64_t dk = smem_desc_sw128(smem_u32(sm + Ly::kK), 16, 1024);
    const uint64_t dkt = smem_desc_sw128(smem_u32(sm + Ly::kK), Ly::kTile64 / 2, 1024);   // K as an MN-major B
    const uint64_t dv = smem_desc_sw128(smem_u32(sm + Ly::kV), 16, 1024);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, bar, parity));
    };
    bool ok = wait_warp(q_full, 0);
    tc_fence_after();
    // dQ += dS K, dR += dA K of tile jp (with the lo parts of a split tile)
    auto value_products = [&](int jp) {
      const int sp = jp % S;
      const uint64_t kts = dkt + (uint64_t)((sp * Ly::kTile64) >> 4);
      // 16 keys per step: 8 TMEM columns of packed bf16 pairs, 16 rows of K;
      // two steps per issue block
#pragma unroll
      for (int kk = 0; kk < kPfBN / 16; kk += 2) {
        const uint64_t kd0 = kts + (uint64_t)(kk * 16 * 128 / 16), kd1 = kd0 + (uint64_t)(16 * 128 / 16);
        const uint32_t c0 = (jp > 0 || kk > 0) ? 1u : 0u;
        bwd_mma_ts4(tmem + kBwAcc0, tmem + kBwDS + kk * 8, kd0, c0, tmem + kBwAcc1, tmem + kBwDA + kk * 8, kd0, c0,
                    tmem + kBwAcc0, tmem + kBwDS + kk * 8 + 8, kd1, 1u, tmem + kBwAcc1, tmem + kBwDA + kk * 8 + 8, kd1,
                    1u, kIdT);
      }
      if (jp < split_tiles) {   // lo parts: keys 32h.. of dS at D + 32h, of dA at D + 32h + 16
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; kk += 2) {
          const uint64_t kd0 = kts + (uint64_t)(kk * 16 * 128 / 16), kd1 = kd0 + (uint64_t)(16 * 128 / 16);
          const uint32_t pc = kBwD + 32u * (kk >> 1);   // kk even: 8 (kk & 1) = 0, then + 8 for kk + 1
          bwd_mma_ts4(tmem + kBwAcc0, tmem + pc, kd0, 1u, tmem + kBwAcc1, tmem + pc + 16, kd0, 1u, tmem + kBwAcc0,
                      tmem + pc + 8, kd1, 1u, tmem + kBwAcc1, tmem + pc + 24, kd1, 1u, kIdT);
        }
      }
      tc_commit(dd_free);
      tc_commit(&k_empty[sp]);   // K(jp) is done: scores and dQ, dR
    };
    for (int j = 0; ok && j <= n; ++j) {
      // A split tile's lo parts sit in the D columns, so its value products
      // go ahead of the next tile's score products (which rewrite D).
      const bool early = j >= 1 && j - 1 < split_tiles;
      if (early) {
        if (!(ok = wait_warp(dd_full, (j - 1) & 1))) break;
        tc_fence_after();
        value_products(j - 1);
      }
      if (j < n) {
        const int s = j % S;
        if (!(ok = wait_warp(&k_full[s], (j / S) & 1))) break;
        if (!(ok = wait_warp(&v_full[s], (j / S) & 1))) break;
        if (j >= 1 && !(ok = wait_warp(sad_free, (j - 1) & 1))) break;
        tc_fence_after();
        const uint64_t dks = dk + (uint64_t)((s * Ly::kTile64) >> 4);
        const uint64_t dvs = dv + (uint64_t)((s * Ly::kTile64) >> 4);
        // S, A, D for k-steps kk = 0..7 in that order, four products per issue block
#pragma unroll
        for (int g4 = 0; g4 < 3 * (kPfD / 16) / 4; ++g4) {
          uint32_t d[4], c[4];
          uint64_t aa[4], bb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = 4 * g4 + u, kk = i / 3, which = i % 3;
            const uint64_t oa = (uint64_t)((kk >> 2) * (Ly::kTile128 / 2 / 16) + (kk & 3) * 2);
            const uint64_t ob = (uint64_t)((kk >> 2) * (Ly::kTile64 / 2 / 16) + (kk & 3) * 2);
            d[u] = tmem + (which == 0 ? kBwS : which == 1 ? kBwA : kBwD);
            aa[u] = (which == 0 ? dq : which == 1 ? dr : dg) + oa;
            bb[u] = (which == 2 ? dvs : dks) + ob;
            c[u] = kk > 0 ? 1u : 0u;
          }
          bwd_mma_ss4(d[0], aa[0], bb[0], c[0], d[1], aa[1], bb[1], c[1], d[2], aa[2], bb[2], c[2], d[3], aa[3], bb[3],
                      c[3], kIdS);
        }
        tc_commit(sad_full);
        tc_commit(&v_empty[s]);   // V(j) only enters D
      }
      if (j >= 1 && !early) {
        if (!(ok = wait_warp(dd_full, (j - 1) & 1))) break;
        tc_fence_after();
        value_products(j - 1);
      }
    }
    if (!ok && lane == 0) report_error(2 /* PLX_DEVERR_TIMEOUT */);
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise
    const int g = (warp - 2) >> 2;           // key-column half of every tile
    const int wq = warp & 3;
    const int r = wq * 32 + lane;            // query row within the tile
    const int t = m0 + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int key_lim = a.causal ? min(t + 1, a.T) : a.T;
    const float4 rs = t < a.T ? a.rows[(size_t)(b * a.H + h) * a.T + t] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float lse2 = rs.x, abar = rs.y, gbar = rs.z, gmd = rs.w;   // abar holds 1 + abar
    bool fine = true;
    int j = 0;
    for (; j < n; ++j) {
      fine = __all_sync(0xffffffffu, fine && mbar_wait_bounded(a.wait_ns, sad_full, j & 1));
      if (!fine) break;
      tc_fence_after();
      uint32_t sr[32], ar[32], dr[32];
      tmem_ld32(tmem + lane_off + kBwS + 32 * g, sr);
      tmem_ld32(tmem + lane_off + kBwA + 32 * g, ar);
      tmem_ld32(tmem + lane_off + kBwD + 32 * g, dr);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(sad_free);
      const int key0 = j * kPfBN + 32 * g;
      // The split and the mask are separate instantiations so that ordinary
      // tiles (every key of this half visible to every row of this warp) run
      // a loop without either, on f32x2 pair arithmetic.
      auto form = [&](auto split_tag, auto mask_tag) -> bool {
        constexpr bool kSplit = decltype(split_tag)::value;
        constexpr bool kMask = decltype(mask_tag)::value;
        uint32_t pds[16], pda[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if constexpr (!kMask) {
            const float4 r4 = make_float4(lse2, abar, gbar, gmd);
            const uint3 pk = bwd_pair_visible(
                make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                make_float2(__uint_as_float(ar[2 * i]), __uint_as_float(ar[2 * i + 1])),
                make_float2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])), r4, r4, a.scale_log2,
                a.scale);
            pds[i] = pk.y;
            pda[i] = pk.z;
            static_assert(!kSplit || kMask, "split tiles take the masked path, which keeps fp32 values");
          } else {
            const BwdElem e0 = bwd_elem(__uint_as_float(sr[2 * i]), __uint_as_float(ar[2 * i]),
                                        __uint_as_float(dr[2 * i]), lse2, abar, gbar, gmd, a.scale_log2, a.scale,
                                        key0 + 2 * i < key_lim);
            const BwdElem e1 = bwd_elem(__uint_as_float(sr[2 * i + 1]), __uint_as_float(ar[2 * i + 1]),
                                        __uint_as_float(dr[2 * i + 1]), lse2, abar, gbar, gmd, a.scale_log2,
                                        a.scale, key0 + 2 * i + 1 < key_lim);
            pds[i] = pack_bf16(e0.ds, e1.ds);
            pda[i] = pack_bf16(e0.da, e1.da);
            if constexpr (kSplit) {   // lo parts reuse entries already consumed (sr[i], ar[i]: i <= 2i)
              sr[i] = pack_bf16(e0.ds - bf16_lo_f(pds[i]), e1.ds - bf16_hi_f(pds[i]));
              ar[i] = pack_bf16(e0.da - bf16_lo_f(pda[i]), e1.da - bf16_hi_f(pda[i]));
            }
          }
        }
        // The products of tile j-1 must be done with the dS / dA columns.
        if (j >= 1) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, dd_free, (j - 1) & 1))) return false;
          tc_fence_after();
        }
        tmem_st16(tmem + lane_off + kBwDS + 16 * g, pds);
        tmem_st16(tmem + lane_off + kBwDA + 16 * g, pda);
        if constexpr (kSplit) {   // into this half's own D columns, already read
          tmem_st16(tmem + lane_off + kBwD + 32 * g, sr);
          tmem_st16(tmem + lane_off + kBwD + 32 * g + 16, ar);
        }
        return true;
      };
      // rows t0w..t0w+31 of this warp against keys key0..key0+31 of this half
      const int t0w = m0 + wq * 32;
      const bool all_vis = key0 + 31 < a.T && (a.causal ? key0 + 31 <= t0w : true);
      if (j < split_tiles)
        fine = form(std::true_type{}, std::true_type{});
      else
        fine = all_vis ? form(std::false_type{}, std::false_type{}) : form(std::false_type{}, std::true_type{});
      if (!fine) break;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(dd_full);
    }
    // ---- epilogue: the last dQ, dR products, then the rows
    fine = __all_sync(0xffffffffu, fine && j == n && mbar_wait_bounded(a.wait_ns, dd_free, (n - 1) & 1));
    if (fine) {
      tc_fence_after();
      const size_t orow = ((size_t)(b * a.H + h) * a.T + t) * kPfD + 64 * g;
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {   // dQ cols 64g, 64g+32; dR cols 64g, 64g+32
        uint32_t o[32];
        const int acc = part >> 1, half = part & 1;
        tmem_ld32(tmem + lane_off + (acc ? kBwAcc1 : kBwAcc0) + 64 * g + 32 * half, o);
        tmem_wait_ld();
        if (t < a.T) {
          void* base = acc ? a.drho : a.dq;
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + orow + 32 * half);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(__uint_as_float(o[8 * i]), __uint_as_float(o[8 * i + 1])),
                                  pack_bf16(__uint_as_float(o[8 * i + 2]), __uint_as_float(o[8 * i + 3])),
                                  pack_bf16(__uint_as_float(o[8 * i + 4]), __uint_as_float(o[8 * i + 5])),
                                  pack_bf16(__uint_as_float(o[8 * i + 6]), __uint_as_float(o[8 * i + 7])));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + orow + 32 * half);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                   __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ dkv kernel
constexpr int kBkStages = 2;
struct BkLayout {
  static constexpr int kTile128 = 128 * kPfD * 2;   // 32 KB
  static constexpr int kTile64 = 64 * kPfD * 2;     // 16 KB
  static constexpr int kSlab64 = 64 * 64 * 2;       // 8 KB: 64 rows of 64 bf16 columns
  static constexpr int kK = 0, kV = kK + kTile128;
  static constexpr int kOnes = kV + kTile128;       // 128 rows of 64 bf16 ones (the A side of the offset k-step)
  // one stage: Q, R, G tiles of 64 query rows, their offset slab and their
  // 64 row records (they arrive with the tiles, long before they are read)
  static constexpr int kStQ = 0, kStR = kTile64, kStG = 2 * kTile64, kStSlab = 3 * kTile64;
  static constexpr int kStRows = kStSlab + kSlab64;
  static constexpr int kStage = kStRows + 1024;       // 57 KB, a multiple of 1024
  static constexpr int kRing = kOnes + 2 * kSlab64;
  static constexpr int kBar = kRing + kBkStages * kStage;
  // kv_full, op_full[S], op_empty[S], sad_full, sad_free, dd_full[2], dd_free, drain
  static constexpr int kNumBars = 1 + 2 * kBkStages + 6;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;
};

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                           const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_slab,
                           const BwdArgs a) {
  using Ly = BkLayout;
  constexpr int S = kBkStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* kv_full = bars;
  uint64_t* op_full = bars + 1;
  uint64_t* op_empty = op_full + S;
  uint64_t* sad_full = op_empty + S;
  uint64_t* sad_free = sad_full + 1;
  uint64_t* dd_full = sad_free + 1;   // [2]: U, dS, dA of pass 0 / 1 are in TMEM
  uint64_t* dd_free = dd_full + 2;    // the products reading them are done
  uint64_t* drain = dd_free + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kMisc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BHk = a.B * a.Hkv;
  const int kb = (int)(blockIdx.x / BHk);   // causal: the first key tiles see the most queries
  const int bk = blockIdx.x % BHk;
  const int b = bk / a.Hkv, kvh = bk % a.Hkv;
  const int k0 = kb * kPfBM;
  const int nq_all = (a.T + kPfBN - 1) / kPfBN;
  const int qb0 = a.causal ? k0 / kPfBN : 0;
  const int nq = nq_all - qb0;                // query tiles per query head
  const int N = a.group * nq;                  // iterations: (head of the group, query tile)
  const int kv_row = (b * a.Hkv + kvh) * a.T + k0;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&op_full[s], 1);
      mbar_init(&op_empty[s], 1);
    }
    mbar_init(sad_full, 1);
    mbar_init(sad_free, kPfSoftmax);
    mbar_init(&dd_full[0], kPfSoftmax);
    mbar_init(&dd_full[1], kPfSoftmax);
    mbar_init(dd_free, 1);
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, 512);
    tmem_relinquish();
  }
  // The A side of the offset k-step: bf16 ones (every column, so the swizzle
  // does not matter).
  for (int i = threadIdx.x; i < 2 * Ly::kSlab64 / 16; i += kPfThreads)
    reinterpret_cast<uint4*>(sm + Ly::kOnes)[i] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  auto head_of = [&](int it) { return kvh * a.group + it / nq; };
  auto tile_of = [&](int it) { return qb0 + it % nq; };
  // Query tiles whose rows see fewer than 128 keys (the first two, causal)
  // do not average out the bf16 rounding of U, dS and dA: they also enter
  // the products as bf16 lo parts, kept in this half's A / D columns.
  auto split_of = [&](int it) {
    return a.causal ? tile_of(it) * kPfBN + 1 < 2 * kPfBN : a.T < 2 * kPfBN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_r);
      prefetch_tmap(&tm_g);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_slab);
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(kv_full, 2 * Ly::kTile128);
      for (int bx = 0; bx < 2; ++bx) {
        tma_load_2d(sm + Ly::kK + bx * (Ly::kTile128 / 2), &tm_k, bx * 64, kv_row, kv_full, once);
        tma_load_2d(sm + Ly::kV + bx * (Ly::kTile128 / 2), &tm_v, bx * 64, kv_row, kv_full, once);
      }
      int issued = 0;
      for (int it = 0; it < N; ++it) {
        const int s = it % S;
        if (it >= S && !mbar_wait_bounded(a.wait_ns, &op_empty[s], ((it / S) - 1) & 1)) break;
        const int hq = head_of(it), t0 = tile_of(it) * kPfBN;
        const int row = (b * a.H + hq) * a.T + t0;
        const int nrows = min(kPfBN, a.T - t0);   // row records past T are not read
        uint8_t* st = sm + Ly::kRing + s * Ly::kStage;
        mbar_arrive_expect_tx(&op_full[s], 3 * Ly::kTile64 + Ly::kSlab64 + nrows * 16);
        for (int bx = 0; bx < 2; ++bx) {
          tma_load_2d(st + Ly::kStQ + bx * (Ly::kTile64 / 2), &tm_q, bx * 64, row, &op_full[s], keep);
          tma_load_2d(st + Ly::kStR + bx * (Ly::kTile64 / 2), &tm_r, bx * 64, row, &op_full[s], keep);
          tma_load_2d(st + Ly::kStG + bx * (Ly::kTile64 / 2), &tm_g, bx * 64, row, &op_full[s], keep);
        }
        tma_load_2d(st + Ly::kStSlab, &tm_slab, 0, row, &op_full[s], keep);
        bulk_load(st + Ly::kStRows, a.rows + (size_t)(b * a.H + hq) * a.T + t0, (uint32_t)nrows * 16, &op_full[s]);
        ++issued;
      }
      mbar_wait_drain(kv_full, 0);
      for (int s = 0; s < S && s < issued; ++s)
        mbar_wait_drain(&op_full[s], ((s + ((issued - 1 - s) / S) * S) / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_bf16(kPfBM, kPfBN, false);   // 128 keys x 64 queries, K-major B
    constexpr uint32_t kIdT = idesc_bf16(kPfBM, kPfD, true);     // 128 keys x 128, MN-major B
    const uint64_t dk = smem_desc_sw128(smem_u32(sm + Ly::kK), 16, 1024);
    const uint64_t dvv = smem_desc_sw128(smem_u32(sm + Ly::kV), 16, 1024);
    const uint64_t dones = smem_desc_sw128(smem_u32(sm + Ly::kOnes), 16, 1024);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, bar, parity));
    };
    bool ok = wait_warp(kv_full, 0);
    tc_fence_after();
    // dV += U^T G, dK += dS^T Q + dA^T R of query tile ip, for the queries of
    // elementwise pass q: 16q.. (first warpgroup) and 32 + 16q.. (second),
    // i.e. k-steps kk = q and q + 2 (plus lo parts if split).
    auto value_products = [&](int ip, int q) {
      const int sp = ip % S;
      const uint32_t stp = smem_u32(sm + Ly::kRing + sp * Ly::kStage);
      const uint64_t tq = smem_desc_sw128(stp + Ly::kStQ, Ly::kTile64 / 2, 1024);
      const uint64_t tr = smem_desc_sw128(stp + Ly::kStR, Ly::kTile64 / 2, 1024);
      const uint64_t tg = smem_desc_sw128(stp + Ly::kStG, Ly::kTile64 / 2, 1024);
      // 16 queries per step.  U of queries 16kk.. sits in columns 16kk..16kk+7
      // of the S^T block (its lo parts in 16kk+8..), dS / dA in 8kk..8kk+7 of
      // their own blocks (lo parts: 16kk.. and 16kk+8.. of the A^T block).
      // Steps kk = q and q + 2; the products go out four (or two) per issue
      // block in the order: hi parts of kk = q, then of q + 2, then the lo parts.
      const int k0 = q, k1 = q + 2;
      const uint64_t ko0 = (uint64_t)(k0 * 16 * 128 / 16), ko1 = (uint64_t)(k1 * 16 * 128 / 16);
      const uint32_t acc0 = (ip > 0 || k0 > 0) ? 1u : 0u;   // k1 > 0: always accumulates
      bwd_mma_ts4(tmem + kBwAcc1, tmem + kBwS + 16 * k0, tg + ko0, acc0, tmem + kBwAcc0, tmem + kBwDS + k0 * 8,
                  tq + ko0, acc0, tmem + kBwAcc0, tmem + kBwDA + k0 * 8, tr + ko0, 1u, tmem + kBwAcc1,
                  tmem + kBwS + 16 * k1, tg + ko1, 1u, kIdT);
      bwd_mma_ts2(tmem + kBwAcc0, tmem + kBwDS + k1 * 8, tq + ko1, 1u, tmem + kBwAcc0, tmem + kBwDA + k1 * 8,
                  tr + ko1, 1u, kIdT);
      if (split_of(ip)) {
        bwd_mma_ts4(tmem + kBwAcc1, tmem + kBwS + 16 * k0 + 8, tg + ko0, 1u, tmem + kBwAcc0, tmem + kBwA + 16 * k0,
                    tq + ko0, 1u, tmem + kBwAcc0, tmem + kBwA + 16 * k0 + 8, tr + ko0, 1u, tmem + kBwAcc1,
                    tmem + kBwS + 16 * k1 + 8, tg + ko1, 1u, kIdT);
        bwd_mma_ts2(tmem + kBwAcc0, tmem + kBwA + 16 * k1, tq + ko1, 1u, tmem + kBwAcc0, tmem + kBwA + 16 * k1 + 8,
                    tr + ko1, 1u, kIdT);
      }
      if (q == 1) {
        tc_commit(dd_free);
        tc_commit(&op_empty[sp]);
      }
    };
    auto both_passes = [&](int ip) -> bool {
      for (int q = 0; q < 2; ++q) {
        if (!wait_warp(&dd_full[q], ip & 1)) return false;
        tc_fence_after();
        value_products(ip, q);
      }
      return true;
    };
    for (int it = 0; ok && it <= N; ++it) {
      const int s = it % S;
      const uint32_t st = smem_u32(sm + Ly::kRing + s * Ly::kStage);
      // A split tile's lo parts sit in the A columns, so its products go
      // ahead of this tile's A^T, D^T (which rewrite them).
      const bool early = it >= 1 && split_of(it - 1);
      if (early && !(ok = both_passes(it - 1))) break;
      if (it < N) {
        if (!(ok = wait_warp(&op_full[s], (it / S) & 1))) break;
        if (it >= 1 && !(ok = wait_warp(sad_free, (it - 1) & 1))) break;
        tc_fence_after();
        const uint64_t br = smem_desc_sw128(st + Ly::kStR, 16, 1024);
        const uint64_t bg = smem_desc_sw128(st + Ly::kStG, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; kk += 2) {   // A^T, D^T of steps kk and kk + 1 per issue block
          const uint64_t oa0 = (uint64_t)((kk >> 2) * (Ly::kTile128 / 2 / 16) + (kk & 3) * 2), oa1 = oa0 + 2;
          const uint64_t ob0 = (uint64_t)((kk >> 2) * (Ly::kTile64 / 2 / 16) + (kk & 3) * 2), ob1 = ob0 + 2;
          const uint32_t c0 = kk > 0 ? 1u : 0u;
          bwd_mma_ss4(tmem + kBwA, dk + oa0, br + ob0, c0, tmem + kBwD, dvv + oa0, bg + ob0, c0, tmem + kBwA,
                      dk + oa1, br + ob1, 1u, tmem + kBwD, dvv + oa1, bg + ob1, 1u, kIdS);
        }
        // offsets: A^T -= 1 + abar (slab columns 16..31), D^T -= Gbar (32..47)
        const uint64_t bsl = smem_desc_sw128(st + Ly::kStSlab, 16, 1024);
        tc_mma_ss(tmem + kBwA, dones, bsl + 2, kIdS, 1u);
        tc_mma_ss(tmem + kBwD, dones, bsl + 4, kIdS, 1u);
      }
      // U of the previous tile sits in the S^T columns, which S^T of this
      // tile overwrites below.
      if (it >= 1 && !early && !(ok = both_passes(it - 1))) break;
      if (it < N) {
        const uint64_t bq = smem_desc_sw128(st + Ly::kStQ, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; kk += 4) {   // four k-steps per issue block
          uint64_t aa[4], bb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            aa[u] = dk + (uint64_t)(((kk + u) >> 2) * (Ly::kTile128 / 2 / 16) + ((kk + u) & 3) * 2);
            bb[u] = bq + (uint64_t)(((kk + u) >> 2) * (Ly::kTile64 / 2 / 16) + ((kk + u) & 3) * 2);
          }
          bwd_mma_ss4(tmem + kBwS, aa[0], bb[0], kk > 0 ? 1u : 0u, tmem + kBwS, aa[1], bb[1], 1u, tmem + kBwS, aa[2],
                      bb[2], 1u, tmem + kBwS, aa[3], bb[3], 1u, kIdS);
        }
        tc_mma_ss(tmem + kBwS, dones, smem_desc_sw128(st + Ly::kStSlab, 16, 1024), kIdS, 1u);   // S^T -= lse2 / c
        tc_commit(sad_full);
      }
    }
    if (!ok && lane == 0) report_error(2 /* PLX_DEVERR_TIMEOUT */);
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise
    const int g = (warp - 2) >> 2;           // query-column half of every tile
    const int wq = warp & 3;
    const int r = wq * 32 + lane;            // key row within the tile
    const int key = k0 + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    bool fine = true;
    int it = 0;
    for (; it < N; ++it) {
      fine = __all_sync(0xffffffffu, fine && mbar_wait_bounded(a.wait_ns, sad_full, it & 1));
      if (!fine) break;
      tc_fence_after();
      const int t0 = tile_of(it) * kPfBN + 32 * g;   // query of this thread's first column
      // this half's 32 queries' row records, in the stage (entries past T are stale and masked)
      const float4* rows_s =
          reinterpret_cast<const float4*>(sm + Ly::kRing + (it % S) * Ly::kStage + Ly::kStRows) + 32 * g;
      // every pair of this warp's 32 keys and this half's 32 queries visible?
      const int kw0 = k0 + wq * 32;
      const bool all_vis = kw0 + 31 < a.T && t0 + 31 < a.T && (!a.causal || t0 >= kw0 + 31);
      const bool split = split_of(it);   // rare: the first two query tiles of the first key tile
      // S^T, A^T, D^T of this half's 32 queries, all read at once so that the
      // next tile's A^T, D^T products can start while this tile is worked on.
      uint32_t sr[32], ar[32], dr[32];
      tmem_ld32(tmem + lane_off + kBwS + 32 * g, sr);
      tmem_ld32(tmem + lane_off + kBwA + 32 * g, ar);
      tmem_ld32(tmem + lane_off + kBwD + 32 * g, dr);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(sad_free);
      // Two passes of 16 queries; after each, the value products of its
      // queries may start (dd_full[q]).  Every output lands in columns
      // already read: U of queries 16kk.. (kk = 2g + q) in S^T columns
      // 16kk..16kk+7 (lo parts 16kk+8..), dS / dA in their own blocks, the lo
      // parts of dS / dA in A^T columns 16kk.. and 16kk+8..
      auto pass = [&](auto q_tag, auto split_tag, auto mask_tag) -> bool {
        constexpr int q = decltype(q_tag)::value;
        constexpr bool kSplit = decltype(split_tag)::value;
        constexpr bool kMask = decltype(mask_tag)::value;
        const uint32_t col = 32u * g + 16u * q;
        float gw[16];   // Gbar - Delta of the pass's 16 queries (the rest is folded into S, A, D)
#pragma unroll
        for (int c = 0; c < 16; ++c) gw[c] = rows_s[16 * q + c].w;
        uint32_t pu[8], pds[8], pda[8], lu[8], lds[8], lda[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int cc = 16 * q + 2 * i;
          if constexpr (!kMask) {
            const uint3 pk = bwd_pair_folded(make_float2(__uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1])),
                                             make_float2(__uint_as_float(ar[cc]), __uint_as_float(ar[cc + 1])),
                                             make_float2(__uint_as_float(dr[cc]), __uint_as_float(dr[cc + 1])),
                                             make_float2(gw[2 * i], gw[2 * i + 1]), a.scale_log2, a.scale);
            pu[i] = pk.x;
            pds[i] = pk.y;
            pda[i] = pk.z;
            static_assert(!kSplit || kMask, "split tiles take the masked path, which keeps fp32 values");
          } else {
            BwdElem e[2];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int tq = t0 + cc + c;
              const bool vis = key < a.T && tq < a.T && (!a.causal || key <= tq);
              e[c] = bwd_elem_folded(__uint_as_float(sr[cc + c]), __uint_as_float(ar[cc + c]),
                                     __uint_as_float(dr[cc + c]), gw[2 * i + c], a.scale_log2, a.scale, vis);
            }
            pu[i] = pack_bf16(e[0].u, e[1].u);
            pds[i] = pack_bf16(e[0].ds, e[1].ds);
            pda[i] = pack_bf16(e[0].da, e[1].da);
            if constexpr (kSplit) {
              lu[i] = pack_bf16(e[0].u - bf16_lo_f(pu[i]), e[1].u - bf16_hi_f(pu[i]));
              lds[i] = pack_bf16(e[0].ds - bf16_lo_f(pds[i]), e[1].ds - bf16_hi_f(pds[i]));
              lda[i] = pack_bf16(e[0].da - bf16_lo_f(pda[i]), e[1].da - bf16_hi_f(pda[i]));
            }
          }
        }
        // The products of the previous tile must be done with the dS / dA columns.
        if (q == 0 && it >= 1) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, dd_free, (it - 1) & 1))) return false;
          tc_fence_after();
        }
        tmem_st8(tmem + lane_off + kBwS + col, pu);
        tmem_st8(tmem + lane_off + kBwDS + 16 * g + 8 * q, pds);
        tmem_st8(tmem + lane_off + kBwDA + 16 * g + 8 * q, pda);
        if constexpr (kSplit) {
          tmem_st8(tmem + lane_off + kBwS + col + 8, lu);
          tmem_st8(tmem + lane_off + kBwA + col, lds);
          tmem_st8(tmem + lane_off + kBwA + col + 8, lda);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&dd_full[q]);
        return true;
      };
      auto run_pass = [&](auto q_tag) {
        if (split)
          return pass(q_tag, std::true_type{}, std::true_type{});
        return all_vis ? pass(q_tag, std::false_type{}, std::false_type{})
                       : pass(q_tag, std::false_type{}, std::true_type{});
      };
      fine = run_pass(std::integral_constant<int, 0>{}) && run_pass(std::integral_constant<int, 1>{});
      if (!fine) break;
    }
    // ---- epilogue: the last products, then the key rows
    fine = __all_sync(0xffffffffu, fine && it == N && mbar_wait_bounded(a.wait_ns, dd_free, (N - 1) & 1));
    if (fine) {
      tc_fence_after();
      const size_t orow = ((size_t)(b * a.Hkv + kvh) * a.T + key) * kPfD + 64 * g;
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {   // dK cols 64g, 64g+32; dV cols 64g, 64g+32
        uint32_t o[32];
        const int acc = part >> 1, half = part & 1;
        tmem_ld32(tmem + lane_off + (acc ? kBwAcc1 : kBwAcc0) + 64 * g + 32 * half, o);
        tmem_wait_ld();
        if (key < a.T) {
          void* base = acc ? a.dv : a.dk;
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + orow + 32 * half);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(__uint_as_float(o[8 * i]), __uint_as_float(o[8 * i + 1])),
                                  pack_bf16(__uint_as_float(o[8 * i + 2]), __uint_as_float(o[8 * i + 3])),
                                  pack_bf16(__uint_as_float(o[8 * i + 4]), __uint_as_float(o[8 * i + 5])),
                                  pack_bf16(__uint_as_float(o[8 * i + 6]), __uint_as_float(o[8 * i + 7])));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + orow + 32 * half);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                   __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace plx
