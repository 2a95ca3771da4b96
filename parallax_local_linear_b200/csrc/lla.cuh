// Local Linear Attention (LLA) with the solved probe, decode form, sm_100a.
//
// LLA is the local linear estimate at the query: the intercept of the
// softmax-weighted least-squares fit v ~ a + M^T (k - q) (newx.sg page
// "Parallax: Parameterized Local Linear Attention for Language Modeling",
// section "Abstract"; the wispaper.ai blog "Parallax: Breaking the Boundary
// Bias with Parameterized Local Linear Attention", section "Context: Why
// Softmax is Not Enough", where LLA solves a linear system for every token).
// With weights w_i = softmax(scale q.k_i), kbar = sum w k, vbar = sum w v,
//     S_KK = sum w (k - kbar)(k - kbar)^T,  S_KV = sum w (k - kbar)(v - vbar)^T,
//     (S_KK + ridge I) rho* = kbar - q,       out = vbar - S_KV^T rho*,
// the same output as Parallax with the probe solved instead of learned.
// `ridge` penalises the slope (the pages name no regularisation; 0 is plain
// LLA).
//
// Two kernels per call:
//
//   lla_moments_kernel  one CTA per (sequence, query head, piece of its keys):
//     a single pass over the piece's K and V tiles accumulates, relative to
//     a running max m (2^(s - m) weights, rescaled lazily as in the prefill),
//         l = sum e,  ks = sum e k,  vs = sum e v,
//         D_KK = sum e k k^T,  D_KV = sum e k v^T          (128 x 128 each)
//     The products over keys run on the tensor cores: per 64-key tile the
//     scores S = K q (M = 64 keys, N = 8: q is row 0 of an 8-row operand),
//     read back by four warps, 16 keys each; the weights e (rounded to bf16
//     once, so that every sum uses the same values) go into diag(e) in
//     shared memory; the MMA G = K^T diag(e) (the K tile read as an MN-major
//     A operand) puts e_i k_ia, exact in fp32, in row a of G; the compute
//     warps pack G into A = (e o K)^T in tensor memory (bf16 pairs) and sum
//     its rows into ks; then [D_KK | D_KV] += A . [K | V] (N = 256: a
//     stage's K and V tiles are one MN-major B operand).  The issuing warp
//     spends ~40 cycles per MMA, so the count matters more than the size:
//     sixteen per tile.  vs is summed on the CUDA cores from the V tile
//     while the compute warps wait for the gather.  For sequences shorter
//     than kLlaSplitLen the bf16 rounding of e o K is not averaged away (the
//     solve amplifies it along directions the few keys do not span), so a
//     second product adds its lo part (x = hi + lo).  The piece's record
//     goes to the workspace.
//
//   lla_solve_kernel  one CTA per (sequence, query head): merges the pieces
//     like online softmax (weights 2^(m_j - M)), forms S_KK + ridge I and
//     kbar - q in fp32, solves by Cholesky, and writes rho* and
//         out = vbar (1 + kbar . rho*) - (1 / l) sum_a D_KV[a, :] rho*_a,
//     which is vbar - S_KV^T rho* (S_KV = D_KV / l - kbar vbar^T).
#pragma once

#include "ptx.cuh"
#include "decode.cuh"    // kTile (64-token tiles and pages)
#include "prefill.cuh"   // tc_mma_ts4

#include <type_traits>

namespace plx {

constexpr int kLlaD = 128;
constexpr int kLlaStages = 4;            // K and V ring depth (tiles)
constexpr int kLlaThreads = 320;         // TMA producer warp, MMA warp, eight compute warps
constexpr int kLlaCompute = 256;
constexpr int kLlaSplitLen = 1024;       // shorter sequences add the lo part of e o K
constexpr float kLlaRescaleLog2 = 8.f;   // lazy rescale threshold (factor 256)
constexpr int kLlaMaxPieces = 16;
// Record of one piece: D_KK, D_KV (column-major: [a][b] at b * 128 + a), ks,
// vs, then m, l.
constexpr int kLlaRecKK = 0;
constexpr int kLlaRecKV = kLlaD * kLlaD;
constexpr int kLlaRecKs = 2 * kLlaD * kLlaD;
constexpr int kLlaRecVs = kLlaRecKs + kLlaD;
constexpr int kLlaRecM = kLlaRecVs + kLlaD;
constexpr int kLlaRecFloats = kLlaRecM + 16;

#define PLX_DEVERR_SINGULAR_BIT 8   // PLX_DEVERR_SINGULAR in parallax.h

struct LlaArgs {
  const __nv_bfloat16* q;          // [B, Hq, D]
  const int32_t* page_table;       // [B, max_pages] or null (contiguous)
  const int32_t* seq_lens;         // [B] or null (every sequence kv_len)
  float* rec;                      // [B * Hq * pieces][kLlaRecFloats]
  void* out;                       // [B, Hq, D] of out dtype
  float* rho;                      // [B, Hq, D] or null
  int B, Hq, Hkv, group, kv_len, paged, num_pages, max_pages, pieces;
  float scale_log2, ridge;
  int out_bf16;
  unsigned long long wait_ns;      // limit of one pipeline wait
};

struct LlaLayout {
  static constexpr int kTileBytes = kTile * kLlaD * 2;   // 16 KB: two 64-column boxes of 64 rows
  // Stage s: the K tile, then the V tile, so that the four 64-column boxes
  // [K lo | K hi | V lo | V hi] are one MN-major operand of 256 columns.
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kKV = 0;
  static constexpr int kDiagBytes = kTile * kTile * 2;        // bf16 [64][64]: diag(e), 128-byte swizzle
  static constexpr int kDiag = kKV + kLlaStages * kStageBytes;   // two buffers (tile parity)
  static constexpr int kQBytes = 8 * kLlaD * 2;               // bf16 [8][128]: row 0 = q, rows 1.. zero
  static constexpr int kQ = kDiag + 2 * kDiagBytes;           // K-major B operand, two 64-column atoms
  static constexpr int kE = kQ + kQBytes;                     // float [2][64]: the tile's weights e
  static constexpr int kRed = kE + 2 * kTile * 4;             // float [8 warps][2]
  static constexpr int kBar = kRed + 64;
  // full[S], empty[S], e_ready[2], da_full[2], da_free[2], a_full, a_free,
  // drain, s_full[2] (the per-tile hand-offs that run a tile ahead alternate
  // between two barriers by tile parity, so neither side can be two phases
  // ahead)
  static constexpr int kNumBars = 2 * kLlaStages + 11;
  static constexpr int kMisc = kBar + kNumBars * 8;           // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16 + 1024;            // + alignment slack
};

// TMEM columns: D = [D_KK | D_KV] in [0, 256); A: hi words at 256, lo words
// at 288 (keys 2c, 2c+1 in word c); the gather G = K^T diag(e) of tile j at
// 320 + 64 (j % 2); the scores of tile j at 480 + 8 (j % 2) (M = 64: key r
// in lane (r % 16) + 32 (r / 16), column 0).
constexpr uint32_t kLlaColKK = 0, kLlaColKV = 128, kLlaColA = 256;
__device__ __forceinline__ uint32_t lla_col_g(int buf) { return 320u + 64u * buf; }
__device__ __forceinline__ uint32_t lla_col_s(int buf) { return 480u + 8u * buf; }

// Four MMAs into one accumulator under one elect.sync (four k-steps): the
// first takes the accumulate flag acc0, the others accumulate.
__device__ __forceinline__ void lla_mma4_ss(uint32_t d, uint64_t a0, uint64_t b0, uint64_t a1, uint64_t b1,
                                            uint64_t a2, uint64_t b2, uint64_t a3, uint64_t b3, uint32_t idesc,
                                            uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1, e;\n\tsetp.ne.b32 p0, %10, 0;\n\tsetp.eq.b32 p1, %10, %10;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %9, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %9, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %9, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %9, p1;\n\t}" ::"r"(d),
      "l"(a0), "l"(b0), "l"(a1), "l"(b1), "l"(a2), "l"(b2), "l"(a3), "l"(b3), "r"(idesc), "r"(acc0)
      : "memory");
}

__device__ __forceinline__ void lla_mma4_ts(uint32_t d, uint32_t a0, uint64_t b0, uint32_t a1, uint64_t b1,
                                            uint32_t a2, uint64_t b2, uint32_t a3, uint64_t b3, uint32_t idesc,
                                            uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1, e;\n\tsetp.ne.b32 p0, %10, 0;\n\tsetp.eq.b32 p1, %10, %10;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %9, p0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %4, %9, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %6, %9, p1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %8, %9, p1;\n\t}" ::"r"(d),
      "r"(a0), "l"(b0), "r"(a1), "l"(b1), "r"(a2), "l"(b2), "r"(a3), "l"(b3), "r"(idesc), "r"(acc0)
      : "memory");
}

// One 32-bit column of this thread's TMEM lane.
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}

// Named barrier over nthreads threads; true in all of them if v is true in any.
__device__ __forceinline__ bool bar_or(uint32_t id, uint32_t nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ int lla_seq_len(const LlaArgs& a, int b) {
  if (a.seq_lens == nullptr) return a.kv_len;
  int n = __ldg(a.seq_lens + b);
  if (n < 0 || n > a.kv_len) {
    report_error(4 /* PLX_DEVERR_BAD_LENGTH */);
    n = n < 0 ? 0 : a.kv_len;
  }
  return n;
}

// Byte offset of element (row, col) of a [rows][64] bf16 tile with the
// 128-byte swizzle (16-byte chunks XORed with the row within each 8 rows).
__device__ __forceinline__ int sw128_off(int row, int col) {
  return row * 128 + ((((col >> 3) ^ (row & 7)) << 4)) + (col & 7) * 2;
}

// Instruction descriptor of kind::f16 with both operands' majorness given
// (bf16 A and B, fp32 accumulator, shape M x N).
__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__global__ void __launch_bounds__(kLlaThreads, 1)
    lla_moments_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const LlaArgs a) {
  using Ly = LlaLayout;
  constexpr int S = kLlaStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* empty = full + S;
  uint64_t* e_ready = empty + S;
  uint64_t* da_full = e_ready + 2;
  uint64_t* da_free = da_full + 2;
  uint64_t* a_full = da_free + 2;
  uint64_t* a_free = a_full + 1;
  uint64_t* drain = a_free + 1;
  uint64_t* s_full = drain + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::kMisc + 4);
  float* red_s = reinterpret_cast<float*>(sm + Ly::kRed);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int piece = blockIdx.x % a.pieces;
  const int bh = blockIdx.x / a.pieces;
  const int b = bh / a.Hq, h = bh % a.Hq, kvh = h / a.group;
  float* rec = a.rec + (size_t)blockIdx.x * kLlaRecFloats;
  const int len = lla_seq_len(a, b);
  const int tiles = (len + kTile - 1) / kTile;
  const int t0 = (int)((long long)piece * tiles / a.pieces);
  const int n = (int)((long long)(piece + 1) * tiles / a.pieces) - t0;
  if (n == 0) {   // no keys in this piece: an empty record
    if (threadIdx.x == 0) {
      rec[kLlaRecM] = -INFINITY;
      rec[kLlaRecM + 1] = 0.f;
    }
    return;
  }
  const int32_t* pt = a.paged ? a.page_table + (size_t)b * a.max_pages : nullptr;
  if (a.paged) {   // every page this piece reads must lie in the pool
    bool bad = false;
    for (int i = threadIdx.x; i < n; i += kLlaThreads) {
      const int pg = __ldg(pt + t0 + i);
      bad |= pg < 0 || pg >= a.num_pages;
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) {
        report_error(1 /* PLX_DEVERR_BAD_PAGE */);
        rec[kLlaRecM] = -INFINITY;
        rec[kLlaRecM + 1] = 0.f;
      }
      return;
    }
  }
  const bool split_lo = len < kLlaSplitLen;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&e_ready[i], kLlaCompute);
      mbar_init(&da_full[i], 1);
      mbar_init(&da_free[i], kLlaCompute);
      mbar_init(&s_full[i], 1);
    }
    mbar_init(a_full, kLlaCompute);
    mbar_init(a_free, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x < Ly::kQBytes / 16) {
    // 16-byte chunk i of the q operand: atom i / 64 (components 64 (i / 64) ..),
    // row (i / 8) % 8, chunk i % 8; row 0 is not swizzled and holds q
    const int i = threadIdx.x;
    alignas(16) __nv_bfloat16 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = ((i >> 3) & 7) == 0 ? a.q[(size_t)bh * kLlaD + (i >> 6) * 64 + (i & 7) * 8 + e] : __float2bfloat16_rn(0.f);
    *reinterpret_cast<uint4*>(sm + Ly::kQ + i * 16) = *reinterpret_cast<const uint4*>(v);
  }
  // diag(e) starts as zeros; only its diagonal changes per tile
  for (int i = threadIdx.x; i < 2 * Ly::kDiagBytes / 16; i += kLlaThreads)
    reinterpret_cast<uint4*>(sm + Ly::kDiag)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
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
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % S;
        if (j >= S && !mbar_wait_bounded(a.wait_ns, &empty[s], ((j / S) - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int tile = t0 + j;
        const int row = a.paged ? (__ldg(pt + tile) * a.Hkv + kvh) * kTile   // page ids checked above
                                : (b * a.Hkv + kvh) * a.kv_len + tile * kTile;
        uint8_t* st = sm + Ly::kKV + s * Ly::kStageBytes;
        mbar_arrive_expect_tx(&full[s], Ly::kStageBytes);
        for (int bx = 0; bx < 2; ++bx) {
          tma_load_2d(st + bx * (Ly::kTileBytes / 2), &tm_k, bx * 64, row, &full[s], pol);
          tma_load_2d(st + Ly::kTileBytes + bx * (Ly::kTileBytes / 2), &tm_v, bx * 64, row, &full[s], pol);
        }
        ++issued;
      }
      // Every issued load must land before the CTA exits.
      for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / S) * S;
        mbar_wait_drain(&full[s], (last / S) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per tile: the scores S = K q (M = 64 keys, N = 8, K-major A and B); the
    // gather G = K^T diag(e) (128 x 64, A = the K tile read as MN-major,
    // B = diag(e)); once the compute warps have packed G into
    // A = (e o K)^T: [D_KK | D_KV] += A . [K | V] (TS, 128 x 256, the stage's
    // K and V tiles as one MN-major B operand).  Sixteen MMAs per tile (24
    // below kLlaSplitLen keys), four under each elect.
    constexpr uint32_t kIdS = idesc_bf16_ab(kTile, 8, false, false);
    constexpr uint32_t kIdG = idesc_bf16_ab(128, kTile, true, false);
    constexpr uint32_t kIdD = idesc_bf16(128, 2 * kLlaD, true);
    const uint64_t dkS = smem_desc_sw128(smem_u32(sm + Ly::kKV), 16, 1024);                  // K, K-major A
    const uint64_t dqS = smem_desc_sw128(smem_u32(sm + Ly::kQ), 16, 1024);                   // q, K-major B
    const uint64_t dkvM = smem_desc_sw128(smem_u32(sm + Ly::kKV), Ly::kTileBytes / 2, 1024);   // MN-major, 64-col atoms
    const uint64_t dd = smem_desc_sw128(smem_u32(sm + Ly::kDiag), 16, 1024);                 // diag(e), K-major B
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, bar, parity));
    };
    auto stage_off = [&](int j) { return (uint64_t)(((j % S) * Ly::kStageBytes) >> 4); };
    // main(j) = [D_KK | D_KV] += A . [K(j) | V(j)]; A holds tile j's packed
    // gather (16 keys = 8 A words and 16 B rows, 2048 bytes, per step).
    // Issue order S(0), S(1), then per tile j: G(j), main(j - 1), S(j + 2):
    // the gather of the next tile runs while the compute warps pack this
    // one, and the scores are two tiles ahead.
    auto issue_main = [&](int jm) {
      const uint64_t kv = dkvM + stage_off(jm);
      const uint32_t ahi = tmem + kLlaColA;
      lla_mma4_ts(tmem + kLlaColKK, ahi, kv, ahi + 8u, kv + 128, ahi + 16u, kv + 256, ahi + 24u, kv + 384, kIdD,
                  jm > 0 ? 1u : 0u);
      if (split_lo) {
        const uint32_t alo = ahi + 32u;
        lla_mma4_ts(tmem + kLlaColKK, alo, kv, alo + 8u, kv + 128, alo + 16u, kv + 256, alo + 24u, kv + 384, kIdD,
                    1u);
      }
      tc_commit(a_free);
      tc_commit(&empty[jm % S]);
    };
    // S(js) once tile js has landed (buffer js % 2: the scores of tile js - 2
    // have been read, which e_ready(js - 2) reported before G(js - 2)).
    // 16 components per step: box kk / 4, 32 bytes into the 128-byte row.
    auto issue_s = [&](int js) -> bool {
      if (!wait_warp(&full[js % S], (js / S) & 1)) return false;
      tc_fence_after();
      const uint64_t ka = dkS + stage_off(js);
      constexpr uint64_t kBoxA = Ly::kTileBytes / 2 / 16, kBoxB = Ly::kQBytes / 2 / 16;
      const uint32_t d = tmem + lla_col_s(js & 1);
      lla_mma4_ss(d, ka, dqS, ka + 2, dqS + 2, ka + 4, dqS + 4, ka + 6, dqS + 6, kIdS, 0u);
      lla_mma4_ss(d, ka + kBoxA, dqS + kBoxB, ka + kBoxA + 2, dqS + kBoxB + 2, ka + kBoxA + 4, dqS + kBoxB + 4,
                  ka + kBoxA + 6, dqS + kBoxB + 6, kIdS, 1u);
      tc_commit(&s_full[js & 1]);
      return true;
    };
    bool ok = issue_s(0) && (n < 2 || issue_s(1));
    for (int j = 0; ok && j <= n; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (j < n) {   // G(j) (tile j has landed: S(j) waited for it)
        const int gb = j & 1;
        if (!(ok = wait_warp(&e_ready[gb], (j >> 1) & 1))) break;
        if (j >= 2 && !(ok = wait_warp(&da_free[gb], ((j >> 1) - 1) & 1))) break;   // G buffer gb was read
        tc_fence_after();
        // 16 keys per step: 16 rows (2048 bytes) of the K tile, 32 bytes of diag(e)
        const uint64_t ks = dkvM + stage_off(j);
        const uint64_t ddb = dd + (uint64_t)((gb * Ly::kDiagBytes) >> 4);
        lla_mma4_ss(tmem + lla_col_g(gb), ks, ddb, ks + 128, ddb + 2, ks + 256, ddb + 4, ks + 384, ddb + 6, kIdG, 0u);
        tc_commit(&da_full[gb]);
      }
      if (j >= 1) {   // main(j - 1), once the compute warps have packed tile j - 1
        if (!(ok = wait_warp(a_full, (j - 1) & 1))) break;
        tc_fence_after();
        issue_main(j - 1);
      }
      if (j + 2 < n && !(ok = issue_s(j + 2))) break;
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // Every issued MMA must complete before tensor memory is released.
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute
    // Two warps per TMEM lane quarter: warp cw (0..7) takes rows 32 (warp % 4)
    // .. of the accumulators and the keys 32 kh .. 32 kh + 31 of each tile's
    // gather (kh = cw / 4).
    const int c = threadIdx.x - 64;            // 0..255
    const int cw = warp - 2;                   // compute warp 0..7
    const int kh = cw >> 2;                    // key half of the gather this thread packs
    const int wq = warp & 3;                   // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;            // TMEM lane = component a of k
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // Score phase: warps with cw < 4 read the scores of keys 16 wq .. 16 wq + 15
    // (TMEM lanes 32 wq .. 32 wq + 15 of the M = 64 product), one per lane.
    const bool skey = cw < 4 && lane < 16;
    const int key = 16 * wq + lane;
    // sum e v: thread c takes components 2 (c % 64), + 1 and keys 16 (c / 64) ..
    // of each tile (a warp reads whole 128-byte rows of one V box).
    const int vcp = c & 63, vkq = c >> 6, vchunk = (vcp & 31) >> 2;
    const int voff = Ly::kTileBytes + (vcp >> 5) * (Ly::kTileBytes / 2) + (vcp & 3) * 4;   // + row, swizzled chunk
    float m_ref = -INFINITY, l_acc = 0.f;
    float ks_acc = 0.f;                        // sum e k_row over this thread's key half
    float vs0 = 0.f, vs1 = 0.f;                // sum e v over this thread's key quarter
    // Tile t's scores, weights, diag(e) and e (buffers t % 2), then e_ready.
    // The running max moves only when a score passes it by kLlaRescaleLog2
    // (one barrier reduction per tile decides; the first tile always takes
    // its max).  A new running max returns the factor that everything
    // accumulated over tiles < t takes before tile t is added.
    auto scores_phase = [&](int t, float& alpha_d) -> bool {
      const int gb = t & 1;
      const bool w = __all_sync(0xffffffffu, !*abort_flag && mbar_wait_bounded(a.wait_ns, &s_full[gb], (t >> 1) & 1));
      const int nvalid = min(kTile, len - (t0 + t) * kTile);
      float sc = -INFINITY;
      if (w && cw < 4) {   // warp-uniform
        tc_fence_after();
        const uint32_t r = tmem_ld1(tmem + lane_off + lla_col_s(gb));
        tmem_wait_ld();
        if (skey && key < nvalid) sc = __uint_as_float(r) * a.scale_log2;
      }
      alpha_d = 1.f;
      if (bar_or(1, kLlaCompute, t == 0 || !w || sc > m_ref + kLlaRescaleLog2)) {   // uniform
        if (!bar_and(2, kLlaCompute, w)) return false;
        const float wmax = warp_max(sc);
        if (lane == 0) red_s[cw] = wmax;
        bar_and(3, kLlaCompute, true);
        const float tmax = fmaxf(fmaxf(fmaxf(red_s[0], red_s[1]), fmaxf(red_s[2], red_s[3])),
                                 fmaxf(fmaxf(red_s[4], red_s[5]), fmaxf(red_s[6], red_s[7])));
        if (t == 0) {
          m_ref = tmax;   // the piece's first tile holds a key: tmax is finite
        } else if (tmax > m_ref + kLlaRescaleLog2) {   // uniform: every compute thread saw the same maxima
          alpha_d = ex2(m_ref - tmax);
          m_ref = tmax;
          l_acc *= alpha_d;
        }
      }
      // ---- the weights, rounded to bf16: every product below uses these values
      if (skey) {   // every key of the tile, its weight 0 past the end
        const float e = key < nvalid ? __bfloat162float(__float2bfloat16_rn(ex2(sc - m_ref))) : 0.f;
        l_acc += e;
        __nv_bfloat16* diag_s = reinterpret_cast<__nv_bfloat16*>(sm + Ly::kDiag + gb * Ly::kDiagBytes);
        diag_s[sw128_off(key, key) >> 1] = __float2bfloat16_rn(e);
        reinterpret_cast<float*>(sm + Ly::kE)[gb * kTile + key] = e;
      }
      if (nvalid < kTile) {
        // Rows past the end are operands of the gather and the products
        // (their weights are 0, but 0 * NaN is not): zero them in K and V.
        // S(t), the only earlier reader of the tile, is done (s_full).
        uint8_t* st = sm + Ly::kKV + (t % S) * Ly::kStageBytes;
        for (int i = c; i < (kTile - nvalid) * 16; i += kLlaCompute) {
          const int r = nvalid + (i >> 4), cc = i & 15;   // cc: box (cc >> 3), chunk (cc & 7)
          const int off = (cc >> 3) * (Ly::kTileBytes / 2) + r * 128 + (cc & 7) * 16;
          *reinterpret_cast<uint4*>(st + off) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(st + Ly::kTileBytes + off) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&e_ready[gb]);
      return true;
    };
    // Tile t: sum e v over this thread's keys (while G(t) and main(t - 1) run;
    // V(t) stays resident until main(t), after a_full(t), is done), then the
    // gather into A = (e o K)^T (after main(t - 1) has read A), the deferred
    // rescale of D, and sum e k from the gather's rows.
    auto pack_phase = [&](int t, float alpha_d) -> bool {
      const int gb = t & 1;
      {
        const float* et = reinterpret_cast<const float*>(sm + Ly::kE) + gb * kTile + 16 * vkq;
        const uint8_t* vt = sm + Ly::kKV + (t % S) * Ly::kStageBytes + voff;
        // Rows past the end hold zeros (scores(t) cleared them; a barrier
        // since orders that before these reads) and weight 0.
        uint32_t w2[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)   // row 16 vkq + jj, whose swizzle is jj % 8
          w2[jj] = *reinterpret_cast<const uint32_t*>(vt + (16 * vkq + jj) * 128 + ((vchunk ^ (jj & 7)) << 4));
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 e4 = lds_f4(smem_u32(et + 4 * q4));
          const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            a0 = fmaf(ev[u], bf16_lo_f(w2[4 * q4 + u]), a0);
            a1 = fmaf(ev[u], bf16_hi_f(w2[4 * q4 + u]), a1);
            b0 = fmaf(ev[u + 1], bf16_lo_f(w2[4 * q4 + u + 1]), b0);
            b1 = fmaf(ev[u + 1], bf16_hi_f(w2[4 * q4 + u + 1]), b1);
          }
        }
        vs0 = fmaf(vs0, alpha_d, a0 + b0);
        vs1 = fmaf(vs1, alpha_d, a1 + b1);
      }
      const bool wg = mbar_wait_bounded(a.wait_ns, &da_full[gb], (t >> 1) & 1);
      const bool wa = t == 0 || mbar_wait_bounded(a.wait_ns, a_free, (t - 1) & 1);
      if (!bar_and(2, kLlaCompute, wg && wa)) return false;
      tc_fence_after();
      if (alpha_d != 1.f) {   // uniform; main(t - 1) is done
#pragma unroll 1
        for (int part = 4 * kh; part < 4 * kh + 4; ++part) {   // D_KK (kh 0) or D_KV (kh 1), 32 columns at a time
          uint32_t r[32];
          const uint32_t addr = tmem + lane_off + (uint32_t)(part * 32);
          tmem_ld32(addr, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha_d);
          tmem_st32(addr, r);
        }
      }
      uint32_t g[32];
      tmem_ld32(tmem + lane_off + lla_col_g(gb) + 32u * kh, g);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&da_free[gb]);
      auto pack = [&](auto split_tag) {
        constexpr bool kSplit = decltype(split_tag)::value;
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float p0 = __uint_as_float(g[2 * p]), p1 = __uint_as_float(g[2 * p + 1]);
          hi[p] = pack_bf16(p0, p1);
          if constexpr (kSplit) lo[p] = pack_bf16(p0 - bf16_lo_f(hi[p]), p1 - bf16_hi_f(hi[p]));
        }
        tmem_st16(tmem + lane_off + kLlaColA + 16u * kh, hi);
        if constexpr (kSplit) tmem_st16(tmem + lane_off + kLlaColA + 32u + 16u * kh, lo);
      };
      if (split_lo)
        pack(std::true_type{});
      else
        pack(std::false_type{});
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(a_full);
      // G holds e_i k_ia exactly (one nonzero product per entry)
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 32; ++i) s4[i & 3] += __uint_as_float(g[i]);
      ks_acc = fmaf(ks_acc, alpha_d, (s4[0] + s4[1]) + (s4[2] + s4[3]));
      return true;
    };
    // scores(t + 1) runs before pack(t), so the gather of tile t + 1 overlaps
    // the packing of tile t and main(t).
    float alpha_pack = 1.f;   // the rescale before tile t is added, decided by scores(t)
    bool fine = scores_phase(0, alpha_pack);
    int j = 0;
    for (; fine && j < n; ++j) {
      float alpha_next = 1.f;
      if (j + 1 < n) {
        if (!(fine = scores_phase(j + 1, alpha_next))) break;
      } else {
        bar_and(1, kLlaCompute, true);   // the last tile's weights, visible to every compute thread
      }
      if (!(fine = pack_phase(j, alpha_pack))) break;
      alpha_pack = alpha_next;
    }
    // ---- the piece's record: wait for the last products, then write
    bool wl = fine && j == n && !*abort_flag && mbar_wait_bounded(a.wait_ns, a_free, (n - 1) & 1);
    wl = bar_and(3, kLlaCompute, wl);
    const float lw = warp_sum(l_acc);
    if (lane == 0) red_s[8 + cw] = lw;
    // the first moments' partial sums meet in the diag buffers, idle once
    // the last products are done: [2][128] halves of sum e k, [4][128]
    // quarters of sum e v
    float* scr = reinterpret_cast<float*>(sm + Ly::kDiag);
    if (wl) {
      scr[kh * kLlaD + row] = ks_acc;
      scr[2 * kLlaD + vkq * kLlaD + 2 * vcp] = vs0;
      scr[2 * kLlaD + vkq * kLlaD + 2 * vcp + 1] = vs1;
    }
    bar_and(2, kLlaCompute, true);
    if (wl) {
      tc_fence_after();
#pragma unroll 1
      for (int part = 4 * kh; part < 4 * kh + 4; ++part) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + (uint32_t)(part * 32), r);
        tmem_wait_ld();
        // column-major: element [a][b] at b * 128 + a, so that the warp's 32
        // lanes (consecutive a) write 128 contiguous bytes per column
        float* dst = rec + (part < 4 ? kLlaRecKK : kLlaRecKV) + (part & 3) * 32 * kLlaD + row;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[i * kLlaD] = __uint_as_float(r[i]);
      }
      if (kh == 0)
        rec[kLlaRecKs + row] = scr[row] + scr[kLlaD + row];
      else
        rec[kLlaRecVs + row] = (scr[2 * kLlaD + row] + scr[3 * kLlaD + row]) +
                               (scr[4 * kLlaD + row] + scr[5 * kLlaD + row]);
      if (c == 0) {
        float lt = 0.f;
        for (int w = 0; w < 8; ++w) lt += red_s[8 + w];
        rec[kLlaRecM] = m_ref;
        rec[kLlaRecM + 1] = lt;
      }
    } else if (c == 0) {   // abandoned after a wait ran out (already reported): an empty record
      rec[kLlaRecM] = -INFINITY;
      rec[kLlaRecM + 1] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- solve
// One CTA (256 threads) per (sequence, query head).  Thread (bi, bj) of a
// 16 x 16 grid holds the 8 x 8 block of S_KK + ridge I at rows 8 bi..,
// columns 8 bj.. in registers (blocks on or below the diagonal; the others
// idle in the factorisation).  Blocked right-looking Cholesky, 8 columns per
// step: 16 steps of two barriers each.  The factor goes to shared memory for
// the two triangular solves, which one warp runs with the vector in
// registers.
constexpr int kLlaSolveThreads = 256;
constexpr int kLlaLd = kLlaD + 1;   // padded row stride of the factor in shared memory

__global__ void __launch_bounds__(kLlaSolveThreads) lla_solve_kernel(const LlaArgs a) {
  extern __shared__ float smf[];
  float* Lm = smf;                         // [128][129]: column k of the factor, rows >= k
  float* kb = Lm + kLlaD * kLlaLd;         // kbar
  float* vb = kb + kLlaD;                  // vbar
  float* rho_s = vb + kLlaD;               // rho*
  float* invp = rho_s + kLlaD;             // 1 / L[k][k]
  float* part = invp + kLlaD;              // [8][128] partial matrix-vector products
  float* wts = part + 8 * kLlaD;           // [kLlaMaxPieces] piece weights 2^(m_j - M)
  float* misc = wts + kLlaMaxPieces;       // [0] l, [1] kbar . rho*

  const int tid = threadIdx.x;
  const int bh = blockIdx.x, b = bh / a.Hq;
  const size_t orow = (size_t)bh * kLlaD;
  const int len = lla_seq_len(a, b);
  auto store_out = [&](int i, float v) {
    if (a.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(a.out)[orow + i] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(a.out)[orow + i] = v;
  };
  if (len == 0) {   // no keys: out = 0, rho* = 0
    if (tid < kLlaD) {
      store_out(tid, 0.f);
      if (a.rho) a.rho[orow + tid] = 0.f;
    }
    return;
  }
  const float* rec0 = a.rec + (size_t)bh * a.pieces * kLlaRecFloats;
  if (tid == 0) {
    float M = -INFINITY;
    for (int p = 0; p < a.pieces; ++p) {
      const float* r = rec0 + (size_t)p * kLlaRecFloats;
      if (r[kLlaRecM + 1] > 0.f) M = fmaxf(M, r[kLlaRecM]);
    }
    float L = 0.f;
    for (int p = 0; p < a.pieces; ++p) {
      const float* r = rec0 + (size_t)p * kLlaRecFloats;
      const float w = r[kLlaRecM + 1] > 0.f ? ex2(r[kLlaRecM] - M) : 0.f;
      wts[p] = w;
      L += w * r[kLlaRecM + 1];
    }
    misc[0] = L;
  }
  __syncthreads();
  const float invL = 1.f / misc[0];
  if (tid < kLlaD) {
    float ks = 0.f, vs = 0.f;
    for (int p = 0; p < a.pieces; ++p) {
      if (wts[p] == 0.f) continue;
      const float* r = rec0 + (size_t)p * kLlaRecFloats;
      ks = fmaf(wts[p], r[kLlaRecKs + tid], ks);
      vs = fmaf(wts[p], r[kLlaRecVs + tid], vs);
    }
    kb[tid] = ks * invL;
    vb[tid] = vs * invL;
  }
  __syncthreads();

  // ---- this thread's block of S_KK + ridge I = D_KK / l - kbar kbar^T + ridge I
  const int bi = tid >> 4, bj = tid & 15, r0 = 8 * bi, c0 = 8 * bj;
  const bool active = bi >= bj;
  float blk[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) blk[r][c] = 0.f;
  if (active) {
    for (int p = 0; p < a.pieces; ++p) {
      if (wts[p] == 0.f) continue;
      // column c0 + c of the block: rows r0 .. r0 + 7 are contiguous
      const float* d = rec0 + (size_t)p * kLlaRecFloats + kLlaRecKK + c0 * kLlaD + r0;
      float4 v[8][2];
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // all 16 loads in flight before any use
        v[c][0] = *reinterpret_cast<const float4*>(d + c * kLlaD);
        v[c][1] = *reinterpret_cast<const float4*>(d + c * kLlaD + 4);
      }
      const float w = wts[p];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        blk[0][c] = fmaf(w, v[c][0].x, blk[0][c]);
        blk[1][c] = fmaf(w, v[c][0].y, blk[1][c]);
        blk[2][c] = fmaf(w, v[c][0].z, blk[2][c]);
        blk[3][c] = fmaf(w, v[c][0].w, blk[3][c]);
        blk[4][c] = fmaf(w, v[c][1].x, blk[4][c]);
        blk[5][c] = fmaf(w, v[c][1].y, blk[5][c]);
        blk[6][c] = fmaf(w, v[c][1].z, blk[6][c]);
        blk[7][c] = fmaf(w, v[c][1].w, blk[7][c]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        blk[r][c] = fmaf(blk[r][c], invL, -kb[r0 + r] * kb[c0 + c]) + (r0 + r == c0 + c ? a.ridge : 0.f);
  }

  // ---- blocked Cholesky, one panel of 8 columns per step P: the diagonal
  // block's owner factors it in registers; the blocks below it solve
  // against that factor (X L_PP^T = A); the blocks right of the panel and
  // on or below the diagonal take the rank-8 update.  Lm ends up holding L.
  int* flag_s = reinterpret_cast<int*>(misc + 2);
  if (tid == 0) *flag_s = 0;
  bool bad = false;
#pragma unroll 1
  for (int P = 0; P < 16; ++P) {
    if (bi == P && bj == P) {   // the diagonal block: L_PP L_PP^T = A_PP
      bool ok = true;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float akk = blk[k][k];
        ok = ok && akk > 0.f && isfinite(akk);
        const float invd = rsqrtf(akk);
        blk[k][k] = akk * invd;
        invp[8 * P + k] = invd;
#pragma unroll
        for (int i = k + 1; i < 8; ++i) blk[i][k] *= invd;
#pragma unroll
        for (int i = k + 1; i < 8; ++i)
#pragma unroll
          for (int jj = k + 1; jj <= i; ++jj) blk[i][jj] = fmaf(-blk[i][k], blk[jj][k], blk[i][jj]);
      }
      if (!ok) *flag_s = 1;
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c <= r; ++c) Lm[(r0 + r) * kLlaLd + c0 + c] = blk[r][c];
    }
    __syncthreads();
    if (*flag_s != 0) {   // not numerically positive definite (uniform)
      bad = true;
      break;
    }
    if (bj == P && bi > P) {   // the panel: X L_PP^T = A, column by column
      const float* lpp = Lm + (8 * P) * kLlaLd + 8 * P;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float invd = invp[8 * P + c];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          float x = blk[r][c];
#pragma unroll
          for (int m = 0; m < c; ++m) x = fmaf(-blk[r][m], lpp[c * kLlaLd + m], x);
          blk[r][c] = x * invd;
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) Lm[(r0 + r) * kLlaLd + c0 + c] = blk[r][c];
    }
    __syncthreads();
    if (active && bj > P) {   // rank-8 update of the trailing blocks
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        float li[8], lj[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) li[r] = Lm[(r0 + r) * kLlaLd + 8 * P + m];
#pragma unroll
        for (int c = 0; c < 8; ++c) lj[c] = Lm[(c0 + c) * kLlaLd + 8 * P + m];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) blk[r][c] = fmaf(-li[r], lj[c], blk[r][c]);
      }
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) report_error(PLX_DEVERR_SINGULAR_BIT);
    if (tid < kLlaD) {   // rho* = 0: the output falls back to vbar
      store_out(tid, vb[tid]);
      if (a.rho) a.rho[orow + tid] = 0.f;
    }
    return;
  }
  // ---- L z = kbar - q, then L^T rho = z: one warp, rows lane + 32u in registers
  if (tid < 32) {
    const int lane = tid;
    float yv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) yv[u] = kb[lane + 32 * u] - __bfloat162float(a.q[orow + lane + 32 * u]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll 1
      for (int kk = 0; kk < 32; ++kk) {
        const int k = 32 * u + kk;
        const float zk = __shfl_sync(0xffffffffu, yv[u], kk) * invp[k];
        if (lane == kk) yv[u] = zk;
#pragma unroll
        for (int v = u; v < 4; ++v) {
          const int i = lane + 32 * v;
          if (i > k) yv[v] = fmaf(-Lm[i * kLlaLd + k], zk, yv[v]);
        }
      }
    }
#pragma unroll
    for (int u = 3; u >= 0; --u) {
#pragma unroll 1
      for (int kk = 31; kk >= 0; --kk) {
        const int k = 32 * u + kk;
        const float xk = __shfl_sync(0xffffffffu, yv[u], kk) * invp[k];
        if (lane == kk) yv[u] = xk;
#pragma unroll
        for (int v = 0; v <= u; ++v) {
          const int jj = lane + 32 * v;
          if (jj < k) yv[v] = fmaf(-Lm[k * kLlaLd + jj], xk, yv[v]);
        }
      }
    }
    float kr = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      rho_s[lane + 32 * u] = yv[u];
      kr = fmaf(kb[lane + 32 * u], yv[u], kr);
    }
    kr = warp_sum(kr);
    if (lane == 0) misc[1] = kr;
  }
  __syncthreads();
  // ---- out = vbar (1 + kbar . rho*) - (1 / l) sum_a D_KV[a, :] rho*_a
  {
    const int col = tid >> 1, half = tid & 1;   // rows a = 64 half .. 64 half + 63 of column col
    float acc = 0.f;
    for (int p = 0; p < a.pieces; ++p) {
      if (wts[p] == 0.f) continue;
      const float* dkv = rec0 + (size_t)p * kLlaRecFloats + kLlaRecKV + col * kLlaD + 64 * half;
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = *reinterpret_cast<const float4*>(dkv + 4 * u);
      float sp = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float* rr = rho_s + 64 * half + 4 * u;
        sp = fmaf(v[u].x, rr[0], fmaf(v[u].y, rr[1], fmaf(v[u].z, rr[2], fmaf(v[u].w, rr[3], sp))));
      }
      acc = fmaf(wts[p], sp, acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) part[col] = acc;
  }
  __syncthreads();
  if (tid < kLlaD) {
    const float corr = part[tid];
    store_out(tid, fmaf(vb[tid], 1.f + misc[1], -corr * invL));
    if (a.rho) a.rho[orow + tid] = rho_s[tid];
  }
}

constexpr int lla_solve_smem_bytes() {
  return (kLlaD * kLlaLd + 4 * kLlaD + 8 * kLlaD + kLlaMaxPieces + 4) * 4;
}

}  // namespace plx
