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
// One or two kernels per call:
//
//   lla_moments_kernel  one CTA per (sequence, query head, piece of its keys):
//     a single pass over the piece's K and V tiles accumulates, relative to
//     a running max m (2^(s - m) weights, rescaled lazily as in the prefill),
//         l = sum e,  ks = sum e k,  vs = sum e v,
//         D_KK = sum e k k^T,  D_KV = sum e k v^T          (128 x 128 each)
//     Per 64-key tile: the scores S = K q on the tensor cores (M = 64 keys,
//     N = 8: q is row 0 of an 8-row operand), read back by four warps, 16
//     keys each (the score warps), with the weights e, rounded to bf16 once
//     so that every sum uses the same values; then eight scale warps scale
//     the K tile's rows by e into A = (e o K)^T in shared memory (as an
//     MN-major operand A has the K tile's own layout, so this is a row
//     scaling, not a transpose) and sum ks and vs from the same rows on the
//     CUDA cores, while the score warps take the next tile; and the tensor
//     cores add [D_KK | D_KV] += A . [K | V] (N = 256: a stage's K and V
//     tiles are one MN-major B operand).  The issuing warp spends tens of
//     cycles per MMA, so the count matters as much as the size: twelve per
//     tile.  For sequences shorter than kLlaSplitLen the bf16 rounding of
//     e o K is not averaged away (the solve amplifies it along directions
//     the few keys do not span), so a second product adds its lo part
//     (x = hi + lo).  The piece's record goes to the workspace; with one
//     piece per head the kernel instead solves in place (below), D_KK and
//     D_KV never leaving tensor memory, and the second kernel is not run.
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
constexpr int kLlaStages = 5;            // K and V ring depth (tiles)
constexpr int kLlaThreads = 448;         // TMA producer warp, MMA warp, four score warps, eight scale warps
constexpr int kLlaScore = 128;           // score warps 2..5 (one per TMEM lane quarter)
constexpr int kLlaScale = 256;           // scale warps 6..13 (two per TMEM lane quarter)
constexpr int kLlaSplitLen = 1024;       // shorter sequences add the lo part of e o K
constexpr float kLlaRescaleLog2 = 8.f;   // lazy rescale threshold (factor 256)
constexpr int kLlaMaxPieces = 16;      // at most 32: the solve merges one piece per lane
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
  int fused;                       // 1 (one piece per head): the moments kernel solves in place
  unsigned long long wait_ns;      // limit of one pipeline wait
};

struct LlaLayout {
  static constexpr int kTileBytes = kTile * kLlaD * 2;   // 16 KB: two 64-column boxes of 64 rows
  // Stage s: the K tile, then the V tile, so that the four 64-column boxes
  // [K lo | K hi | V lo | V hi] are one MN-major operand of 256 columns.
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kKV = 0;
  // A = (e o K)^T as an MN-major operand: the K tile's layout with row i
  // scaled by e_i, in bf16.  Two buffers: hi of tile t in buffer t % 2; below
  // kLlaSplitLen keys hi in buffer 0 and lo = x - hi in buffer 1.
  static constexpr int kA = kKV + kLlaStages * kStageBytes;
  // The score product's B operand, bf16 [16][64], K-major, 128-byte swizzle:
  // row 0 = q[0:64], row 8 = q[64:128], the rest zero.
  static constexpr int kQBytes = 16 * 64 * 2;
  static constexpr int kQ = kA + 2 * kTileBytes;
  static constexpr int kE = kQ + kQBytes;                     // float [2][64]: the tile's weights e
  // float [32]: [0, 4) the score warps' maxima, [4, 8) their sums of e,
  // [8, 10) the rescale factor of the tile in e buffer 0 / 1
  static constexpr int kRed = kE + 2 * kTile * 4;
  static constexpr int kPart = kRed + 128;                    // float [64]: the second half of each score
  static constexpr int kBar = kPart + 256;
  // full[S], empty[S], s_full[3], e_full[2], e_free[2], a_full[2], a_free[2],
  // drain (the per-tile hand-offs rotate through two or three barriers by
  // tile index)
  static constexpr int kNumBars = 2 * kLlaStages + 12;
  static constexpr int kMisc = kBar + kNumBars * 8;           // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16 + 1024;            // + alignment slack
};

// TMEM columns: D = [D_KK | D_KV] in [0, 256); the score product of tile j
// at 256 + 16 (j % 3): key r's score is lane r, column 0 (components 0..63)
// plus lane 64 + r, column 8 (components 64..127).
constexpr uint32_t kLlaColKK = 0, kLlaColKV = 128;
__device__ __forceinline__ uint32_t lla_col_s(int buf) { return 256u + 16u * buf; }

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


// Instruction descriptor of kind::f16 with both operands' majorness given
// (bf16 A and B, fp32 accumulator, shape M x N).
__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- solve
// Per (sequence, query head), four row warps, row a of the system in TMEM
// lane a: S = S_KK + ridge I (fp32) lives in tensor memory.  Blocked
// right-looking Cholesky, 8 columns per panel: every row thread reads its 8
// panel entries; the diagonal block goes through shared memory and each
// thread factors it redundantly (no further synchronisation), solves its own
// row against it and carries the forward substitution z = L^-1 (kbar - q)
// along; the trailing update S -= L_P L_P^T runs on the tensor cores, with
// each panel value split into three bf16 parts (hi + mid + lo carries the
// fp32 value) and six products (hi hi, hi mid, mid hi, hi lo, lo hi, mid
// mid) of a 128 x 128 x 16 MMA with A negated, issued by the first warp once
// a named barrier says the panel is written; the next panel's columns are
// updated by the row threads themselves (look-ahead).  The factor also goes
// to shared memory, transposed, for the blocked back substitution
// L^T rho = z, whose diagonal blocks are inverted all at once (one column
// per thread) first.  The body runs in lla_solve_kernel (one CTA per head,
// for heads cut into pieces: the records are merged and D_KV comes into
// shared memory by cp.async while the factorisation runs) or in place in
// lla_moments_kernel (one piece per head: D_KK and D_KV are already in its
// tensor memory).
constexpr int kLlaSolveThreads = 128;
constexpr int kLlaLt = kLlaD + 4;                // row stride of L^T (padding against bank conflicts)

struct LlaSolveLayout {
  static constexpr int kDkv = 0;                              // float [128][128]: D_KV of piece 0
  static constexpr int kLt = kDkv + kLlaD * kLlaD * 4;        // float [128][kLlaLt]: L^T
  static constexpr int kOpBytes = kLlaD * 128;                // bf16 [128][64], 128-byte swizzle (16 columns used)
  static constexpr int kOp = (kLt + kLlaD * kLlaLt * 4 + 1023) & ~1023;   // three parts: hi, mid, lo
  static constexpr int kD8 = kOp + 3 * kOpBytes;              // float [8][8] diagonal block + [8] its z rhs
  static constexpr int kMinv = kD8 + 72 * 4;                  // float [16][8][8]: (L_II^T)^-1
  static constexpr int kVec = kMinv + 16 * 64 * 4;            // float [7][128]: kbar, vbar, rho, r, z, part, 1/L_kk
  static constexpr int kWts = kVec + 7 * kLlaD * 4;           // float [kLlaMaxPieces]
  static constexpr int kMisc = kWts + kLlaMaxPieces * 4;      // float [8]: l, kbar.rho, bad, stop, ...
  static constexpr int kBar = (kMisc + 32 + 7) & ~7;          // upd_done, drain
  static constexpr int kTmem = kBar + 24;
  static constexpr int kBytes = kTmem + 16 + 1024;
};

// The solve inside the moments kernel (one piece per head) uses the K/V
// ring once its last products are done: no D_KV copy (it stays in tensor
// memory) and no tensor-memory allocation of its own.
struct LlaFusedSolveLayout {
  static constexpr int kLt = 0;
  static constexpr int kOpBytes = LlaSolveLayout::kOpBytes;
  static constexpr int kOp = (kLt + kLlaD * kLlaLt * 4 + 1023) & ~1023;
  static constexpr int kD8 = kOp + 3 * kOpBytes;
  static constexpr int kMinv = kD8 + 72 * 4;
  static constexpr int kVec = kMinv + 16 * 64 * 4;
  static constexpr int kWts = kVec + 7 * kLlaD * 4;
  static constexpr int kMisc = kWts + kLlaMaxPieces * 4;
  static constexpr int kBar = (kMisc + 32 + 7) & ~7;
  static constexpr int kBytes = kBar + 16;
};
static_assert(LlaFusedSolveLayout::kBytes <= kLlaStages * LlaLayout::kStageBytes, "the fused solve fits in the ring");

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_group1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// 8 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// Cholesky of the 8 x 8 block d (lower triangle used) in place, with the
// reciprocals of the diagonal; false if a pivot is not positive.
__device__ __forceinline__ bool lla_chol8(float (&d)[8][8], float (&inv)[8]) {
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float akk = d[k][k];
    ok = ok && akk > 0.f && isfinite(akk);
    const float invd = rsqrtf(akk);
    d[k][k] = akk * invd;
    inv[k] = invd;
#pragma unroll
    for (int i = k + 1; i < 8; ++i) d[i][k] *= invd;
#pragma unroll
    for (int i = k + 1; i < 8; ++i)
#pragma unroll
      for (int jj = k + 1; jj <= i; ++jj) d[i][jj] = fmaf(-d[i][k], d[jj][k], d[i][jj]);
  }
  return ok;
}

// The factorisation, the two triangular solves and the output of one
// (sequence, query head), by 128 threads in four warps: thread tid owns row
// tid of the system, in tensor memory lane tid (warp w of the four must be
// a warp whose id is w mod 4), columns 0..127 of `tmem` holding
// S_KK + ridge I on entry; kbar, vbar and l are in place.  kFused: the
// threads are four warps of the moments kernel, D_KV is in tensor memory
// columns 128..255 (row a in lane a) and the tensor memory is freed by that
// kernel; otherwise D_KV of piece 0 is in shared memory (Dkv, column-major)
// and the other pieces' in their records.  bar_row and bar_all are the
// named barriers of the 128 threads (bar_all 0 when they are the whole CTA).
template <bool kFused, class Ly>
__device__ __forceinline__ void lla_solve_body(const LlaArgs& a, uint8_t* sm, const uint32_t tmem, const int tid,
                                               const int warp, const int lane, const uint32_t bar_row,
                                               const uint32_t bar_all, const float* Dkv, const float* rec0,
                                               const float invL, const size_t orow) {
  float* Lt = reinterpret_cast<float*>(sm + Ly::kLt);     // Lt[k * kLlaLt + i] = L[i][k]
  float* d8 = reinterpret_cast<float*>(sm + Ly::kD8);     // [8][8] diagonal block, then [8] its rhs
  float* kb = reinterpret_cast<float*>(sm + Ly::kVec);    // kbar
  float* vb = kb + kLlaD;                                 // vbar
  float* rho_s = vb + kLlaD;                              // rho*
  float* rb = rho_s + kLlaD;                              // back substitution right-hand side
  float* z_s = rb + kLlaD;                                // z = L^-1 (kbar - q)
  float* part = z_s + kLlaD;                              // D_KV^T rho*
  float* inv_s = part + kLlaD;                            // 1 / L[k][k]
  float* minv = reinterpret_cast<float*>(sm + Ly::kMinv); // [I][c][r]: (L_II^T)^-1
  const float* wts = reinterpret_cast<const float*>(sm + Ly::kWts);   // piece weights 2^(m_j - M)
  float* misc = reinterpret_cast<float*>(sm + Ly::kMisc); // [0] l, [1] kbar . rho*, [2] bad pivot, [3] stop
  uint64_t* upd_done = reinterpret_cast<uint64_t*>(sm + Ly::kBar);   // the panel's update is done
  uint64_t* drain = upd_done + 1;                                    // every product has completed
  auto store_out = [&](int i, float v) {
    if (a.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(a.out)[orow + i] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(a.out)[orow + i] = v;
  };
  auto sync_all = [&] { asm volatile("bar.sync %0, %1;" ::"r"(bar_all), "n"(kLlaSolveThreads) : "memory"); };
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t kIdUpd = idesc_bf16(kLlaD, kLlaD, false) | (1u << 13);   // 128 x 128 x 16, A negated
  const int r_ = tid;   // row a of S, TMEM lane a
  float rr_a = kb[r_] - __bfloat162float(a.q[orow + r_]);   // forward right-hand side of row a
  bool fine = true;
  // x holds this row's entries in panel P's columns, fully updated.  The
  // tensor-core update of panel P leaves out panel P + 1's columns (their
  // rows are zero in its operand): those the row threads update themselves
  // in fp32 right after issuing it (look-ahead), so panel P + 1 can be
  // factored while the tensor cores update the rest.
  float x[8];
  {
    uint32_t xr[8];
    tmem_ld8(tmem + lane_off, xr);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 8; ++c) x[c] = __uint_as_float(xr[c]);
  }
#pragma unroll 1
  for (int P = 0; P < 16; ++P) {
    const int c0 = 8 * P;
    if (r_ >= c0 && r_ < c0 + 8) {
#pragma unroll
      for (int c = 0; c < 8; ++c) d8[(r_ - c0) * 8 + c] = x[c];
      d8[64 + (r_ - c0)] = rr_a;
    }
    bar_and(bar_row, kLlaSolveThreads, true);
    // every row thread factors the diagonal block and solves L_PP z_P = r_P
    float dd[8][8], inv[8], zz[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 8; ++c) dd[i][c] = d8[i * 8 + c];
    const bool ok = lla_chol8(dd, inv);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v = d8[64 + c];
#pragma unroll
      for (int m = 0; m < c; ++m) v = fmaf(-dd[c][m], zz[m], v);
      zz[c] = v * inv[c];
    }
    if (!ok) {   // not numerically positive definite (every row thread sees it)
      fine = false;
      if (r_ == 0) {
        misc[2] = 1.f;
        misc[3] = 1.f;
      }
      break;
    }
    // this row's entries of L in the panel
    float l[8];
    if (r_ >= c0 + 8) {   // below the panel's diagonal block: l L_PP^T = x
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v = x[c];
#pragma unroll
        for (int m = 0; m < c; ++m) v = fmaf(-l[m], dd[c][m], v);
        l[c] = v * inv[c];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) rr_a = fmaf(-l[c], zz[c], rr_a);
    } else if (r_ >= c0) {   // a row of the diagonal block: that row of L_PP
      const int ri = r_ - c0;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v = 0.f;
#pragma unroll
        for (int i = c; i < 8; ++i) v = i == ri ? dd[i][c] : v;
        l[c] = v;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) l[c] = 0.f;
    }
    if (r_ >= c0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) Lt[(c0 + c) * kLlaLt + r_] = l[c];
    }
    if (r_ == c0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        z_s[c0 + c] = zz[c];
        inv_s[c0 + c] = inv[c];
      }
    }
    const bool mma = P < 14;   // columns past panel P + 1 remain
    // The previous panel's products are done: their operand may be
    // rewritten, and panel P + 1's columns in tensor memory are current.
    bool w = true;
    if (P >= 1 && P <= 14) w = mbar_wait_bounded(a.wait_ns, upd_done, (P - 1) & 1);
    if (mma && w) {
      // the update's operand: rows below panel P + 1, split into bf16 hi +
      // mid + lo (16-byte chunk 0 of the row; the rest is zero)
      const bool live = r_ >= c0 + 16;
      uint32_t ph[4], pm[4], pl[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float v0 = live ? l[2 * c] : 0.f, v1 = live ? l[2 * c + 1] : 0.f;
        ph[c] = pack_bf16(v0, v1);
        const float m0 = v0 - bf16_lo_f(ph[c]), m1 = v1 - bf16_hi_f(ph[c]);
        pm[c] = pack_bf16(m0, m1);
        pl[c] = pack_bf16(m0 - bf16_lo_f(pm[c]), m1 - bf16_hi_f(pm[c]));
      }
      const int off = r_ * 128 + ((r_ & 7) << 4);   // chunk 0 of row a, swizzled
      *reinterpret_cast<uint4*>(sm + Ly::kOp + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(sm + Ly::kOp + Ly::kOpBytes + off) = make_uint4(pm[0], pm[1], pm[2], pm[3]);
      *reinterpret_cast<uint4*>(sm + Ly::kOp + 2 * Ly::kOpBytes + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (!bar_and(bar_row, kLlaSolveThreads, w)) {   // the operand and this panel's L^T are written, or a wait ran out (reported)
      fine = false;
      if (r_ == 0) misc[3] = 1.f;
      break;
    }
    if (mma && warp == 0) {
      // S -= L L^T over six products of the parts (hi hi, hi mid, mid hi, hi lo, lo hi, mid mid)
      tc_fence_after();
      const uint64_t dh = smem_desc_sw128(smem_u32(sm + Ly::kOp), 16, 1024);
      const uint64_t dm = dh + (uint64_t)(Ly::kOpBytes >> 4), dl = dh + (uint64_t)((2 * Ly::kOpBytes) >> 4);
      lla_mma4_ss(tmem, dh, dh, dh, dm, dm, dh, dh, dl, kIdUpd, 1u);
      tc_mma_ss(tmem, dl, dh, kIdUpd, 1u);
      tc_mma_ss(tmem, dm, dm, kIdUpd, 1u);
      tc_commit(upd_done);
    }
    if (P == 15) break;
    // panel P + 1's columns, then this panel's part of their update
    tc_fence_after();
    {
      uint32_t xr[8];
      tmem_ld8(tmem + lane_off + (uint32_t)(c0 + 8), xr);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 8; ++c) x[c] = __uint_as_float(xr[c]);
    }
    if (r_ >= c0 + 8) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float* lrow = Lt + c0 * kLlaLt + c0 + 8 + c;   // L[c0 + 8 + c][c0 + k] at k * kLlaLt
        float v = x[c];
#pragma unroll
        for (int k = 0; k < 8; ++k) v = fmaf(-l[k], lrow[k * kLlaLt], v);
        x[c] = v;
      }
    }
  }
  if (warp == 0) {   // every product issued completes before tensor memory is freed
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  }
  tc_fence_before();
  sync_all();
  tc_fence_after();
  if constexpr (!kFused) {
    if (warp == 0) tmem_dealloc(tmem, 128);
  }
  if (!fine) {   // (a wait that ran out has reported itself)
    if constexpr (!kFused) cp_async_wait_all();
    if (tid == 0 && misc[2] != 0.f) report_error(PLX_DEVERR_SINGULAR_BIT);
    store_out(tid, vb[tid]);   // rho* = 0: the output falls back to vbar
    if (a.rho) a.rho[orow + tid] = 0.f;
    return;
  }
  // ---- L^T rho = z.  First the inverses of the transposed diagonal blocks,
  // one column per thread: column j of (L_II^T)^-1 for I = tid / 8, j = tid % 8.
  {
    const int I = tid >> 3, j = tid & 7;
    float xx[8];
#pragma unroll
    for (int c = 7; c >= 0; --c) {
      float v = c == j ? 1.f : 0.f;
#pragma unroll
      for (int rr2 = c + 1; rr2 < 8; ++rr2) v = fmaf(-Lt[(8 * I + c) * kLlaLt + 8 * I + rr2], xx[rr2], v);
      xx[c] = v * inv_s[8 * I + c];
      minv[I * 64 + c * 8 + j] = xx[c];
    }
    rb[r_] = z_s[r_];
  }
  sync_all();
  // Then blockwise from the last block: rho_I = (L_II^T)^-1 r_I (eight
  // threads), and every row above takes L_IJ^T rho_I off its r_J.
#pragma unroll 1
  for (int I = 15; I >= 0; --I) {
    if (r_ < 8) {
      float t = 0.f;
#pragma unroll
      for (int rr2 = 0; rr2 < 8; ++rr2) t = fmaf(minv[I * 64 + r_ * 8 + rr2], rb[8 * I + rr2], t);
      rho_s[8 * I + r_] = t;
    }
    sync_all();
    if (r_ < 8 * I) {
      float t = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) t = fmaf(Lt[r_ * kLlaLt + 8 * I + c], rho_s[8 * I + c], t);
      rb[r_] -= t;
    }
    sync_all();
  }
  if (tid < 32) {
    float kr = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) kr = fmaf(kb[tid + 32 * u], rho_s[tid + 32 * u], kr);
    kr = warp_sum(kr);
    if (tid == 0) misc[1] = kr;
  }
  if constexpr (!kFused) cp_async_wait_all();
  sync_all();
  if constexpr (kFused) {
  // ---- out = vbar (1 + kbar . rho*) - (1 / l) sum_a D_KV[a, :] rho*_a with
  // D_KV in tensor memory (columns 128..255, row a in lane a): thread a
  // scales its row by rho*_a; per 32-column chunk the halving exchange
  // leaves lane j with the warp's sum of column j, and the four warps'
  // sums meet in shared memory (the inverse blocks' place, free by now).
  {
    const float ra = rho_s[tid];
    float* wsum = minv;   // [4][128]
    tc_fence_after();
#pragma unroll 1
    for (int c32 = 0; c32 < 4; ++c32) {
      uint32_t rv[32];
      tmem_ld32(tmem + lane_off + (uint32_t)(kLlaD + 32 * c32), rv);
      tmem_wait_ld();
      float acc[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) acc[k] = __uint_as_float(rv[k]) * ra;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = up ? acc[i] : acc[i + o];
          const float keep = up ? acc[i + o] : acc[i];
          acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      wsum[warp * kLlaD + 32 * c32 + lane] = acc[0];
    }
    sync_all();
    part[tid] = (wsum[tid] + wsum[kLlaD + tid]) + (wsum[2 * kLlaD + tid] + wsum[3 * kLlaD + tid]);
  }
  } else {
  // ---- out = vbar (1 + kbar . rho*) - (1 / l) sum_a D_KV[a, :] rho*_a: warp w
  // takes columns 32 w .. 32 w + 31, lane l rows 4 l .. 4 l + 3 of each (a
  // column of D_KV is 512 contiguous bytes).  Every lane forms its 32
  // partial dot products; a halving exchange across the lanes (16 + 8 + 4 +
  // 2 + 1 shuffles) then leaves lane j with the sum of column 32 w + j.
  {
    const float4 rr = *reinterpret_cast<const float4*>(rho_s + 4 * lane);
    auto dot4 = [&](const float4 v) { return fmaf(v.x, rr.x, fmaf(v.y, rr.y, fmaf(v.z, rr.z, v.w * rr.w))); };
    float acc[32];
    const float w0 = wts[0];
#pragma unroll
    for (int k = 0; k < 32; ++k)
      acc[k] = w0 == 0.f ? 0.f : w0 * dot4(*reinterpret_cast<const float4*>(Dkv + (32 * warp + k) * kLlaD + 4 * lane));
#pragma unroll 1
    for (int p = 1; p < a.pieces; ++p) {
      const float wp = wts[p];
      if (wp == 0.f) continue;
      const float* src = rec0 + (size_t)p * kLlaRecFloats + kLlaRecKV + 4 * lane;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        acc[k] = fmaf(wp, dot4(__ldg(reinterpret_cast<const float4*>(src + (32 * warp + k) * kLlaD))), acc[k]);
    }
    // step o: the lanes with bit o set keep the upper half of their columns
    // and send the lower half to lane ^ o, the others the reverse
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float send = up ? acc[i] : acc[i + o];
        const float keep = up ? acc[i + o] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    part[32 * warp + lane] = acc[0];
  }
  }
  sync_all();
  store_out(tid, fmaf(vb[tid], 1.f + misc[1], -part[tid] * invL));
  if (a.rho) a.rho[orow + tid] = rho_s[tid];
}

// The in-place solve of the moments kernel, kept out of line so that the
// moments loop keeps its own register allocation.
__device__ __noinline__ void lla_fused_solve(const LlaArgs& a, uint8_t* sm, const uint32_t tmem, const int tid,
                                             const int warp, const int lane, const float invL, const size_t orow) {
  lla_solve_body<true, LlaFusedSolveLayout>(a, sm, tmem, tid, warp, lane, 7, 8, nullptr, nullptr, invL, orow);
}

__global__ void __launch_bounds__(kLlaSolveThreads, 1) lla_solve_kernel(const LlaArgs a) {
  using Ly = LlaSolveLayout;
  extern __shared__ uint8_t smem_raw_s[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw_s) + 1023) & ~uintptr_t(1023));
  float* Dkv = reinterpret_cast<float*>(sm + Ly::kDkv);   // column-major as recorded
  float* Lt = reinterpret_cast<float*>(sm + Ly::kLt);     // D_KK is staged where L^T goes later
  float* kb = reinterpret_cast<float*>(sm + Ly::kVec);    // kbar
  float* vb = kb + kLlaD;                                 // vbar
  float* wts = reinterpret_cast<float*>(sm + Ly::kWts);   // piece weights 2^(m_j - M)
  float* misc = reinterpret_cast<float*>(sm + Ly::kMisc); // [0] l, [1] kbar . rho*, [2] bad pivot, [3] stop
  uint64_t* upd_done = reinterpret_cast<uint64_t*>(sm + Ly::kBar);   // the panel's update is done
  uint64_t* drain = upd_done + 1;                                    // every product has completed
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kTmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / a.Hq;
  const size_t orow = (size_t)bh * kLlaD;
  // Launched with a programmatic dependency on the moments grid: the records
  // are read only after it has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  float* Dkk_s = Lt;   // D_KK of piece 0, [128][128] column-major as recorded, until the panels write L^T
  {   // D_KK, then D_KV, of piece 0 into shared memory, in the background
    const float* src = rec0 + kLlaRecKK;
    for (int i = tid; i < kLlaD * kLlaD / 4; i += kLlaSolveThreads) cp_async16(Dkk_s + 4 * i, src + 4 * i);
    cp_async_commit();
    src = rec0 + kLlaRecKV;
    for (int i = tid; i < kLlaD * kLlaD / 4; i += kLlaSolveThreads) cp_async16(Dkv + 4 * i, src + 4 * i);
    cp_async_commit();
  }
  const float ks0 = rec0[kLlaRecKs + tid], vs0 = rec0[kLlaRecVs + tid];   // piece 0's sums, loaded early
  if (warp == 0) {   // lane p merges piece p (at most 32 pieces)
    const bool has = lane < a.pieces;
    const float* r = rec0 + (size_t)lane * kLlaRecFloats;
    const float lp = has ? r[kLlaRecM + 1] : 0.f;
    const float mp = lp > 0.f ? r[kLlaRecM] : -INFINITY;
    float M = mp;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = lp > 0.f ? ex2(mp - M) : 0.f;
    if (has) wts[lane] = w;
    const float L = warp_sum(w * lp);
    if (lane == 0) {
      misc[0] = L;
      misc[2] = 0.f;
      misc[3] = 0.f;
      mbar_init(upd_done, 1);
      mbar_init(drain, 1);
      fence_mbarrier_init();
    }
  }
  // The products read columns 0..15 of each operand row (its 16-byte chunks
  // 0 and 1, at swizzled places): chunk 0 is written every panel, chunk 1
  // (columns 8..15) stays zero.  Thread a clears chunk 1 of row a in each part.
#pragma unroll
  for (int part_i = 0; part_i < 3; ++part_i)
    *reinterpret_cast<uint4*>(sm + Ly::kOp + part_i * Ly::kOpBytes + tid * 128 + ((1 ^ (tid & 7)) << 4)) =
        make_uint4(0u, 0u, 0u, 0u);
  if (warp == 0) {
    tmem_alloc(tmem_base_s, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  const float invL = 1.f / misc[0];
  {
    // (an empty piece has weight 0 and is skipped, whatever its record holds)
    float ks = wts[0] == 0.f ? 0.f : wts[0] * ks0, vs = wts[0] == 0.f ? 0.f : wts[0] * vs0;
    for (int p = 1; p < a.pieces; ++p) {
      if (wts[p] == 0.f) continue;
      const float* r = rec0 + (size_t)p * kLlaRecFloats;
      ks = fmaf(wts[p], r[kLlaRecKs + tid], ks);
      vs = fmaf(wts[p], r[kLlaRecVs + tid], vs);
    }
    kb[tid] = ks * invL;
    vb[tid] = vs * invL;
  }
  cp_async_wait_group1();   // this thread's part of D_KK has landed (D_KV may still be on its way)
  __syncthreads();          // and everyone's

  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int r_ = tid;   // row a of S, TMEM lane a
  // ---- row a of S_KK + ridge I = D_KK / l - kbar kbar^T + ridge I into tensor
  // memory (D_KK is recorded column-major: entry [a][j] at j * 128 + a, so a
  // warp's 32 rows read 128 contiguous bytes per column): piece 0 from
  // shared memory, any other piece from global memory, 64 loads in flight
#pragma unroll 1
  for (int c64 = 0; c64 < 2; ++c64) {
    float sv[64];
    const float w0 = wts[0];
#pragma unroll
    for (int j = 0; j < 64; ++j) sv[j] = w0 == 0.f ? 0.f : w0 * Dkk_s[(64 * c64 + j) * kLlaD + r_];
#pragma unroll 1
    for (int p = 1; p < a.pieces; ++p) {
      const float w = wts[p];
      if (w == 0.f) continue;
      const float* col0 = rec0 + (size_t)p * kLlaRecFloats + kLlaRecKK + (size_t)(64 * c64) * kLlaD + r_;
      float v[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) v[j] = __ldg(col0 + (size_t)j * kLlaD);
#pragma unroll
      for (int j = 0; j < 64; ++j) sv[j] = fmaf(w, v[j], sv[j]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = 64 * c64 + 32 * h + j;
        v[j] = __float_as_uint(fmaf(sv[32 * h + j], invL, -kb[r_] * kb[col]) + (col == r_ ? a.ridge : 0.f));
      }
      tmem_st32(tmem + lane_off + (uint32_t)(64 * c64 + 32 * h), v);
    }
  }
  tmem_wait_st();
  lla_solve_body<false, LlaSolveLayout>(a, sm, tmem, tid, warp, lane, 1, 0, Dkv, rec0, invL, orow);
}

// ---------------------------------------------------------------- moments
__global__ void __launch_bounds__(kLlaThreads, 1)
    lla_moments_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const LlaArgs a) {
  using Ly = LlaLayout;
  constexpr int S = kLlaStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Ly::kBar);
  uint64_t* empty = full + S;
  uint64_t* s_full = empty + S;
  uint64_t* e_full = s_full + 3;
  uint64_t* e_free = e_full + 2;
  uint64_t* a_full = e_free + 2;
  uint64_t* a_free = a_full + 2;
  uint64_t* drain = a_free + 2;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::kMisc + 4);
  float* red_s = reinterpret_cast<float*>(sm + Ly::kRed);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int piece = blockIdx.x % a.pieces;
  const int bh = blockIdx.x / a.pieces;
  const int b = bh / a.Hq, h = bh % a.Hq, kvh = h / a.group;
  float* rec = a.rec + (size_t)blockIdx.x * kLlaRecFloats;
  // Launched with a programmatic dependency on the kernel before it, which
  // any input may come from: wait for it before touching global memory; let
  // the next kernel (the solve) launch as soon as every CTA is here.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int len = lla_seq_len(a, b);
  const int tiles = (len + kTile - 1) / kTile;
  const int t0 = (int)((long long)piece * tiles / a.pieces);
  const int n = (int)((long long)(piece + 1) * tiles / a.pieces) - t0;
  auto zero_out = [&] {   // the head's output and rho* when it has no usable keys
    for (int i = threadIdx.x; i < kLlaD; i += kLlaThreads) {
      if (a.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(a.out)[(size_t)bh * kLlaD + i] = __float2bfloat16_rn(0.f);
      else
        reinterpret_cast<float*>(a.out)[(size_t)bh * kLlaD + i] = 0.f;
      if (a.rho) a.rho[(size_t)bh * kLlaD + i] = 0.f;
    }
  };
  if (n == 0) {   // no keys in this piece: an empty record (no keys at all: zeros)
    if (a.fused) {
      zero_out();
    } else if (threadIdx.x == 0) {
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
      if (threadIdx.x == 0) report_error(1 /* PLX_DEVERR_BAD_PAGE */);
      if (a.fused) {
        zero_out();
      } else if (threadIdx.x == 0) {
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
      mbar_init(&e_full[i], kLlaScore);
      mbar_init(&e_free[i], kLlaScale);
      mbar_init(&a_full[i], kLlaScale);
      mbar_init(&a_free[i], 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&s_full[i], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x < Ly::kQBytes / 16) {
    // 16-byte chunk i of the q operand: rows 8 (i / 64) + (i / 8) % 8, chunk
    // i % 8; rows 0 and 8 (unswizzled) hold components 64 (i / 64) + 8 (i % 8) ..
    const int i = threadIdx.x;
    alignas(16) __nv_bfloat16 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = ((i >> 3) & 7) == 0 ? a.q[(size_t)bh * kLlaD + (i >> 6) * 64 + (i & 7) * 8 + e] : __float2bfloat16_rn(0.f);
    *reinterpret_cast<uint4*>(sm + Ly::kQ + i * 16) = *reinterpret_cast<const uint4*>(v);
  }
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
    // Per tile: the scores S = K q (M = 128: the K tile's two 64-column boxes
    // stacked, so rows r and 64 + r hold key r's two halves; N = 16: q's
    // halves in B rows 0 and 8; K-major A and B) and,
    // once the compute warps have written A = (e o K)^T, the products
    // [D_KK | D_KV] += A . [K | V] (SS, 128 x 256, A and the stage's K and V
    // tiles as MN-major operands).  Twelve MMAs per tile (sixteen below
    // kLlaSplitLen keys), four under each elect.
    constexpr uint32_t kIdS = idesc_bf16_ab(128, 16, false, false);
    constexpr uint32_t kIdD = idesc_bf16_ab(128, 2 * kLlaD, true, true);
    const uint64_t dkS = smem_desc_sw128(smem_u32(sm + Ly::kKV), 16, 1024);                  // K, K-major A
    const uint64_t dqS = smem_desc_sw128(smem_u32(sm + Ly::kQ), 16, 1024);                   // q, K-major B
    const uint64_t dkvM = smem_desc_sw128(smem_u32(sm + Ly::kKV), Ly::kTileBytes / 2, 1024);   // MN-major, 64-col atoms
    const uint64_t daM = smem_desc_sw128(smem_u32(sm + Ly::kA), Ly::kTileBytes / 2, 1024);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, bar, parity));
    };
    constexpr uint64_t kStageU = Ly::kStageBytes >> 4, kRingU = S * kStageU;   // descriptor units (16 bytes)
    uint64_t so_s = 0, so_m = 0;   // descriptor offsets of the stages of the next S and the next main
    int st_s = 0, ph_s = 0, st_m = 0;
    // main(j): 16 keys per step, 16 rows (2048 bytes) of A and of [K | V].
    auto issue_main = [&](int jm) {
      const uint64_t kv = dkvM + so_m;
      const uint64_t ah = daM + (split_lo ? 0 : (uint64_t)(((jm & 1) * Ly::kTileBytes) >> 4));
      lla_mma4_ss(tmem + kLlaColKK, ah, kv, ah + 128, kv + 128, ah + 256, kv + 256, ah + 384, kv + 384, kIdD,
                  jm > 0 ? 1u : 0u);
      if (split_lo) {
        const uint64_t al = daM + (uint64_t)(Ly::kTileBytes >> 4);
        lla_mma4_ss(tmem + kLlaColKK, al, kv, al + 128, kv + 128, al + 256, kv + 256, al + 384, kv + 384, kIdD, 1u);
      }
      tc_commit(&a_free[jm & 1]);
      tc_commit(&empty[st_m]);
      so_m = so_m + kStageU == kRingU ? 0 : so_m + kStageU;
      if (++st_m == S) st_m = 0;
    };
    // S(js) once tile js has landed: 16 components of each half per step,
    // 32 bytes into the 128-byte rows.
    auto issue_s = [&](int js) {
      const uint64_t ka = dkS + so_s;
      const uint32_t d = tmem + lla_col_s(js % 3);
      lla_mma4_ss(d, ka, dqS, ka + 2, dqS + 2, ka + 4, dqS + 4, ka + 6, dqS + 6, kIdS, 0u);
      tc_commit(&s_full[js % 3]);
      so_s = so_s + kStageU == kRingU ? 0 : so_s + kStageU;
      if (++st_s == S) {
        st_s = 0;
        ph_s ^= 1;
      }
    };
    // Issue order S(0), S(1), S(2), then per tile j, once A(j) is written:
    // main(j), then S(j + 3) once its tile has landed (the scores of tile j,
    // in the same TMEM buffer, have been read by then).  The scores run three
    // tiles ahead of the products.
    bool ok = true;
    for (int js = 0; ok && js < 3 && js < n; ++js) {
      if (!(ok = wait_warp(&full[st_s], ph_s))) break;
      tc_fence_after();
      issue_s(js);
    }
    for (int j = 0; ok && j < n; ++j) {   // a role that gave up leaves a wait here to run out
      // a_full(j) also means the scores of tile j were read (the score
      // warps handed tile j's weights to the scale warps after reading them)
      if (!(ok = wait_warp(&a_full[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      issue_main(j);   // first: tile j + 3 may not have landed yet
      if (j + 3 < n) {
        if (!(ok = wait_warp(&full[st_s], ph_s))) break;
        tc_fence_after();
        issue_s(j + 3);
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // Every issued MMA must complete before tensor memory is released.
    tc_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ score warps
    // Warp 2 + i reads TMEM lane quarter wq = warp % 4: quarters 0 and 1 hold
    // the first halves of the scores of keys 0..63 (column 0), quarters 2 and
    // 3 the second halves (column 8), which they pass on through shared
    // memory; the warps of quarters 0 and 1 then own one key per lane.  Per
    // tile t (buffers t % 2): the weights e, taken against
    // the running max before the warps' one barrier, which also decides (a
    // reduction) whether the running max moves: only when a score passes it
    // by kLlaRescaleLog2, or on the first tile.  On that rare path the max
    // is reduced and the weights are taken again.  The weights and the
    // tile's rescale factor go to the scale warps (e_full).
    const int c = threadIdx.x - 64;            // 0..127
    const int wq = warp & 3;
    const bool skey = wq < 2;
    const int key = 32 * (wq & 1) + lane;
    float* part_s = reinterpret_cast<float*>(sm + Ly::kPart);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    float m_ref = -INFINITY, l_acc = 0.f;
    bool fine = true;
    int t = 0;
    for (; fine && t < n; ++t) {
      const int gb = t & 1;
      // the e buffer was read by the scale warps (tile t - 2)
      const bool wf = t < 2 || mbar_wait_bounded(a.wait_ns, &e_free[gb], ((t >> 1) - 1) & 1);
      const int sb = t % 3;   // score buffer
      const bool w = __all_sync(0xffffffffu, wf && !*abort_flag && mbar_wait_bounded(a.wait_ns, &s_full[sb], (t / 3) & 1));
      const int nvalid = min(kTile, len - (t0 + t) * kTile);
      float sc = -INFINITY;
      float half = 0.f;
      if (w) {   // warp-uniform
        tc_fence_after();
        half = __uint_as_float(tmem_ld1(tmem + lane_off + lla_col_s(sb) + (skey ? 0u : 8u)));
        tmem_wait_ld();
      }
      tc_fence_before();   // S(t + 3) overwrites the buffer after a_full(t)
      if (!skey) part_s[key] = half;
      asm volatile("bar.sync 6, %0;" ::"n"(kLlaScore) : "memory");
      if (w && skey && key < nvalid) sc = (half + part_s[key]) * a.scale_log2;
      // the weights, rounded to bf16: every sum and product uses these values
      auto weight = [&]() { return key < nvalid ? __bfloat162float(__float2bfloat16_rn(ex2(sc - m_ref))) : 0.f; };
      float e = skey ? weight() : 0.f;
      if (nvalid < kTile) {
        // Rows past the end are operands of the products (their weights are
        // 0, but 0 * NaN is not): zero them in K and V.  S(t), the only
        // earlier reader of the tile, is done (s_full).
        uint8_t* st = sm + Ly::kKV + (t % S) * Ly::kStageBytes;
        for (int i = c; i < (kTile - nvalid) * 16; i += kLlaScore) {
          const int r = nvalid + (i >> 4), ci = i & 15;   // ci: box (ci >> 3), chunk (ci & 7)
          const int off = (ci >> 3) * (Ly::kTileBytes / 2) + r * 128 + (ci & 7) * 16;
          *reinterpret_cast<uint4*>(st + off) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(st + Ly::kTileBytes + off) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();   // the products read these rows
      }
      float alpha = 1.f;
      if (bar_or(1, kLlaScore, t == 0 || !w || sc > m_ref + kLlaRescaleLog2)) {   // uniform
        if (!(fine = bar_and(2, kLlaScore, w))) break;
        const float wmax = warp_max(sc);
        if (lane == 0) red_s[wq] = wmax;
        bar_and(3, kLlaScore, true);
        // (the next write of red_s[0..3] comes after the next tile's barrier)
        const float tmax = fmaxf(fmaxf(red_s[0], red_s[1]), fmaxf(red_s[2], red_s[3]));
        if (t == 0) {
          m_ref = tmax;   // the piece's first tile holds a key: tmax is finite
        } else if (tmax > m_ref + kLlaRescaleLog2) {   // uniform: every score thread saw the same maxima
          alpha = ex2(m_ref - tmax);
          m_ref = tmax;
          l_acc *= alpha;
        }
        if (skey) e = weight();
      }
      l_acc += e;
      if (skey) reinterpret_cast<float*>(sm + Ly::kE)[gb * kTile + key] = e;
      if (c == 0) red_s[8 + gb] = alpha;
      mbar_arrive(&e_full[gb]);
    }
    // the piece's l and m (combined with the scale warps' outcome below)
    const float lw = warp_sum(l_acc);
    if (lane == 0) red_s[4 + wq] = lw;
    const bool ok = fine && t == n;
    // ---- the piece's record (score side): wait for the scale warps' outcome
    const bool rec_ok = bar_and(4, kLlaScore + kLlaScale, ok);
    bar_and(5, kLlaScore + kLlaScale, true);   // the scale warps' partial sums are in place
    if (c == 0 && !a.fused) {
      if (rec_ok) {
        rec[kLlaRecM] = m_ref;
        rec[kLlaRecM + 1] = (red_s[4] + red_s[5]) + (red_s[6] + red_s[7]);
      } else {   // abandoned after a wait ran out (already reported): an empty record
        rec[kLlaRecM] = -INFINITY;
        rec[kLlaRecM + 1] = 0.f;
      }
    }
  } else {
    // ------------------------------------------------------------ scale warps
    // Per tile t, once its weights are in (e_full): the deferred rescale of D
    // (a new running max; main(t - 1) done), then A = (e o K)^T into its A
    // buffer (main(t - 2) done; main(t - 1) when lo takes the second
    // buffer), sum e k and sum e v from the same rows; a_full, e_free.
    // Thread c takes the 16-byte chunk cc = c % 16 of rows kg + 16 m
    // (kg = c / 16, m = 0..3) of the K and V tiles: components
    // 64 (cc / 8) + 8 (cc % 8) .. + 7; a warp covers two whole rows.  For D,
    // warp 6 + i takes TMEM lane quarter warp % 4 and half i / 4 (D_KK,
    // D_KV).
    const int c = threadIdx.x - 192;           // 0..255
    const int kh = (warp - 6) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;            // TMEM lane = component a of k
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int cc = c & 15, kg = c >> 4;
    // row kg + 16 m has swizzle kg % 8
    const int roff = (cc >> 3) * (Ly::kTileBytes / 2) + (((cc & 7) ^ (kg & 7)) << 4) + kg * 128;
    float ks[8], vs[8];                        // sum e k, sum e v over this thread's rows, its 8 components
#pragma unroll
    for (int i = 0; i < 8; ++i) ks[i] = vs[i] = 0.f;
    auto scale = [&](int t, auto split_tag) -> bool {
      constexpr bool kSplit = decltype(split_tag)::value;
      const int gb = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(a.wait_ns, &e_full[gb], (t >> 1) & 1))) return false;
      const float alpha = red_s[8 + gb];
      const int jb = t - (kSplit ? 1 : 2);   // the products that last read the A buffers
      bool wv = jb < 0 || mbar_wait_bounded(a.wait_ns, &a_free[jb & 1], (jb >> 1) & 1);
      if (alpha != 1.f && !kSplit)   // uniform; D needs main(t - 1) done
        wv = wv && mbar_wait_bounded(a.wait_ns, &a_free[(t - 1) & 1], ((t - 1) >> 1) & 1);
      if (!__all_sync(0xffffffffu, wv)) return false;
      tc_fence_after();
      if (alpha != 1.f) {
#pragma unroll 1
        for (int part = 4 * kh; part < 4 * kh + 4; ++part) {   // D_KK (kh 0) or D_KV (kh 1), 32 columns at a time
          uint32_t r[32];
          const uint32_t addr = tmem + lane_off + (uint32_t)(part * 32);
          tmem_ld32(addr, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(addr, r);
        }
        tmem_wait_st();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ks[i] *= alpha;
          vs[i] *= alpha;
        }
      }
      const float* et = reinterpret_cast<const float*>(sm + Ly::kE) + gb * kTile;
      const uint8_t* st = sm + Ly::kKV + (t % S) * Ly::kStageBytes;
      uint8_t* ah = sm + Ly::kA + (kSplit ? 0 : gb * Ly::kTileBytes);
      uint8_t* al = sm + Ly::kA + Ly::kTileBytes;
      uint4 kw[4], vw[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        kw[m] = *reinterpret_cast<const uint4*>(st + roff + m * 2048);
        vw[m] = *reinterpret_cast<const uint4*>(st + Ly::kTileBytes + roff + m * 2048);
      }
      float ev[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) ev[m] = et[kg + 16 * m];
      tc_fence_before();
      mbar_arrive(&e_free[gb]);   // e and alpha of this tile are read
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float e = ev[m];
        const uint32_t kx[4] = {kw[m].x, kw[m].y, kw[m].z, kw[m].w};
        const uint32_t vx[4] = {vw[m].x, vw[m].y, vw[m].z, vw[m].w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          // e k is exact in fp32 (a product of two bf16 values)
          const float p0 = e * bf16_lo_f(kx[p]), p1 = e * bf16_hi_f(kx[p]);
          ks[2 * p] += p0;
          ks[2 * p + 1] += p1;
          vs[2 * p] = fmaf(e, bf16_lo_f(vx[p]), vs[2 * p]);
          vs[2 * p + 1] = fmaf(e, bf16_hi_f(vx[p]), vs[2 * p + 1]);
          hi[p] = pack_bf16(p0, p1);
          if constexpr (kSplit) lo[p] = pack_bf16(p0 - bf16_lo_f(hi[p]), p1 - bf16_hi_f(hi[p]));
        }
        *reinterpret_cast<uint4*>(ah + roff + m * 2048) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if constexpr (kSplit) *reinterpret_cast<uint4*>(al + roff + m * 2048) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&a_full[gb]);
      return true;
    };
    bool fine = true;
    int t = 0;
    for (; fine && t < n; ++t) fine = split_lo ? scale(t, std::true_type{}) : scale(t, std::false_type{});
    // ---- the piece's record (scale side): wait for the last products, then write
    bool wl = fine && t == n && !*abort_flag && mbar_wait_bounded(a.wait_ns, &a_free[(n - 1) & 1], ((n - 1) >> 1) & 1);
    wl = bar_and(4, kLlaScore + kLlaScale, wl);
    // the first moments' partial sums meet in the A buffers, idle once the
    // last products are done: [16 row groups][128] of sum e k, then of sum e v
    float* scr = reinterpret_cast<float*>(sm + Ly::kA);
    if (wl) {
      const int d0 = 64 * (cc >> 3) + 8 * (cc & 7);
      float4* pk = reinterpret_cast<float4*>(scr + kg * kLlaD + d0);
      float4* pv = reinterpret_cast<float4*>(scr + 16 * kLlaD + kg * kLlaD + d0);
      pk[0] = make_float4(ks[0], ks[1], ks[2], ks[3]);
      pk[1] = make_float4(ks[4], ks[5], ks[6], ks[7]);
      pv[0] = make_float4(vs[0], vs[1], vs[2], vs[3]);
      pv[1] = make_float4(vs[4], vs[5], vs[6], vs[7]);
    }
    bar_and(5, kLlaScore + kLlaScale, true);
    if (a.fused) {
      // ---- the solve in place, by the scale warps 8..11 (TMEM lane
      // quarters 0..3 in order): S_KK + ridge I from D_KK in tensor memory,
      // kbar and vbar from the partial sums, then the common solve body
      if (warp >= 8 && warp < 12) {
        using FL = LlaFusedSolveLayout;
        const int sw = warp - 8, stid = sw * 32 + lane;
        uint8_t* ss = sm + Ly::kKV;   // the ring, idle once the last products are done
        float* kbf = reinterpret_cast<float*>(ss + FL::kVec);
        float* vbf = kbf + kLlaD;
        float* miscf = reinterpret_cast<float*>(ss + FL::kMisc);
        float* wtsf = reinterpret_cast<float*>(ss + FL::kWts);
        uint64_t* updf = reinterpret_cast<uint64_t*>(ss + FL::kBar);
        const size_t orow = (size_t)bh * kLlaD;
        const float lsum = (red_s[4] + red_s[5]) + (red_s[6] + red_s[7]);
        const float invL = 1.f / lsum;
        if (wl) {
          float s4k[4] = {0.f, 0.f, 0.f, 0.f}, s4v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int g = 0; g < 16; ++g) {
            s4k[g & 3] += scr[g * kLlaD + stid];
            s4v[g & 3] += scr[16 * kLlaD + g * kLlaD + stid];
          }
          kbf[stid] = ((s4k[0] + s4k[1]) + (s4k[2] + s4k[3])) * invL;
          vbf[stid] = ((s4v[0] + s4v[1]) + (s4v[2] + s4v[3])) * invL;
#pragma unroll
          for (int part_i = 0; part_i < 3; ++part_i)   // chunk 1 of each operand row stays zero
            *reinterpret_cast<uint4*>(ss + FL::kOp + part_i * FL::kOpBytes + stid * 128 + ((1 ^ (stid & 7)) << 4)) =
                make_uint4(0u, 0u, 0u, 0u);
          if (stid == 0) {
            miscf[0] = lsum;
            miscf[2] = 0.f;
            miscf[3] = 0.f;
            wtsf[0] = 1.f;
            mbar_init(updf, 1);
            mbar_init(updf + 1, 1);
            fence_mbarrier_init();
          }
        }
        asm volatile("bar.sync 8, %0;" ::"n"(kLlaSolveThreads) : "memory");
        if (wl) {
          // S = D_KK / l - kbar kbar^T + ridge I over D_KK, row a in lane a
          tc_fence_after();
          const uint32_t loff = (uint32_t)(sw * 32) << 16;
#pragma unroll 1
          for (int c32 = 0; c32 < 4; ++c32) {
            uint32_t r[32];
            tmem_ld32(tmem + loff + (uint32_t)(32 * c32), r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int col = 32 * c32 + j;
              r[j] = __float_as_uint(fmaf(__uint_as_float(r[j]), invL, -kbf[stid] * kbf[col]) +
                                     (col == stid ? a.ridge : 0.f));
            }
            tmem_st32(tmem + loff + (uint32_t)(32 * c32), r);
          }
          tmem_wait_st();
          lla_fused_solve(a, ss, tmem, stid, sw, lane, invL, orow);
        } else {   // abandoned after a wait ran out (already reported)
          if (a.out_bf16)
            reinterpret_cast<__nv_bfloat16*>(a.out)[orow + stid] = __float2bfloat16_rn(0.f);
          else
            reinterpret_cast<float*>(a.out)[orow + stid] = 0.f;
          if (a.rho) a.rho[orow + stid] = 0.f;
        }
      }
    } else if (wl) {
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
      const int comp = c & (kLlaD - 1);
      const float* src = scr + (c >= kLlaD ? 16 * kLlaD : 0) + comp;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int g = 0; g < 16; ++g) s4[g & 3] += src[g * kLlaD];
      rec[(c >= kLlaD ? kLlaRecVs : kLlaRecKs) + comp] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

constexpr int lla_solve_smem_bytes() { return LlaSolveLayout::kBytes; }

}  // namespace plx
