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
//     (x = hi + lo).  The piece's record goes to the workspace.
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
    if (c == 0) {
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

// ---------------------------------------------------------------- solve
// One CTA per (sequence, query head).  Thread (bi, bj) of a 16 x 16 grid
// holds the 8 x 8 block of S_KK + ridge I at rows 8 bi.., columns 8 bj.. in
// registers (blocks on or below the diagonal; the others idle in the
// factorisation); a 17th block row (threads 256..271) holds b = kbar - q as
// its first row, so that the factorisation of [S; b^T] leaves z = L^-1 b in
// it (the forward substitution rides along).  Blocked right-looking
// Cholesky, 8 columns per step: 16 steps of two barriers each; the factor
// goes to shared memory transposed (row k of L^T contiguous), so that the
// rank-8 updates read it as float4.  The back substitution L^T rho = z is
// blocked too: 16 steps, each a diagonal 8 x 8 solve and the blocks of one
// row of L updating the rest of the vector, with every block still in its
// thread's registers.  D_KV comes into shared memory by cp.async while the
// factorisation runs.
constexpr int kLlaSolveThreads = 288;            // 256 matrix blocks, 16 for the b row, 16 spare
constexpr int kLlaLt = kLlaD + 8 + 4;            // row stride of L^T: 136 entries (b row included) + 4 of padding

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__global__ void __launch_bounds__(kLlaSolveThreads) lla_solve_kernel(const LlaArgs a) {
  extern __shared__ float smf[];
  float* Dkv = smf;                        // [128 columns][128]: D_KV of piece 0, column-major as recorded
  float* Lt = Dkv + kLlaD * kLlaD;         // [128][kLlaLt]: Lt[k * kLlaLt + i] = L[i][k], i = 128: z
  float* kb = Lt + kLlaD * kLlaLt;         // kbar
  float* vb = kb + kLlaD;                  // vbar
  float* rho_s = vb + kLlaD;               // rho*
  float* r_s = rho_s + kLlaD;              // the back substitution's right-hand side (z, updated)
  float* inv_s = r_s + kLlaD;              // 1 / L[k][k]
  float* part = inv_s + kLlaD;             // [128] D_KV^T rho*
  float* wts = part + kLlaD;               // [kLlaMaxPieces] piece weights 2^(m_j - M)
  float* misc = wts + kLlaMaxPieces;       // [0] l, [1] kbar . rho*, [2] non-positive pivot flag

  const int tid = threadIdx.x;
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
  {   // D_KV of piece 0 into shared memory, in the background
    const float* src = rec0 + kLlaRecKV;
    for (int i = tid; i < kLlaD * kLlaD / 4; i += kLlaSolveThreads) cp_async16(Dkv + 4 * i, src + 4 * i);
    cp_async_commit();
  }
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
    misc[2] = 0.f;
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
  // (block row 16: row 0 of the block is b = kbar - q, the rest zero)
  const int bi = tid >> 4, bj = tid & 15, r0 = 8 * bi, c0 = 8 * bj;
  const bool active = bi < 16 ? bi >= bj : bi == 16;
  float blk[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) blk[r][c] = 0.f;
  if (bi < 16 && active) {
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
  } else if (active) {   // the b row
#pragma unroll
    for (int c = 0; c < 8; ++c) blk[0][c] = kb[c0 + c] - __bfloat162float(a.q[orow + c0 + c]);
  }

  // ---- blocked Cholesky, one panel of 8 columns per step P: the diagonal
  // block's owner factors it in registers; the blocks below it (the b row
  // included) solve against that factor (X L_PP^T = A); the blocks right of
  // the panel and on or below the diagonal take the rank-8 update.
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
        inv_s[8 * P + k] = invd;
#pragma unroll
        for (int i = k + 1; i < 8; ++i) blk[i][k] *= invd;
#pragma unroll
        for (int i = k + 1; i < 8; ++i)
#pragma unroll
          for (int jj = k + 1; jj <= i; ++jj) blk[i][jj] = fmaf(-blk[i][k], blk[jj][k], blk[i][jj]);
      }
      if (!ok) misc[2] = 1.f;
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int r = c; r < 8; ++r) Lt[(c0 + c) * kLlaLt + r0 + r] = blk[r][c];
    }
    __syncthreads();
    if (misc[2] != 0.f) {   // not numerically positive definite (uniform)
      bad = true;
      break;
    }
    if (active && bj == P && bi > P) {   // the panel: X L_PP^T = A, column by column
      const float* lpp = Lt + (8 * P) * kLlaLt + 8 * P;   // lpp[m * kLlaLt + c] = L_PP[c][m]
      float lp[8][8], invd[8];   // L_PP below the diagonal and 1 / L_PP[c][c], loaded before the chain
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        invd[c] = inv_s[8 * P + c];
#pragma unroll
        for (int m = 0; m < c; ++m) lp[c][m] = lpp[m * kLlaLt + c];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          float x = blk[r][c];
#pragma unroll
          for (int m = 0; m < c; ++m) x = fmaf(-blk[r][m], lp[c][m], x);
          blk[r][c] = x * invd[c];
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float4* dst = reinterpret_cast<float4*>(Lt + (c0 + c) * kLlaLt + r0);
        dst[0] = make_float4(blk[0][c], blk[1][c], blk[2][c], blk[3][c]);
        dst[1] = make_float4(blk[4][c], blk[5][c], blk[6][c], blk[7][c]);
      }
    }
    __syncthreads();
    if (active && bj > P) {   // rank-8 update of the trailing blocks
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float* lk = Lt + (8 * P + m) * kLlaLt;   // column 8 P + m of L
        const float4 i0 = *reinterpret_cast<const float4*>(lk + r0), i1 = *reinterpret_cast<const float4*>(lk + r0 + 4);
        const float4 j0 = *reinterpret_cast<const float4*>(lk + c0), j1 = *reinterpret_cast<const float4*>(lk + c0 + 4);
        const float li[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
        const float2 lj[4] = {make_float2(j0.x, j0.y), make_float2(j0.z, j0.w), make_float2(j1.x, j1.y),
                              make_float2(j1.z, j1.w)};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int h = 0; h < 4; ++h) {   // packed pairs of columns
            const float2 t = fma2(make_float2(-li[r], -li[r]), lj[h], make_float2(blk[r][2 * h], blk[r][2 * h + 1]));
            blk[r][2 * h] = t.x;
            blk[r][2 * h + 1] = t.y;
          }
      }
    }
  }
  if (bad) {
    cp_async_wait_all();
    if (tid == 0) report_error(PLX_DEVERR_SINGULAR_BIT);
    if (tid < kLlaD) {   // rho* = 0: the output falls back to vbar
      store_out(tid, vb[tid]);
      if (a.rho) a.rho[orow + tid] = 0.f;
    }
    return;
  }
  // ---- L^T rho = z, blockwise from the last block: the diagonal block's
  // owner solves L_II^T rho_I = r_I; the owners of row I of L then take
  // L_IJ^T rho_I off r_J (J < I).
  if (bi == 16 && bj < 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) r_s[c0 + c] = blk[0][c];   // z
  }
  __syncthreads();
#pragma unroll 1
  for (int I = 15; I >= 0; --I) {
    if (bi == I && bj == I) {
      float x[8];
#pragma unroll
      for (int c = 7; c >= 0; --c) {
        float v = r_s[8 * I + c];
#pragma unroll
        for (int rr = c + 1; rr < 8; ++rr) v = fmaf(-blk[rr][c], x[rr], v);
        x[c] = v * inv_s[8 * I + c];
        rho_s[8 * I + c] = x[c];
      }
    }
    __syncthreads();
    if (bi == I && bj < I) {
      float x[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) x[r] = rho_s[8 * I + r];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float t = 0.f;
#pragma unroll
        for (int r = 0; r < 8; ++r) t = fmaf(blk[r][c], x[r], t);
        r_s[c0 + c] -= t;
      }
    }
    __syncthreads();
  }
  if (tid < 32) {
    float kr = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) kr = fmaf(kb[tid + 32 * u], rho_s[tid + 32 * u], kr);
    kr = warp_sum(kr);
    if (tid == 0) misc[1] = kr;
  }
  cp_async_wait_all();
  __syncthreads();
  // ---- out = vbar (1 + kbar . rho*) - (1 / l) sum_a D_KV[a, :] rho*_a: warp w
  // takes columns 16 w .. 16 w + 15, lane l rows 4 l .. 4 l + 3 of each (a
  // column of D_KV is 512 contiguous bytes)
  if (tid < 8 * 32) {
    const int wid = tid >> 5, lane = tid & 31;
    const float4 rr = *reinterpret_cast<const float4*>(rho_s + 4 * lane);
    auto dot4 = [&](const float* p4) {
      const float4 v = *reinterpret_cast<const float4*>(p4);
      return fmaf(v.x, rr.x, fmaf(v.y, rr.y, fmaf(v.z, rr.z, v.w * rr.w)));
    };
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      const int col = 16 * wid + k;
      float acc = wts[0] == 0.f ? 0.f : wts[0] * dot4(Dkv + col * kLlaD + 4 * lane);
      for (int p = 1; p < a.pieces; ++p)
        if (wts[p] != 0.f)
          acc = fmaf(wts[p], dot4(rec0 + (size_t)p * kLlaRecFloats + kLlaRecKV + col * kLlaD + 4 * lane), acc);
      acc = warp_sum(acc);
      if (lane == 0) part[col] = acc;
    }
  }
  __syncthreads();
  if (tid < kLlaD) {
    const float corr = part[tid];
    store_out(tid, fmaf(vb[tid], 1.f + misc[1], -corr * invL));
    if (a.rho) a.rho[orow + tid] = rho_s[tid];
  }
}

constexpr int lla_solve_smem_bytes() {
  return (kLlaD * kLlaD + kLlaD * kLlaLt + 6 * kLlaD + kLlaMaxPieces + 4) * 4;
}

}  // namespace plx
