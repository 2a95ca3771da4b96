// Parallax decode kernels for sm_100a.
//
// What one query computes.  For every KV token i, with e_i = exp(scale q.k_i - m)
// and a_i = rho.k_i - a_ref, a CTA keeps the online-softmax running max m and
// the four sums of the single-pass form
//     l = sum e_i,  c = sum e_i a_i,  O1 = sum e_i v_i,  O2 = sum e_i a_i v_i,
// and the output is out = (O1/l)(1 + c/l) - O2/l.  That equals vbar - S_KV^T rho
// because the softmax weights sum to one (S_KV^T rho = O2/l - (c/l)(O1/l)), so
// the covariance branch costs no byte beyond softmax attention's K and V: the
// single pass over the KV stream that joins the softmax and covariance
// branches (wispaper.ai blog "Parallax: Breaking the Boundary Bias with
// Parameterized Local Linear Attention", section "Hardware Efficiency").
//
// a_ref = rho.k_0 (first key of the sequence).  Any per-query constant leaves
// the output unchanged (O2 and c shift by a_ref*O1 and a_ref*l, which cancel);
// this one removes a common key offset from the products before they are
// rounded and summed.
//
// Work decomposition (stream-K).  The 64-token tiles of all units (a unit is a
// (sequence, KV head) on the bf16 path, a (sequence, query head) on the fp32
// path) are laid end to end, unit after unit, and cut into gridDim.x equal
// contiguous chunks, one per persistent CTA.  A CTA streams its chunk without
// pause across unit boundaries.  A unit that lies inside one chunk is finished
// by that CTA; a unit cut by chunk boundaries leaves one partial
// (m, l, c, O1, O2) per piece, and the last CTA to finish a piece (an atomic
// counter per unit, reset by that CTA) merges the pieces like online softmax:
// with M = max_j m_j and alpha_j = 2^(m_j - M), each of l, c, O1, O2 is the
// alpha-weighted sum.  One launch does the whole decode.
#pragma once

#include "ptx.cuh"

namespace plx {

constexpr int kTile = 64;          // tokens per KV tile; equals the page size
constexpr int kMaxGroup = 8;       // query heads per KV head on the bf16 path
constexpr int kMaxBatch = 8192;    // sequences per call (prefix table in smem)

struct DecodeArgs {
  const void* q;                   // [B, Hq, D]
  const void* rho;                 // [B, Hq, D]
  const void* k;                   // cache base (contiguous) or pool base (paged)
  const void* v;
  const int32_t* page_table;       // [B, max_pages] or null
  const int32_t* seq_lens;         // [B] or null
  void* out;                       // [B, Hq, D]
  float* slots;                    // [2 * gridDim.x][heads_per_unit][2D + 4]
  int32_t* counters;               // [B * units_per_seq]
  int B, Hq, Hkv, group;
  int units_per_seq;               // Hkv (bf16 path) or Hq (fp32 path)
  int heads_per_unit;              // group (bf16 path) or 1 (fp32 path)
  int kv_len, paged, num_pages, max_pages;
  float scale_log2;                // scale * log2(e)
  int out_bf16;
  int cluster;                     // > 1: each unit is one cluster of this many CTAs (bf16 path)
  int pdl_all;                     // 1: launched with a programmatic dependency on the previous
                                   // kernel, which any input may come from: every thread waits for it
                                   // before touching global memory (bf16 path)
  int qr_early;                    // 1: q and rho are supplied by the host, not by earlier work in
                                   // the stream, and are read before that wait (bf16 path)
  unsigned long long wait_ns;      // limit of one pipeline wait (0: give up unless complete)
};

// ------------------------------------------------------------ addressing

// Physical page of logical tile `tile` of sequence b (0 if out of range, reported).
__device__ __forceinline__ int page_of(const DecodeArgs& a, int b, int tile) {
  int p = __ldg(a.page_table + (size_t)b * a.max_pages + tile);
  if (p < 0 || p >= a.num_pages) {
    report_error(1 /* PLX_DEVERR_BAD_PAGE */);
    p = 0;
  }
  return p;
}

// Row index (in units of D elements) of token t of (b, kvh) in the cache.
__device__ __forceinline__ size_t cache_row(const DecodeArgs& a, int b, int kvh, int t) {
  if (a.paged) {
    const int page = page_of(a, b, t / kTile);
    return ((size_t)page * a.Hkv + kvh) * kTile + (t % kTile);
  }
  return ((size_t)b * a.Hkv + kvh) * a.kv_len + t;
}

__device__ __forceinline__ void store_out(const DecodeArgs& a, size_t idx, float val) {
  if (a.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(val);
  else
    reinterpret_cast<float*>(a.out)[idx] = val;
}

__device__ __forceinline__ float finalize(float o1, float o2, float l, float c) {
  const float inv = 1.0f / l;
  return o1 * inv * (1.0f + c * inv) - o2 * inv;
}

// ---------------------------------------------------------- the tile space
//
// pre[b] = number of tiles of all units of sequences before b; pre[B] = T.
// lens[b] = length of sequence b (clamped to [0, kv_len], bad values reported).
struct TileSpace {
  const int* pre;
  const int* lens;
  int B, units;
  long long T, G;

  __device__ __forceinline__ int tiles_of(int b) const { return (pre[b + 1] - pre[b]) / units; }
  __device__ __forceinline__ long long start(long long c) const { return c * T / G; }
  // CTA whose chunk holds tile x.
  __device__ __forceinline__ long long owner(long long x) const { return ((x + 1) * G + T - 1) / T - 1; }
};

// Fills pre[0..B] and lens[0..B) in shared memory; all threads of the CTA
// call it.  Without seq_lens the prefix is closed-form; otherwise it is a
// block-wide scan (per-thread chunk sums, warp shuffles, warp totals).
__device__ void build_tile_space(const DecodeArgs& a, int* pre, int* lens, int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
  if (a.seq_lens == nullptr) {
    const int per_seq = ((a.kv_len + kTile - 1) / kTile) * a.units_per_seq;
    for (int b = tid; b <= a.B; b += nt) {
      pre[b] = b * per_seq;
      if (b < a.B) lens[b] = a.kv_len;
    }
    __syncthreads();
    return;
  }
  const int per = (a.B + nt - 1) / nt;
  const int b0 = min(a.B, tid * per), b1 = min(a.B, b0 + per);
  int sum = 0;
  for (int b = b0; b < b1; ++b) {
    int n = __ldg(a.seq_lens + b);
    if (n < 0 || n > a.kv_len) {
      report_error(4 /* PLX_DEVERR_BAD_LENGTH */);
      n = n < 0 ? 0 : a.kv_len;
    }
    lens[b] = n;
    sum += ((n + kTile - 1) / kTile) * a.units_per_seq;
  }
  // inclusive scan of `sum` within the warp
  int inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) scratch[wid] = inc;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < nw; ++w) {
      const int v = scratch[w];
      scratch[w] = run;
      run += v;
    }
    pre[a.B] = run;
  }
  __syncthreads();
  int run = scratch[wid] + inc - sum;   // exclusive prefix of this thread's chunk
  for (int b = b0; b < b1; ++b) {
    pre[b] = run;
    run += ((lens[b] + kTile - 1) / kTile) * a.units_per_seq;
  }
  __syncthreads();
}

// Walks the units of a chunk in order.
struct UnitCursor {
  int b, hu, local, tiles;   // sequence, unit within it, tile within the unit, tiles per unit

  __device__ __forceinline__ void seek(const TileSpace& ts, long long x) {
    int lo = 0, hi = ts.B - 1;   // last b with pre[b] <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ts.pre[mid] <= x) lo = mid; else hi = mid - 1;
    }
    b = lo;
    while (ts.pre[b + 1] <= x) ++b;   // skip empty sequences sharing the prefix
    tiles = ts.tiles_of(b);
    const int off = (int)(x - ts.pre[b]);
    hu = off / tiles;
    local = off % tiles;
  }
  __device__ __forceinline__ long long unit_begin(const TileSpace& ts) const {
    return ts.pre[b] + (long long)hu * tiles;
  }
  __device__ __forceinline__ void next_tile(const TileSpace& ts) {
    if (++local == tiles) next_unit(ts);
  }
  __device__ __forceinline__ void next_unit(const TileSpace& ts) {
    local = 0;
    if (++hu == ts.units) {
      hu = 0;
      do { ++b; } while (b < ts.B && ts.pre[b + 1] == ts.pre[b]);
      if (b < ts.B) tiles = ts.tiles_of(b);
    }
  }
};

// Merged state of one unit: for each of its heads, m, l, c and O1, O2.
template <int D>
struct CtaState {
  float m[kMaxGroup], l[kMaxGroup], c[kMaxGroup];
  float o1[kMaxGroup][D], o2[kMaxGroup][D];
};

// Writes a unit's result: the output directly when this CTA holds the whole
// unit, otherwise this piece's partial and, in the last CTA to finish a piece
// of the unit, the merge of all pieces.  Called by the `nt` threads (ids
// 0..nt-1) that synchronise through `bar`, after `st` is complete and
// synchronised.  `scratch` is shared memory of `scratch_cap` floats that no
// other code uses meanwhile.
template <int D, typename Bar>
__device__ void finish_unit(const DecodeArgs& a, const TileSpace& ts, const CtaState<D>& st, int b, int hu,
                            long long ua, long long ub, int tid, int nt, int* s_flag, float* scratch,
                            int scratch_cap, Bar bar) {
  const int nheads = a.heads_per_unit;
  const int hq0 = hu * nheads;
  const long long c = blockIdx.x;
  const long long c0 = ts.owner(ua), c1 = ts.owner(ub - 1);
  if (c0 == c1) {
    for (int i = tid; i < nheads * D; i += nt) {
      const int h = i / D, d = i % D;
      store_out(a, ((size_t)b * a.Hq + hq0 + h) * D + d, finalize(st.o1[h][d], st.o2[h][d], st.l[h], st.c[h]));
    }
    return;
  }
  constexpr int P = 2 * D + 4;
  const size_t slot_stride = (size_t)nheads * P;
  // Slot 2c holds a piece of CTA c's first unit, slot 2c + 1 of its last one.
  auto slot_of = [&](long long cc) { return 2 * cc + (ts.start(cc) >= ua ? 0 : 1); };
  float* mine = a.slots + slot_of(c) * slot_stride;
  for (int i = tid; i < nheads * (D + 1); i += nt) {
    const int h = i / (D + 1), d = i % (D + 1);
    float* part = mine + h * P;
    if (d == D) {
      part[0] = st.m[h];
      part[1] = st.l[h];
      part[2] = st.c[h];
    } else {
      part[4 + d] = st.o1[h][d];
      part[4 + D + d] = st.o2[h][d];
    }
  }
  __threadfence();
  bar();
  const int unit = b * a.units_per_seq + hu;
  if (tid == 0) {
    const int prev = atomicAdd(a.counters + unit, 1);
    const int last = (prev == (int)(c1 - c0));
    if (last) atomicExch(a.counters + unit, 0);
    *s_flag = last;
  }
  bar();
  const bool last = *s_flag != 0;
  bar();   // everyone has read the flag before it can be reused
  if (!last) return;
  __threadfence();
  // The pieces' maxima go to shared memory in one round of parallel loads;
  // the sums are then read four pieces at a time, so the merge costs a few
  // L2 round trips instead of one per piece.
  const int np = (int)(c1 - c0 + 1);
  const bool staged = np * nheads <= scratch_cap;
  if (staged) {
    for (int i = tid; i < np * nheads; i += nt)
      scratch[i] = __ldcg(a.slots + slot_of(c0 + i / nheads) * slot_stride + (i % nheads) * P);
    bar();
  }
  for (int i = tid; i < nheads * D; i += nt) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
    for (int q = 0; q < np; ++q)
      M = fmaxf(M, staged ? scratch[q * nheads + h] : __ldcg(a.slots + slot_of(c0 + q) * slot_stride + h * P));
    float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
#pragma unroll 4
    for (int q = 0; q < np; ++q) {
      const float* ps = a.slots + slot_of(c0 + q) * slot_stride + h * P;
      const float mq = staged ? scratch[q * nheads + h] : __ldcg(ps);
      const float al = ex2(mq - M);
      L += al * __ldcg(ps + 1);
      C += al * __ldcg(ps + 2);
      O1 += al * __ldcg(ps + 4 + d);
      O2 += al * __ldcg(ps + 4 + D + d);
    }
    store_out(a, ((size_t)b * a.Hq + hq0 + h) * D + d, finalize(O1, O2, L, C));
  }
  if (staged) bar();   // the scratch is free again
}

// =========================================================================
// bf16 path: persistent CTAs, TMA ring, tensor cores (mma.sync m16n8k16,
// bf16 inputs, fp32 accumulate).
//
// Warp roles: NC consumer warps and one producer warp.  The producer's lane 0
// streams the chunk's K and V tiles (64 tokens x D, bf16) into a STAGES-deep
// ring with 2D TMA loads (128-byte swizzle, 64-column boxes), straight across
// unit boundaries.  Consumer warp w takes tokens 16 w .. 16 w + 15 of every
// tile; each warp keeps its own running state per unit, and at the end of a
// unit the consumer warps merge their states and finish the unit while the
// producer keeps loading.
//
// Per tile a consumer computes, on tensor cores, over its 16 tokens
//     [S; A] (16 x 16) = [Q; R] (16 x D) . K^T (D x 16)
// where rows 0..g-1 of the 16-row operand are the group's queries and rows
// 8..8+g-1 their probes (other rows zero).  The m16n8 accumulator layout then
// gives each thread the score s and the probe value a of the same head (rows
// h and h + 8) for the same two tokens.  It forms e and e*a in registers and
// packs them as the A operand [P; P*A] of the second product
//     [O1; O2] (16 x D) += [P; P*A] (16 x 16) . V (16 x D)
// so both accumulators come from one pass over each V tile.
// =========================================================================
template <int D>
struct TcSmem {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = kTile * 128;              // 64 rows x 128 B
  static constexpr int kTileBytes = kBoxes * kBoxBytes;      // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kWarpStateFloats = 16 * D + 24;       // m[8] l[8] c[8] O[16][D]
};

// Cluster merge: the other CTAs of a unit's cluster deposit their state in
// rank 0's receive area (at most kMaxClusterRecv states).
constexpr int kMaxClusterRecv = 2;

template <int D, int STAGES, int NC>
constexpr int tc_smem_fixed_bytes() {
  // ring + per-warp states + merged state + cluster receive area + barriers +
  // flags + scan scratch + 1 KB alignment slack (the prefix table, (2B + 1)
  // ints, comes on top)
  return STAGES * TcSmem<D>::kStageBytes + NC * TcSmem<D>::kWarpStateFloats * 4 +
         (1 + kMaxClusterRecv) * (int)sizeof(CtaState<D>) + 2 * STAGES * 8 + 16 + (NC + 1) * 32 * 4 + 1024;
}

// 16-byte store to distributed shared memory (a shared::cluster address).
__device__ __forceinline__ void dsmem_st_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}

template <int D, int STAGES, int NC, bool kLoInPad>
__global__ void __launch_bounds__((NC + 1) * 32, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const DecodeArgs a) {
  using SM = TcSmem<D>;
  // Tile t sits in stage t % STAGES and every consumer warp reads 16 of its
  // 64 tokens; the stage is refilled once all NC warps have released it, so
  // no warp can run a whole ring ahead of another and the parity wait on
  // full[t % STAGES] is exact.
  static_assert(kTile == 16 * NC, "each consumer warp takes 16 tokens of a tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* wstate = reinterpret_cast<float*>(ring + STAGES * SM::kStageBytes);
  CtaState<D>& st = *reinterpret_cast<CtaState<D>*>(wstate + NC * SM::kWarpStateFloats);
  CtaState<D>* recv = &st + 1;                               // [kMaxClusterRecv]
  uint64_t* full = reinterpret_cast<uint64_t*>(recv + kMaxClusterRecv);
  uint64_t* empty = full + STAGES;
  int* s_flag = reinterpret_cast<int*>(empty + STAGES);    // [0]: last-piece flag, [1]: abort
  int* scan = s_flag + 4;                                  // [(NC + 1) * 32]
  int* pre = scan + (NC + 1) * 32;                          // [B + 1]
  int* lens = pre + a.B + 1;                                // [B]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.group;
  // The next kernel in the stream may start once every CTA of this grid has
  // got here; a decode launched after this one with a programmatic
  // dependency then has its launch and set-up done by the time this grid
  // ends, and waits below for this grid's results.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Set-up that reads no global memory runs before the wait.  When every
  // sequence has kv_len tokens (no seq_lens) the tile space is closed-form
  // and nothing up to the first K/V load touches global memory: the
  // producer then waits for the previous grid just before that load, the
  // consumers before reading q and rho, and the chunk bounds, the cursor and
  // the first stage's expected bytes are ready by then.  (kv_len is at least
  // 1 here, so there are no empty sequences to write.)
  const bool closed = a.seq_lens == nullptr;
  if (closed) build_tile_space(a, pre, lens, scan);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    s_flag[0] = 0;
    s_flag[1] = 0;
    fence_mbarrier_init();
  }
  if (warp == NC && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (a.pdl_all && !closed) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!closed) build_tile_space(a, pre, lens, scan);

  // Sequences of length zero have no tiles: CTA b % gridDim.x writes their zeros.
  for (int b = blockIdx.x; b < a.B; b += gridDim.x)
    if (lens[b] == 0)
      for (int i = threadIdx.x; i < a.Hq * D; i += blockDim.x) store_out(a, (size_t)b * a.Hq * D + i, 0.f);
  // At most one CTA per tile, so that every chunk is non-empty.
  const long long T = pre[a.B];
  const long long G = T < (long long)gridDim.x ? T : (long long)gridDim.x;
  if ((long long)blockIdx.x >= G) return;
  TileSpace ts{pre, lens, a.B, a.units_per_seq, T, G};
  const long long x0 = ts.start(blockIdx.x), x1 = ts.start(blockIdx.x + 1);

  __syncthreads();   // the barriers' initialisation is visible
  if (a.cluster > 1) cluster_arrive_relaxed();
  volatile int* abort_flag = s_flag + 1;
  const int nchunk = (int)(x1 - x0);

  if (warp == NC) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      UnitCursor cur;
      cur.seek(ts, x0);
      int issued = 0;
      for (int t = 0; t < nchunk; ++t) {
        const int s = t % STAGES;
        if (t >= STAGES && !mbar_wait_bounded(a.wait_ns, &empty[s], ((t / STAGES) - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int kvh = cur.hu;
        const int row = a.paged ? (int)(((size_t)page_of(a, cur.b, cur.local) * a.Hkv + kvh) * kTile)
                                : (int)(((size_t)cur.b * a.Hkv + kvh) * a.kv_len + (size_t)cur.local * kTile);
        uint8_t* kdst = ring + s * SM::kStageBytes;
        uint8_t* vdst = kdst + SM::kTileBytes;
        mbar_arrive_expect_tx(&full[s], SM::kStageBytes);
        if (t == 0 && a.pdl_all) asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
        for (int bx = 0; bx < SM::kBoxes; ++bx) {
          tma_load_2d(kdst + bx * SM::kBoxBytes, &tmap_k, bx * 64, row, &full[s], pol);
          tma_load_2d(vdst + bx * SM::kBoxBytes, &tmap_v, bx * 64, row, &full[s], pol);
        }
        ++issued;
        cur.next_tile(ts);
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for the last load issued into each stage.
        for (int s = 0; s < STAGES && s < issued; ++s) {
          const int last_t = s + ((issued - 1 - s) / STAGES) * STAGES;
          mbar_wait_drain(&full[s], (last_t / STAGES) & 1);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int tid = threadIdx.x;
    constexpr int NT = NC * 32;
    auto bar = [] { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); };
    // The group's q and rho rows of a unit into shared memory, one 16-byte
    // load per 16 bytes (few, wide requests also when they sit in mapped
    // host memory across PCIe); st is unused until the unit's end, and the
    // bar() there orders its next writes after the reads of these rows.
    constexpr int kQsStride = D / 2 + 4;   // words per row: rows land 4 banks apart
    static_assert(16 * kQsStride <= 2 * kMaxGroup * D, "the staging rows fit in st.o1 and st.o2");
    uint32_t* qs = reinterpret_cast<uint32_t*>(&st.o1[0][0]);   // rows 0..g-1 q, 8..8+g-1 rho
    auto stage_qr = [&](int b, int hq0) {
#pragma unroll 1
      for (int i = tid; i < 2 * g * (D / 8); i += NT) {
        const int row = i / (D / 8), v = i % (D / 8);
        const bool isr = row >= g;
        const int h = isr ? row - g : row;
        const uint4 val = __ldg(reinterpret_cast<const uint4*>(
            reinterpret_cast<const __nv_bfloat16*>(isr ? a.rho : a.q) + ((size_t)b * a.Hq + hq0 + h) * D + 8 * v));
        *reinterpret_cast<uint4*>(qs + (isr ? 8 + h : h) * kQsStride + 4 * v) = val;
      }
    };
    UnitCursor cur;
    cur.seek(ts, x0);
    // q and rho supplied by the host are read at once, while the previous
    // grid may still run; otherwise they may come from the grid launched just
    // before this one (the projection of a projected decode, or an earlier
    // call), so the consumers wait for it first.  The producer warp streams
    // K and V meanwhile.
    const bool early = a.qr_early != 0;
    if (early) stage_qr(cur.b, cur.hu * g);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int hr = lane >> 2;          // accumulator row (head) of this thread
    const int qc = (lane & 3) * 2;     // column pair within an 8-wide chunk
    const int rr = lane & 7, mi = lane >> 3;
    float* ws = wstate + warp * SM::kWarpStateFloats;

    long long x = x0;
    bool staged = early;   // the first unit's rows are in qs already
    while (x < x1) {
      const int b = cur.b, kvh = cur.hu, local0 = cur.local;
      const long long ua = cur.unit_begin(ts), ub = ua + cur.tiles;
      const long long seg_end = ub < x1 ? ub : x1;
      const int len = lens[b];
      const int hq0 = kvh * g;

      // [Q; R] A-operand fragments of this unit, and a_ref = rho_h . k_0.
      uint32_t qa[D / 16][4];
      {
        if (!staged) stage_qr(b, hq0);
        staged = false;
        bar();
        const bool live = hr < g;
        const uint32_t* qrow = qs + hr * kQsStride;
        const uint32_t* rrow = qs + (8 + hr) * kQsStride;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c0 = (16 * kk + qc) / 2, c1 = (16 * kk + 8 + qc) / 2;
          qa[kk][0] = live ? qrow[c0] : 0u;
          qa[kk][1] = live ? rrow[c0] : 0u;
          qa[kk][2] = live ? qrow[c1] : 0u;
          qa[kk][3] = live ? rrow[c1] : 0u;
        }
      }
      // a_ref of head hr from the rho pairs this thread already holds (the
      // quad of lanes 4 hr .. 4 hr + 3 covers all D columns) and k_0
      float aref;
      {
        const uint32_t* k0 =
            reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(a.k) + cache_row(a, b, kvh, 0) * D);
        float part = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t k_lo = __ldg(k0 + (16 * kk + qc) / 2), k_hi = __ldg(k0 + (16 * kk + 8 + qc) / 2);
          part = fmaf(bf16_lo_f(qa[kk][1]), bf16_lo_f(k_lo), part);
          part = fmaf(bf16_hi_f(qa[kk][1]), bf16_hi_f(k_lo), part);
          part = fmaf(bf16_lo_f(qa[kk][3]), bf16_lo_f(k_hi), part);
          part = fmaf(bf16_hi_f(qa[kk][3]), bf16_hi_f(k_hi), part);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        aref = part;   // 0 for rows past the group (their fragments are zero)
      }

      float o[D / 8][4];
#pragma unroll
      for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      float m_run = -INFINITY, l_part = 0.f, c_part = 0.f;

      const int i_begin = (int)(x - x0), i_end = (int)(seg_end - x0);
      // Every consumer warp takes its own 16 tokens (rows 16 w .. 16 w + 15)
      // of every tile: a tile is consumed, and its stage freed, in about a
      // quarter of the time one warp would take for all 64 tokens, and the
      // last tile of a chunk does not leave three warps idle.
      for (int t = i_begin; t < i_end; ++t) {
        const int s = t % STAGES;
        if (*abort_flag) break;
        if (!mbar_wait_bounded(a.wait_ns, &full[s], (t / STAGES) & 1)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* kt = ring + s * SM::kStageBytes;
        uint8_t* vt = kt + SM::kTileBytes;
        const int tok0 = (local0 + (t - i_begin)) * kTile;
        const int nvalid = min(kTile, len - tok0);
        const int row0 = 16 * warp;   // this warp's first token row in the tile
        if (nvalid <= row0) {         // all of this warp's tokens lie past the end
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
          continue;
        }
        if (nvalid < row0 + 16) {
          // Zero this warp's V rows past the sequence end: their weight is 0,
          // but 0 * NaN is not.
          for (int i = lane; i < (row0 + 16 - nvalid) * SM::kBoxes * 8; i += 32) {
            const int row = nvalid + i / (SM::kBoxes * 8);
            const int rest = i % (SM::kBoxes * 8);
            *reinterpret_cast<uint4*>(vt + (rest / 8) * SM::kBoxBytes + row * 128 + (rest % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        // ---- [S; A] = [Q; R] K^T over this warp's two 8-token blocks
        float sc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
        const uint32_t kb = smem_u32(kt) + (uint32_t)row0 * 128u;
#pragma unroll
        for (int k2 = 0; k2 < D / 32; ++k2) {
          const uint32_t off = (k2 >> 1) * SM::kBoxBytes + rr * 128 + ((((k2 & 1) * 4 + mi) ^ rr) << 4);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + off + j * 1024, b0, b1, b2, b3);
            mma_bf16_16816(sc[j], qa[2 * k2], b0, b1);
            mma_bf16_16816(sc[j], qa[2 * k2 + 1], b2, b3);
          }
        }
        // ---- online softmax on this thread's row; mask tokens past the end
        float mloc = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool ok = row0 + 8 * j + qc + e < nvalid;
            sc[j][e] = ok ? sc[j][e] * a.scale_log2 : -INFINITY;
            sc[j][2 + e] = ok ? sc[j][2 + e] - aref : 0.f;
            mloc = fmaxf(mloc, sc[j][e]);
          }
        }
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
        const float m_new = fmaxf(m_run, mloc);   // finite: the warp has a valid token here
        const float alpha = ex2(m_run - m_new);
        m_run = m_new;
        l_part *= alpha;
        c_part *= alpha;
        // P and P*A enter the value product as bf16 hi + lo pairs (x = hi + lo
        // with lo = x - bf16(x)), so the rounding of the weights stays near
        // fp32 level instead of 2^-9 relative: |a| is often ~10 for unit-scale
        // probes, and a 2^-9 error on e*a would not average out for short
        // sequences.  With g <= 4 the lo pairs ride in the zero-padding rows
        // 4..7 / 12..15 (handed over from lane - 16), so they cost no extra
        // MMA; otherwise a second MMA consumes them.
        uint32_t pf[4], pl[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float p0 = ex2(sc[j][0] - m_new), p1 = ex2(sc[j][1] - m_new);
          const float pa0 = p0 * sc[j][2], pa1 = p1 * sc[j][3];
          l_part += p0 + p1;
          c_part += pa0 + pa1;
          const uint32_t hp = pack_bf16(p0, p1), ha = pack_bf16(pa0, pa1);
          pf[2 * j + 0] = hp;
          pf[2 * j + 1] = ha;
          pl[2 * j + 0] = pack_bf16(p0 - bf16_lo_f(hp), p1 - bf16_hi_f(hp));
          pl[2 * j + 1] = pack_bf16(pa0 - bf16_lo_f(ha), pa1 - bf16_hi_f(ha));
        }
        float alpha_o = alpha;
        if (kLoInPad) {
          const float a_from = __shfl_xor_sync(0xffffffffu, alpha, 16);
#pragma unroll
          for (int xx = 0; xx < 4; ++xx) {
            const uint32_t from = __shfl_xor_sync(0xffffffffu, pl[xx], 16);
            if (lane & 16) pf[xx] = from;
          }
          if (lane & 16) alpha_o = a_from;
        }
        if (alpha_o != 1.f) {
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= alpha_o;
            o[i][1] *= alpha_o;
            o[i][2] *= alpha_o;
            o[i][3] *= alpha_o;
          }
        }
        // ---- [O1; O2] += [P; P*A] V over this warp's 16 token rows
        const uint32_t vb = smem_u32(vt) + (uint32_t)row0 * 128u;
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {
          const int dcol = 16 * n2 + 8 * (mi >> 1);
          const uint32_t off = (dcol >> 6) * SM::kBoxBytes + (rr + 8 * (mi & 1)) * 128 +
                               ((((dcol & 63) >> 3) ^ rr) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(vb + off, b0, b1, b2, b3);
          mma_bf16_16816(o[2 * n2], pf, b0, b1);
          mma_bf16_16816(o[2 * n2 + 1], pf, b2, b3);
          if (!kLoInPad) {
            mma_bf16_16816(o[2 * n2], pl, b0, b1);
            mma_bf16_16816(o[2 * n2 + 1], pl, b2, b3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }

      // ---- end of this unit's segment: merge the warps, finish the unit
      l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
      l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
      c_part += __shfl_xor_sync(0xffffffffu, c_part, 1);
      c_part += __shfl_xor_sync(0xffffffffu, c_part, 2);
      if ((lane & 3) == 0) {
        ws[hr] = m_run;
        ws[8 + hr] = l_part;
        ws[16 + hr] = c_part;
      }
      float* wo = ws + 24;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        wo[hr * D + 8 * i + qc] = o[i][0];
        wo[hr * D + 8 * i + qc + 1] = o[i][1];
        wo[(hr + 8) * D + 8 * i + qc] = o[i][2];
        wo[(hr + 8) * D + 8 * i + qc + 1] = o[i][3];
      }
      bar();
      for (int i = tid; i < g * D; i += NT) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NC; ++w) M = fmaxf(M, wstate[w * SM::kWarpStateFloats + h]);
        float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
#pragma unroll
        for (int w = 0; w < NC; ++w) {
          const float* wsw = wstate + w * SM::kWarpStateFloats;
          const float al = ex2(wsw[h] - M);   // a warp without tiles here has m = -inf -> 0
          L += al * wsw[8 + h];
          C += al * wsw[16 + h];
          float o1 = wsw[24 + h * D + d], o2 = wsw[24 + (h + 8) * D + d];
          if (kLoInPad) {   // rows h + 4 and h + 12 hold the lo-part products
            o1 += wsw[24 + (h + 4) * D + d];
            o2 += wsw[24 + (h + 12) * D + d];
          }
          O1 += al * o1;
          O2 += al * o2;
        }
        st.o1[h][d] = O1;
        st.o2[h][d] = O2;
        if (d == 0) {
          st.m[h] = M;
          st.l[h] = L;
          st.c[h] = C;
        }
      }
      bar();
      if (a.cluster > 1) break;   // one unit per CTA; merged across the cluster below
      finish_unit<D>(a, ts, st, b, kvh, ua, ub, tid, NT, s_flag, wstate, NC * SM::kWarpStateFloats, bar);
      bar();   // per-warp states and st are free again
      x = seg_end;
      cur.next_unit(ts);
    }
  }
  __syncthreads();
  if (a.cluster > 1) {
    // The cluster's CTAs hold one piece each of the same unit (the grid is
    // unit-aligned).  Ranks >= 1 write their merged state into rank 0's
    // receive area through distributed shared memory; after the cluster
    // barrier (release / acquire) rank 0 merges and writes the output.
    const int k = a.cluster;
    const int rank = blockIdx.x % k;
    const int unit = blockIdx.x / k;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv, hq0 = kvh * g;
    cluster_wait();   // every CTA of the cluster has started
    if (rank > 0) {
      // m, l, c of every head slot, then the O1 and O2 rows of the g live
      // heads, in 16-byte stores (the states are 16-byte aligned: the ring
      // is, and every block before them is a multiple of 16 bytes)
      const uint32_t remote = dsmem_map(smem_u32(&recv[rank - 1]), 0);
      const float4* src = reinterpret_cast<const float4*>(&st);
      constexpr int kHead = 3 * kMaxGroup / 4;             // m, l, c
      constexpr int kO2 = (3 * kMaxGroup + kMaxGroup * D) / 4;
      const int live = g * D / 4;
      for (int i = threadIdx.x; i < kHead + 2 * live; i += blockDim.x) {
        const int v = i < kHead + live ? i : kO2 + (i - kHead - live);
        dsmem_st_v4(remote + 16u * v, src[v]);
      }
    }
    cluster_sync();
    if (rank == 0) {
      // eight consecutive columns per thread, written as one 16-byte store
      // (two for fp32): few, full-line writes, also into mapped host memory
      for (int i = threadIdx.x; i < g * (D / 8); i += blockDim.x) {
        const int h = i / (D / 8), d0 = 8 * (i % (D / 8));
        float M = st.m[h];
        for (int r = 0; r < k - 1; ++r) M = fmaxf(M, recv[r].m[h]);
        const float a0 = ex2(st.m[h] - M);
        float al[kMaxClusterRecv];
        float L = a0 * st.l[h], C = a0 * st.c[h];
#pragma unroll
        for (int r = 0; r < kMaxClusterRecv; ++r) {
          al[r] = r < k - 1 ? ex2(recv[r].m[h] - M) : 0.f;
          if (r < k - 1) {
            L += al[r] * recv[r].l[h];
            C += al[r] * recv[r].c[h];
          }
        }
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float O1 = a0 * st.o1[h][d0 + e], O2 = a0 * st.o2[h][d0 + e];
#pragma unroll
          for (int r = 0; r < kMaxClusterRecv; ++r)
            if (r < k - 1) {
              O1 += al[r] * recv[r].o1[h][d0 + e];
              O2 += al[r] * recv[r].o2[h][d0 + e];
            }
          v[e] = finalize(O1, O2, L, C);
        }
        const size_t idx = ((size_t)b * a.Hq + hq0 + h) * D + d0;
        if (a.out_bf16) {
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + idx) =
              make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
        } else {
          float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + idx);
          o[0] = make_float4(v[0], v[1], v[2], v[3]);
          o[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
      }
    }
  }
}

// =========================================================================
// fp32 path: CUDA-core FFMA, persistent CTAs over units (sequence, query
// head).  Warp w takes the 32-token sub-chunks w, w + NW, ... of each unit
// segment of the CTA's chunk.  Lane j computes the score and probe value of
// token j of a sub-chunk (a full dot product over D); the warp forms the
// sub-chunk max and the weights; then every lane accumulates O1 and O2 for
// its D/32 columns over the sub-chunk's tokens.
// =========================================================================
template <int NW>
constexpr int f32_smem_fixed_bytes() {
  return (16 + NW * 32) * 4;   // flags + scan scratch (the prefix table, (2B + 1) ints, comes on top)
}

template <int D, int NW>
__global__ void __launch_bounds__(NW * 32, NW >= 8 ? 1 : 2)
    decode_f32_kernel(const DecodeArgs a) {
  __shared__ CtaState<D> st;
  __shared__ float s_qr[2][D];
  __shared__ float s_w[NW][3];
  __shared__ float s_o[NW][2][D];
  extern __shared__ int smem_dyn[];
  int* s_flag = smem_dyn;               // [0]: last-piece flag
  int* scan = smem_dyn + 16;            // [NW * 32]
  int* pre = scan + NW * 32;            // [B + 1]
  int* lens = pre + a.B + 1;            // [B]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  constexpr int NT = NW * 32;
  // Launched with a programmatic dependency on the previous kernel: the
  // next grid may launch at once, and this one waits for the previous grid
  // before it touches global memory.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  build_tile_space(a, pre, lens, scan);
  for (int b = blockIdx.x; b < a.B; b += gridDim.x)
    if (lens[b] == 0)
      for (int i = tid; i < a.Hq * D; i += NT) store_out(a, (size_t)b * a.Hq * D + i, 0.f);
  const long long T = pre[a.B];
  const long long G = T < (long long)gridDim.x ? T : (long long)gridDim.x;
  if ((long long)blockIdx.x >= G) return;
  TileSpace ts{pre, lens, a.B, a.units_per_seq, T, G};
  const long long x0 = ts.start(blockIdx.x), x1 = ts.start(blockIdx.x + 1);
  auto bar = [] { __syncthreads(); };

  const float* kc = reinterpret_cast<const float*>(a.k);
  const float* vc = reinterpret_cast<const float*>(a.v);
  UnitCursor cur;
  cur.seek(ts, x0);
  long long x = x0;
  while (x < x1) {
    const int b = cur.b, hq = cur.hu, local0 = cur.local;
    const int kvh = hq / a.group;
    const long long ua = cur.unit_begin(ts), ub = ua + cur.tiles;
    const long long seg_end = ub < x1 ? ub : x1;
    const int len = lens[b];

    const float* qp = reinterpret_cast<const float*>(a.q) + ((size_t)b * a.Hq + hq) * D;
    const float* rp = reinterpret_cast<const float*>(a.rho) + ((size_t)b * a.Hq + hq) * D;
    const int tok_begin = local0 * kTile;
    const int tok_end = min((local0 + (int)(seg_end - x)) * kTile, len);

    // Every global load of a 32-token sub-chunk goes out at once, before
    // any of its arithmetic: the lane's K row (its token's score and probe
    // value) and the warp's V rows (each lane's D/32 columns of every
    // token).  The first sub-chunk's loads go out beside q, rho and the
    // first key; each later one's as soon as the previous scores and
    // products have freed the registers.
    constexpr int VB = D == 64 ? 32 : 16;   // V rows per batch of loads
    float4 kr4[D / 4];
    float vv[VB][D / 32];
    auto load_k = [&](int c0) {
      const int nvalid = min(32, tok_end - c0);
      if (lane < nvalid) {
        const float4* kr = reinterpret_cast<const float4*>(kc + cache_row(a, b, kvh, c0 + lane) * D);
#pragma unroll
        for (int d4 = 0; d4 < D / 4; ++d4) kr4[d4] = kr[d4];
      }
    };
    auto load_v = [&](int c0, int j0) {   // rows j0 .. j0 + VB - 1 (rows past the chunk read as 0)
      const int nvalid = min(32, tok_end - c0);
#pragma unroll
      for (int u = 0; u < VB; ++u) {
        const float* vr = vc + cache_row(a, b, kvh, c0 + min(j0 + u, nvalid - 1)) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) vv[u][i] = j0 + u < nvalid ? vr[lane + 32 * i] : 0.f;
      }
    };
    const int c_first = tok_begin + warp * 32;
    if (c_first < tok_end) {
      load_k(c_first);
      load_v(c_first, 0);
    }
    float k0v[D / 32];
    {
      const float* k0 = kc + cache_row(a, b, kvh, 0) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) k0v[i] = k0[lane + 32 * i];
    }
    for (int d = tid; d < D; d += NT) {
      s_qr[0][d] = qp[d];
      s_qr[1][d] = rp[d];
    }
    __syncthreads();
    float aref;
    {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) acc += s_qr[1][lane + 32 * i] * k0v[i];
      aref = warp_sum(acc);
    }

    float m_run = -INFINITY, l_lane = 0.f, c_lane = 0.f;
    float o1[D / 32], o2[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) o1[i] = o2[i] = 0.f;

    for (int c0 = c_first; c0 < tok_end; c0 += NW * 32) {
      const int nvalid = min(32, tok_end - c0);
      const int c_next = c0 + NW * 32;
      float xs = -INFINITY, av = 0.f;
      if (lane < nvalid) {
        float s = 0.f, pr = 0.f;
#pragma unroll
        for (int d4 = 0; d4 < D / 4; ++d4) {
          const float4 kv = kr4[d4];
          s += s_qr[0][4 * d4] * kv.x + s_qr[0][4 * d4 + 1] * kv.y + s_qr[0][4 * d4 + 2] * kv.z +
               s_qr[0][4 * d4 + 3] * kv.w;
          pr += s_qr[1][4 * d4] * kv.x + s_qr[1][4 * d4 + 1] * kv.y + s_qr[1][4 * d4 + 2] * kv.z +
                s_qr[1][4 * d4 + 3] * kv.w;
        }
        xs = s * a.scale_log2;
        av = pr - aref;
      }
      if (c_next < tok_end) load_k(c_next);
      const float m_new = fmaxf(m_run, warp_max(xs));
      const float alpha = ex2(m_run - m_new);
      m_run = m_new;
      const float p = ex2(xs - m_new);
      const float pa = p * av;
      l_lane = l_lane * alpha + p;
      c_lane = c_lane * alpha + pa;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        o1[i] *= alpha;
        o2[i] *= alpha;
      }
      // the products in token order (rows past nvalid hold 0 and p is 0 there)
#pragma unroll
      for (int j0 = 0; j0 < 32; j0 += VB) {
        if (j0 >= nvalid) break;   // uniform across the warp
        if (j0 > 0) load_v(c0, j0);
#pragma unroll
        for (int u = 0; u < VB; ++u) {
          if (j0 + u >= nvalid) break;   // uniform across the warp
          const float pj = __shfl_sync(0xffffffffu, p, j0 + u);
          const float paj = __shfl_sync(0xffffffffu, pa, j0 + u);
#pragma unroll
          for (int i = 0; i < D / 32; ++i) {
            o1[i] += pj * vv[u][i];
            o2[i] += paj * vv[u][i];
          }
        }
      }
      if (c_next < tok_end) load_v(c_next, 0);
    }
    const float l_w = warp_sum(l_lane), c_w = warp_sum(c_lane);
    if (lane == 0) {
      s_w[warp][0] = m_run;
      s_w[warp][1] = l_w;
      s_w[warp][2] = c_w;
    }
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      s_o[warp][0][lane + 32 * i] = o1[i];
      s_o[warp][1][lane + 32 * i] = o2[i];
    }
    __syncthreads();
    for (int d = tid; d < D; d += NT) {
      float M = -INFINITY;
      for (int w = 0; w < NW; ++w) M = fmaxf(M, s_w[w][0]);
      float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
      for (int w = 0; w < NW; ++w) {
        const float al = ex2(s_w[w][0] - M);
        L += al * s_w[w][1];
        C += al * s_w[w][2];
        O1 += al * s_o[w][0][d];
        O2 += al * s_o[w][1][d];
      }
      st.o1[0][d] = O1;
      st.o2[0][d] = O2;
      if (d == 0) {
        st.m[0] = M;
        st.l[0] = L;
        st.c[0] = C;
      }
    }
    __syncthreads();
    finish_unit<D>(a, ts, st, b, hq, ua, ub, tid, NT, s_flag, &s_o[0][0][0], NW * 2 * D, bar);
    __syncthreads();
    x = seg_end;
    cur.next_unit(ts);
  }
}

}  // namespace plx
