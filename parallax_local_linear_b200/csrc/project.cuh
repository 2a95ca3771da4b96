// Query and probe projections of the new token, ahead of a decode.
//
// Parallax learns its probe as a linear projection of the layer input
// ("Parallax: Breaking the Boundary Bias with Parameterized Local Linear
// Attention", section "The Core Insight: Covariance Correction"): for every
// sequence b and query head h,
//     q[b, h, :]   = W_Q[h*d : (h+1)*d, :] x[b, :]
//     rho[b, h, :] = W_R[h*d : (h+1)*d, :] x[b, :]
// rounded to bfloat16 (nearest, ties to even) from fp32 sums.
//
// Y = X W^T with X [B, hidden] small: the two weight matrices (2 * Hq * d
// rows of `hidden` bf16) are the only large operand and every byte of them is
// read exactly once, so the kernel is bound by HBM bandwidth on W.  A CTA
// owns 16 output features (one m16 row group of mma.sync m16n8k16, W as the
// A operand) and all batch rows (n8 tiles of X as the B operand); its eight
// warps split `hidden` into interleaved 32-column chunks and their fp32
// partials are summed in shared memory in a fixed order (deterministic).
//
// Operand loads skip shared memory: a thread reads 16 contiguous bytes of a
// W row (8 columns) straight into the registers of two mma k-steps.  That
// assigns the columns of a k-step to the fragment slots in a permuted order,
// and X is read with the same permutation, so every product still pairs
// W[n, c] with X[b, c]: the sum over c does not depend on the order.
//
// The kernel allows its dependent grid (the decode) to launch at once; the
// decode waits for this grid's completion (griddepcontrol.wait) only before
// it reads q and rho, so its prologue and first K/V loads overlap this grid.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace plx {

constexpr int kPjWarps = 8;     // k-splits per CTA
constexpr int kPjRows = 16;     // output features per CTA
constexpr int kPjMaxTiles = 8;  // n8 batch tiles per CTA (64 rows); more batch rows take grid.y

struct ProjArgs {
  const __nv_bfloat16* x;    // [B, hidden]
  const __nv_bfloat16* wq;   // [n1, hidden]
  const __nv_bfloat16* wr;   // [n1, hidden]
  __nv_bfloat16* q;          // [B, n1]  (= [B, Hq, d])
  __nv_bfloat16* rho;        // [B, n1]
  int B;
  int n1;                    // Hq * d, a multiple of kPjRows
  int hidden;                // a multiple of 32
};

// 16 bytes of a stream read once: not kept in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// BT: n8 batch tiles per CTA; U: 32-column chunks each warp has in flight.
template <int BT, int U>
__global__ void __launch_bounds__(kPjWarps * 32) project_qr_kernel(const ProjArgs a) {
  griddep_launch_dependents();
  __shared__ float red[kPjWarps][kPjRows][BT * 8];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * kPjRows;           // first output feature of W_Q rows then W_R rows
  const int b0 = blockIdx.y * BT * 8;            // first batch row
  const bool is_q = n0 < a.n1;
  const __nv_bfloat16* W = is_q ? a.wq + (size_t)n0 * a.hidden : a.wr + (size_t)(n0 - a.n1) * a.hidden;
  // Thread (g, t) reads columns 32c + 8t .. 32c + 8t + 7 of rows g and g + 8.
  const uint4* w_lo = reinterpret_cast<const uint4*>(W + (size_t)g * a.hidden) + t;
  const uint4* w_hi = reinterpret_cast<const uint4*>(W + (size_t)(g + 8) * a.hidden) + t;
  const uint4* xrow[BT];
  bool xlive[BT];
#pragma unroll
  for (int bt = 0; bt < BT; ++bt) {
    const int b = b0 + bt * 8 + g;
    xlive[bt] = b < a.B;
    xrow[bt] = reinterpret_cast<const uint4*>(a.x + (size_t)(xlive[bt] ? b : 0) * a.hidden) + t;
  }

  float acc[BT][4];
#pragma unroll
  for (int bt = 0; bt < BT; ++bt) acc[bt][0] = acc[bt][1] = acc[bt][2] = acc[bt][3] = 0.f;

  const int nch = a.hidden / 32;
  for (int c0 = warp; c0 < nch; c0 += kPjWarps * U) {
    uint4 wl[U], wh[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kPjWarps;
      if (c < nch) {
        wl[u] = ld_stream16(w_lo + 4 * c);
        wh[u] = ld_stream16(w_hi + 4 * c);
      } else {
        wl[u] = wh[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kPjWarps;
      if (c >= nch) break;   // uniform across the warp
      // k-step 0 takes columns 8t..8t+3 of the chunk, k-step 1 columns 8t+4..8t+7:
      // fragment slot (2t, 2t+1) <- the first pair, slot (2t+8, 2t+9) <- the second.
      const uint32_t a0[4] = {wl[u].x, wh[u].x, wl[u].y, wh[u].y};
      const uint32_t a1[4] = {wl[u].z, wh[u].z, wl[u].w, wh[u].w};
#pragma unroll
      for (int bt = 0; bt < BT; ++bt) {
        const uint4 xv = xlive[bt] ? __ldg(xrow[bt] + 4 * c) : make_uint4(0u, 0u, 0u, 0u);
        mma_bf16_16816(acc[bt], a0, xv.x, xv.y);
        mma_bf16_16816(acc[bt], a1, xv.z, xv.w);
      }
    }
  }

  // C fragment: acc[bt][0..1] -> feature g, batch columns 2t, 2t+1 of tile bt;
  // acc[bt][2..3] -> feature g + 8.
#pragma unroll
  for (int bt = 0; bt < BT; ++bt) {
    red[warp][g][bt * 8 + 2 * t] = acc[bt][0];
    red[warp][g][bt * 8 + 2 * t + 1] = acc[bt][1];
    red[warp][g + 8][bt * 8 + 2 * t] = acc[bt][2];
    red[warp][g + 8][bt * 8 + 2 * t + 1] = acc[bt][3];
  }
  __syncthreads();
  __nv_bfloat16* Y = is_q ? a.q : a.rho;
  const int f0 = is_q ? n0 : n0 - a.n1;
  for (int i = threadIdx.x; i < kPjRows * BT * 8; i += kPjWarps * 32) {
    const int row = i % kPjRows, col = i / kPjRows;
    const int b = b0 + col;
    if (b >= a.B) continue;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPjWarps; ++w) s += red[w][row][col];
    Y[(size_t)b * a.n1 + f0 + row] = __float2bfloat16_rn(s);
  }
}

}  // namespace plx
