// libparallax.so: the C ABI declared in include/parallax.h.
//
// Host side of every entry point: argument validation, the work plan of a
// decode call, TMA tensor maps, kernel launches.  All arithmetic of the path
// runs in the kernels included below; nothing here touches tensor data.
#include "parallax.h"

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "ptx.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "prefill2.cuh"
#include "prefill_bwd.cuh"
#include "project.cuh"
#include "lla.cuh"

namespace {

using namespace plx;

constexpr int kMaxDevices = 64;

// Decode kernel configuration (bf16 path): consumer warps and ring depth.
#ifndef PLX_DECODE_STAGES
#define PLX_DECODE_STAGES 4
#endif
constexpr int kDecodeNC = 4;
constexpr int kDecodeStages128 = PLX_DECODE_STAGES;   // 5 fit in shared memory for up to ~1100 sequences: no faster
constexpr int kDecodeStages64 = 8;
constexpr int kDecodeF32Warps = 8;

// Persistent grid of the fp32 path, in CTAs per SM: one CTA of eight warps
// (each warp holds a 32-token sub-chunk's K and V rows in registers, up to
// 255 a thread).
constexpr int kF32CtasPerSm = 1;

std::mutex g_mu;
int g_num_sms[kMaxDevices];
// Pipeline wait limit of each device's kernels (parallax_set_wait_limit_ns).
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
unsigned long long g_wait_ns[kMaxDevices];
bool g_wait_set[kMaxDevices];

unsigned long long current_wait_ns() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kDefaultWaitNs;
  std::lock_guard<std::mutex> lk(g_mu);
  return g_wait_set[dev] ? g_wait_ns[dev] : kDefaultWaitNs;
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The last CUDA error a call of this thread met (parallax_last_cuda_error).
thread_local int g_last_cuda_error = 0;

cudaError_t note(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = (int)e;
  return e;
}

template <typename Kernel>
cudaError_t set_smem(Kernel kern, int bytes) {
  return note(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Do the byte ranges [a, a + na) and [b, b + nb) share a byte?
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int current_device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

// Row-major [rows, cols] bf16 tensor, box [box_rows, box_cols], 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                    uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, heads, cols] bf16 tensor (rows of `heads` head vectors), box
// [box_rows, 1, box_cols]: box_rows rows of one head, 128-byte swizzle.
bool make_tmap_bf16_heads(CUtensorMap* m, const void* base, uint64_t cols, uint64_t heads, uint64_t rows,
                          uint32_t box_cols, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {cols, heads, rows};
  cuuint64_t strides[2] = {cols * 2, heads * cols * 2};
  cuuint32_t box[3] = {box_cols, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ decode
struct DecodePlan {
  int ctas;                  // persistent grid size
  int units_per_seq, heads_per_unit;
  size_t counter_bytes, slot_bytes;
};

plx_status validate_decode(const plx_decode_params* p) {
  if (p == nullptr) return PLX_ERR_INVALID_ARG;
  if (p->batch < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1) return PLX_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return PLX_ERR_INVALID_ARG;
  if (p->kv_len < 0 || p->num_ctas < 0) return PLX_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return PLX_ERR_INVALID_ARG;
  if (p->in_dtype != PLX_F32 && p->in_dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  if (p->out_dtype != PLX_F32 && p->out_dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return PLX_ERR_UNSUPPORTED;
  if (p->page_size != 0 && p->page_size != kTile) return PLX_ERR_UNSUPPORTED;
  if (p->in_dtype == PLX_BF16 && p->num_q_heads / p->num_kv_heads > kMaxGroup) return PLX_ERR_UNSUPPORTED;
  if (p->batch > kMaxBatch) return PLX_ERR_UNSUPPORTED;
  if (p->page_size != 0) {
    if (p->num_pages < 1) return PLX_ERR_INVALID_ARG;
    if (p->max_pages_per_seq < (p->kv_len + kTile - 1) / kTile) return PLX_ERR_INVALID_ARG;
    if ((int64_t)p->num_pages * p->num_kv_heads * kTile >= (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  } else {
    if ((int64_t)p->batch * p->num_kv_heads * ((int64_t)p->kv_len + kTile) >= (int64_t)INT32_MAX)
      return PLX_ERR_UNSUPPORTED;
  }
  // total tiles of all units must fit an int
  if ((int64_t)p->batch * p->num_q_heads * (((int64_t)p->kv_len + kTile - 1) / kTile) >= (int64_t)INT32_MAX / 2)
    return PLX_ERR_UNSUPPORTED;
  return PLX_OK;
}

DecodePlan plan_decode(const plx_decode_params* p, int num_sms) {
  DecodePlan pl{};
  const bool bf16 = p->in_dtype == PLX_BF16;
  pl.units_per_seq = bf16 ? p->num_kv_heads : p->num_q_heads;
  pl.heads_per_unit = bf16 ? p->num_q_heads / p->num_kv_heads : 1;
  const int64_t units = (int64_t)p->batch * pl.units_per_seq;
  const int64_t tiles = units * ((p->kv_len + kTile - 1) / kTile);
  int64_t ctas = p->num_ctas > 0 ? p->num_ctas : (int64_t)num_sms * (bf16 ? 1 : kF32CtasPerSm);
  if (p->num_ctas == 0 && bf16 && p->page_size == 0 && units <= num_sms) {
    // A contiguous cache usually holds equal-length sequences: cut each unit
    // into k equal pieces, one per CTA, so that no CTA crosses a unit
    // boundary, as long as that keeps most SMs busy.  Any grid is correct
    // (stream-K handles ragged lengths); paged caches keep one CTA per SM.
    const int64_t k = num_sms / units;
    if (4 * units * k >= 3 * (int64_t)num_sms) ctas = units * k;
  }
  // The fp32 kernel's warps take 32-token sub-chunks: by default a CTA gets at
  // least one per warp (four tiles), so that no warp idles on a short stream.
  const int64_t min_tiles = p->num_ctas == 0 && !bf16 ? kDecodeF32Warps * 32 / kTile : 1;
  if (ctas > (tiles + min_tiles - 1) / min_tiles) ctas = (tiles + min_tiles - 1) / min_tiles;
  if (ctas < 1) ctas = 1;
  if (ctas > INT32_MAX / 4) ctas = INT32_MAX / 4;
  pl.ctas = (int)ctas;
  pl.counter_bytes = (((size_t)p->batch * pl.units_per_seq * 4) + 255) & ~size_t(255);
  pl.slot_bytes = (size_t)2 * pl.ctas * pl.heads_per_unit * (2 * p->head_dim + 4) * 4;
  return pl;
}

size_t decode_smem_bytes(const plx_decode_params* p) {
  const size_t table = (size_t)(2 * p->batch + 1) * 4;
  if (p->in_dtype == PLX_F32) return f32_smem_fixed_bytes<kDecodeF32Warps>() + table;
  return (p->head_dim == 64 ? tc_smem_fixed_bytes<64, kDecodeStages64, kDecodeNC>()
                            : tc_smem_fixed_bytes<128, kDecodeStages128, kDecodeNC>()) +
         table;
}

// Launch with a programmatic dependency on the previous kernel in the stream
// (the kernel waits for it with griddepcontrol.wait before reading its
// inputs; its launch and its CTAs' start overlap the previous grid's tail).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
}

// How a decode grid depends on the kernel before it in the stream:
//   kPdlNone      plain stream order;
//   kPdlQR        programmatic: the previous kernel produces q and rho only
//                 (the projection), so the producer streams K and V at once
//                 and the consumers wait before reading q and rho;
//   kPdlAll       programmatic: any input may come from the previous kernel,
//                 so every thread waits before touching global memory; only
//                 the launch and the CTAs' start overlap the previous grid's
//                 tail.
enum PdlMode { kPdlNone = 0, kPdlQR = 1, kPdlAll = 2 };

template <int D, int STAGES, bool kLoInPad>
plx_status launch_decode_tc(const DecodeArgs& args, const CUtensorMap& tk, const CUtensorMap& tv, int ctas,
                            size_t smem, cudaStream_t stream, PdlMode pdl, bool set_attr) {
  auto kern = decode_tc_kernel<D, STAGES, kDecodeNC, kLoInPad>;
  if (set_attr &&
      set_smem(kern, (int)smem) != cudaSuccess)
    return PLX_ERR_CUDA;
  DecodeArgs a = args;
  a.pdl_all = pdl == kPdlAll ? 1 : 0;
  if (a.cluster <= 1 && pdl == kPdlNone) {
    kern<<<ctas, (kDecodeNC + 1) * 32, smem, stream>>>(tk, tv, a);
    return note(cudaGetLastError()) == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3((kDecodeNC + 1) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl != kPdlNone) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  const int cluster_attr = n;
  if (a.cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = a.cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (note(cudaLaunchKernelEx(&cfg, kern, tk, tv, a)) == cudaSuccess) return PLX_OK;
  (void)cudaGetLastError();
  if (a.cluster <= 1) return PLX_ERR_CUDA;
  // Clusters could not be scheduled (a launch-configuration error, which is
  // not sticky): run the same grid with the global-memory merge instead.
  DecodeArgs b = a;
  b.cluster = 1;
  cfg.numAttrs = cluster_attr;
  if (note(cudaLaunchKernelEx(&cfg, kern, tk, tv, b)) == cudaSuccess) return PLX_OK;
  (void)cudaGetLastError();
  return PLX_ERR_CUDA;
}

template <int D>
plx_status launch_decode_f32(const DecodeArgs& a, int ctas, size_t smem, cudaStream_t stream, bool set_attr) {
  auto kern = decode_f32_kernel<D, kDecodeF32Warps>;
  if (set_attr &&
      set_smem(kern, (int)smem) != cudaSuccess)
    return PLX_ERR_CUDA;
  return note(launch_pdl(kern, dim3(ctas), dim3(kDecodeF32Warps * 32), smem, stream, a)) == cudaSuccess ? PLX_OK
                                                                                                    : PLX_ERR_CUDA;
}

// A validated decode call: kernel arguments, plan and tensor maps.
struct DecodeLaunch {
  DecodeArgs a;
  DecodePlan pl;
  size_t smem;
  CUtensorMap tk, tv;   // bf16 path only
  bool empty;           // every sequence is empty: the output is zero
};

// Validates a decode call and builds its kernel arguments and tensor maps;
// launches nothing.
plx_status prepare_decode(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                          const int32_t* page_table, const int32_t* seq_lens, void* out, void* workspace,
                          size_t workspace_bytes, const plx_decode_params* p, DecodeLaunch* L) {
  plx_status st = validate_decode(p);
  if (st != PLX_OK) return st;
  if (!q || !rho || !k_cache || !v_cache || !out) return PLX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(rho, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return PLX_ERR_INVALID_ARG;
  const bool paged = p->page_size != 0;
  if (paged && (page_table == nullptr || seq_lens == nullptr)) return PLX_ERR_INVALID_ARG;
  if (!paged && page_table != nullptr) return PLX_ERR_INVALID_ARG;
  if ((page_table && !aligned(page_table, 4)) || (seq_lens && !aligned(seq_lens, 4))) return PLX_ERR_INVALID_ARG;

  const int num_sms = current_device_sms();
  if (num_sms <= 0) return PLX_ERR_CUDA;
  const DecodePlan pl = plan_decode(p, num_sms);
  const size_t need = pl.counter_bytes + pl.slot_bytes;
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return PLX_ERR_WORKSPACE;

  const int D = p->head_dim;
  L->pl = pl;
  L->empty = p->kv_len == 0;   // every sequence is empty: the output is zero
  DecodeArgs& a = L->a;
  a = DecodeArgs{};
  a.q = q;
  a.rho = rho;
  a.k = k_cache;
  a.v = v_cache;
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.out = out;
  a.counters = reinterpret_cast<int32_t*>(workspace);
  a.slots = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + pl.counter_bytes);
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.group = p->num_q_heads / p->num_kv_heads;
  a.units_per_seq = pl.units_per_seq;
  a.heads_per_unit = pl.heads_per_unit;
  a.kv_len = p->kv_len;
  a.paged = paged ? 1 : 0;
  a.num_pages = paged ? p->num_pages : 0;
  a.max_pages = paged ? p->max_pages_per_seq : 0;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.out_bf16 = p->out_dtype == PLX_BF16 ? 1 : 0;
  a.wait_ns = current_wait_ns();

  // Units of equal length cut into k pieces each (the unit-aligned grid) are
  // merged through distributed shared memory when each unit is one cluster.
  a.cluster = 1;
  if (p->in_dtype == PLX_BF16 && !paged && seq_lens == nullptr && p->num_ctas == 0) {
    const int64_t units = (int64_t)p->batch * p->num_kv_heads;
    const int64_t k = pl.ctas / units;
    const int64_t tiles_per_unit = (p->kv_len + kTile - 1) / kTile;
    if (k >= 2 && k <= 1 + kMaxClusterRecv && k * units == pl.ctas && tiles_per_unit >= k) a.cluster = (int)k;
  }
  L->smem = decode_smem_bytes(p);
  if (L->smem > 227 * 1024) return PLX_ERR_UNSUPPORTED;
  if (L->empty || p->in_dtype == PLX_F32) return PLX_OK;
  const uint64_t rows = paged ? (uint64_t)p->num_pages * p->num_kv_heads * kTile
                              : (uint64_t)p->batch * p->num_kv_heads * p->kv_len;
  if (!make_tmap_bf16(&L->tk, k_cache, D, rows, 64, kTile) || !make_tmap_bf16(&L->tv, v_cache, D, rows, 64, kTile))
    return PLX_ERR_CUDA;
  return PLX_OK;
}

// `set_attr`: set the kernel's dynamic shared-memory limit first (a prepared
// plan did that once when it was made).
plx_status launch_decode(const DecodeLaunch& L, const plx_decode_params* p, cudaStream_t stream, PdlMode pdl,
                         bool set_attr = true) {
  const DecodeArgs& a = L.a;
  const int D = p->head_dim;
  if (L.empty) {
    const size_t elt = p->out_dtype == PLX_BF16 ? 2 : 4;
    return cudaMemsetAsync(a.out, 0, (size_t)p->batch * p->num_q_heads * D * elt, stream) == cudaSuccess
               ? PLX_OK
               : PLX_ERR_CUDA;
  }
  if (p->in_dtype == PLX_F32)
    return D == 64 ? launch_decode_f32<64>(a, L.pl.ctas, L.smem, stream, set_attr)
                   : launch_decode_f32<128>(a, L.pl.ctas, L.smem, stream, set_attr);
  const bool pad = a.group <= kMaxGroup / 2;
  if (D == 64)
    return pad ? launch_decode_tc<64, kDecodeStages64, true>(a, L.tk, L.tv, L.pl.ctas, L.smem, stream, pdl, set_attr)
               : launch_decode_tc<64, kDecodeStages64, false>(a, L.tk, L.tv, L.pl.ctas, L.smem, stream, pdl,
                                                               set_attr);
  return pad ? launch_decode_tc<128, kDecodeStages128, true>(a, L.tk, L.tv, L.pl.ctas, L.smem, stream, pdl, set_attr)
             : launch_decode_tc<128, kDecodeStages128, false>(a, L.tk, L.tv, L.pl.ctas, L.smem, stream, pdl,
                                                              set_attr);
}

// Sets the dynamic shared-memory limit of the kernel a launch will use.
plx_status set_decode_attr(const DecodeLaunch& L, const plx_decode_params* p) {
  if (L.empty) return PLX_OK;
  const int smem = (int)L.smem;
  cudaError_t e;
  const bool pad = L.a.group <= kMaxGroup / 2;
  if (p->in_dtype == PLX_F32)
    e = p->head_dim == 64 ? set_smem(decode_f32_kernel<64, kDecodeF32Warps>, smem)
                          : set_smem(decode_f32_kernel<128, kDecodeF32Warps>, smem);
  else if (p->head_dim == 64)
    e = pad ? set_smem(decode_tc_kernel<64, kDecodeStages64, kDecodeNC, true>, smem)
            : set_smem(decode_tc_kernel<64, kDecodeStages64, kDecodeNC, false>, smem);
  else
    e = pad ? set_smem(decode_tc_kernel<128, kDecodeStages128, kDecodeNC, true>, smem)
            : set_smem(decode_tc_kernel<128, kDecodeStages128, kDecodeNC, false>, smem);
  return e == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

// q and rho projections of a projected decode (project.cuh).
plx_status launch_project(const ProjArgs& pa, cudaStream_t stream) {
  const int tiles = (pa.B + 7) / 8;
  const int bt = tiles <= 1 ? 1 : tiles <= 2 ? 2 : tiles <= 4 ? 4 : kPjMaxTiles;
  const dim3 grid(2 * pa.n1 / kPjRows, (pa.B + 8 * bt - 1) / (8 * bt));
  const dim3 block(kPjWarps * 32);
  switch (bt) {
    case 1: project_qr_kernel<1, 8><<<grid, block, 0, stream>>>(pa); break;
    case 2: project_qr_kernel<2, 4><<<grid, block, 0, stream>>>(pa); break;
    case 4: project_qr_kernel<4, 4><<<grid, block, 0, stream>>>(pa); break;
    default: project_qr_kernel<kPjMaxTiles, 2><<<grid, block, 0, stream>>>(pa); break;
  }
  return note(cudaGetLastError()) == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}



// ----------------------------------------------------------------- prefill
template <bool kPaged>
plx_status launch_prefill_kernel(const CUtensorMap& tq, const CUtensorMap& tr, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const PrefillArgs& a, cudaStream_t stream) {
  constexpr int smem = PfLayout::kBytes;
  if (set_smem(prefill_tc_kernel<kPaged>, smem) !=
      cudaSuccess)
    return PLX_ERR_CUDA;
  const long long grid = (long long)a.n_mblk * a.B * a.H;
  prefill_tc_kernel<kPaged><<<(unsigned)grid, kPfThreads, smem, stream>>>(tq, tr, tk, tv, a);
  return note(cudaGetLastError()) == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

// Dense prefill: one CTA per 128 query rows (prefill_tc_kernel), or with
// p->cta_pair a cluster of two CTAs per 256 rows (prefill_tc2_kernel).
plx_status launch_prefill(const void* q, const void* rho, const void* k, const void* v, void* out,
                          const plx_prefill_params* p, cudaStream_t stream, float* vbar = nullptr,
                          float2* stats = nullptr) {
  const int hkv = p->num_kv_heads == 0 ? p->num_heads : p->num_kv_heads;
  const uint64_t rows_q = (uint64_t)p->batch * p->num_heads * p->seq_len;
  const uint64_t rows_kv = (uint64_t)p->batch * hkv * p->seq_len;
  const bool pair = p->cta_pair != 0;
  CUtensorMap tq, tr, tk, tv;
  if (!make_tmap_bf16(&tq, q, kPfD, rows_q, 64, kPfBM) || !make_tmap_bf16(&tr, rho, kPfD, rows_q, 64, kPfBM) ||
      !make_tmap_bf16(&tk, k, kPfD, rows_kv, 64, pair ? kPfBN / 2 : kPfBN) ||
      !make_tmap_bf16(&tv, v, kPfD, rows_kv, 64, kPfBN))
    return PLX_ERR_CUDA;
  PrefillArgs a{};
  a.B = p->batch;
  a.H = p->num_heads;
  a.Hkv = hkv;
  a.T = p->seq_len;
  a.group = p->num_heads / hkv;
  a.n_mblk = pair ? (p->seq_len + 2 * kPfBM - 1) / (2 * kPfBM)   // pairs of 128-row tiles
                  : (p->seq_len + kPfBM - 1) / kPfBM;
  a.causal = p->causal;
  a.out_bf16 = p->out_dtype == PLX_BF16 ? 1 : 0;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.out = out;
  a.wait_ns = current_wait_ns();
  a.vbar = vbar;
  a.stats = stats;
  if (!pair) return launch_prefill_kernel<false>(tq, tr, tk, tv, a, stream);
  constexpr int smem = P2Layout::kBytes;
  if (set_smem(prefill_tc2_kernel, smem) != cudaSuccess)
    return PLX_ERR_CUDA;
  const long long grid = 2LL * a.n_mblk * a.B * a.H;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note(cudaLaunchKernelEx(&cfg, prefill_tc2_kernel, tq, tr, tk, tv, a)) == cudaSuccess ? PLX_OK
                                                                                         : PLX_ERR_CUDA;
}

plx_status validate_prefill(const plx_prefill_params* p) {
  if (p == nullptr) return PLX_ERR_INVALID_ARG;
  const int hkv = p->num_kv_heads == 0 ? p->num_heads : p->num_kv_heads;
  if (p->batch < 1 || p->num_heads < 1 || hkv < 1 || p->seq_len < 1) return PLX_ERR_INVALID_ARG;
  if (p->num_heads % hkv != 0) return PLX_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return PLX_ERR_INVALID_ARG;
  if (!(p->scale > 0.f)) return PLX_ERR_INVALID_ARG;   // a softmax temperature is positive
  if (p->in_dtype != PLX_BF16) return p->in_dtype == PLX_F32 ? PLX_ERR_UNSUPPORTED : PLX_ERR_INVALID_ARG;
  if (p->out_dtype != PLX_F32 && p->out_dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  if (p->head_dim != 128) return PLX_ERR_UNSUPPORTED;
  if (p->causal != 0 && p->causal != 1) return PLX_ERR_INVALID_ARG;
  if (p->cta_pair != 0 && p->cta_pair != 1) return PLX_ERR_INVALID_ARG;
  if ((int64_t)p->batch * p->num_heads * ((int64_t)p->seq_len + 256) >= (int64_t)INT32_MAX)
    return PLX_ERR_UNSUPPORTED;
  return PLX_OK;
}

plx_status validate_prefill_paged(const plx_prefill_paged_params* p) {
  if (p == nullptr) return PLX_ERR_INVALID_ARG;
  if (p->batch < 1 || p->num_heads < 1 || p->num_kv_heads < 1) return PLX_ERR_INVALID_ARG;
  if (p->num_heads % p->num_kv_heads != 0) return PLX_ERR_INVALID_ARG;
  if (p->total_q < 0 || p->max_q_len < 0 || p->num_pages < 1 || p->max_pages_per_seq < 1)
    return PLX_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale) || !(p->scale > 0.f)) return PLX_ERR_INVALID_ARG;
  if (p->in_dtype != PLX_BF16) return p->in_dtype == PLX_F32 ? PLX_ERR_UNSUPPORTED : PLX_ERR_INVALID_ARG;
  if (p->out_dtype != PLX_F32 && p->out_dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  if (p->head_dim != 128) return PLX_ERR_UNSUPPORTED;
  if (p->page_size != kPfBN) return PLX_ERR_UNSUPPORTED;
  if (p->causal != 0 && p->causal != 1) return PLX_ERR_INVALID_ARG;
  // int32 TMA coordinates: pool rows and packed query rows; int32 key counts.
  if ((int64_t)p->num_pages * p->num_kv_heads * kPfBN >= (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  if ((int64_t)p->max_pages_per_seq * kPfBN >= (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  if ((int64_t)p->total_q + kPfBM >= (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  if (((int64_t)p->max_q_len + kPfBM - 1) / kPfBM * p->batch * p->num_heads >= (int64_t)INT32_MAX)
    return PLX_ERR_UNSUPPORTED;
  return PLX_OK;
}

// ----------------------------------------------------------- prefill backward
// Workspace of the backward: per row a float4 record and a 128-byte slab row.
size_t backward_records_bytes(const plx_prefill_params* p) {
  return ((size_t)p->batch * p->num_heads * p->seq_len * sizeof(float4) + 255) & ~size_t(255);
}
size_t backward_rows_bytes(const plx_prefill_params* p) {
  return backward_records_bytes(p) + (size_t)p->batch * p->num_heads * p->seq_len * 128;
}

plx_status launch_prefill_backward(const void* q, const void* rho, const void* k, const void* v, const void* out,
                                   const float* vbar, const float2* stats, const void* dout, void* dq, void* drho,
                                   void* dk, void* dv, float4* rows, const plx_prefill_params* p,
                                   cudaStream_t stream) {
  const int hkv = p->num_kv_heads == 0 ? p->num_heads : p->num_kv_heads;
  const long long n_rows = (long long)p->batch * p->num_heads * p->seq_len;
  const unsigned row_blocks = (unsigned)((n_rows + 7) / 8);
  uint32_t* slab = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(rows) + backward_records_bytes(p));
  const float scale_log2 = p->scale * 1.4426950408889634f;
  if (p->out_dtype == PLX_BF16)
    prefill_bwd_rows_kernel<true><<<row_blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(dout), out, vbar, stats, rows, slab, scale_log2, n_rows);
  else
    prefill_bwd_rows_kernel<false><<<row_blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(dout), out, vbar, stats, rows, slab, scale_log2, n_rows);
  if (note(cudaGetLastError()) != cudaSuccess) return PLX_ERR_CUDA;

  BwdArgs a{};
  a.B = p->batch;
  a.H = p->num_heads;
  a.Hkv = hkv;
  a.T = p->seq_len;
  a.group = p->num_heads / hkv;
  a.n_blk = (p->seq_len + kPfBM - 1) / kPfBM;
  a.causal = p->causal;
  a.out_bf16 = p->out_dtype == PLX_BF16 ? 1 : 0;
  a.scale = p->scale;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.rows = rows;
  a.dq = dq;
  a.drho = drho;
  a.dk = dk;
  a.dv = dv;
  a.wait_ns = current_wait_ns();
  const uint64_t rows_q = (uint64_t)n_rows;
  const uint64_t rows_kv = (uint64_t)p->batch * hkv * p->seq_len;
  {  // dq, drho: 128-row query tiles, 64-row key tiles
    CUtensorMap tq, tr, tg, tk, tv;
    if (!make_tmap_bf16(&tq, q, kPfD, rows_q, 64, kPfBM) || !make_tmap_bf16(&tr, rho, kPfD, rows_q, 64, kPfBM) ||
        !make_tmap_bf16(&tg, dout, kPfD, rows_q, 64, kPfBM) || !make_tmap_bf16(&tk, k, kPfD, rows_kv, 64, kPfBN) ||
        !make_tmap_bf16(&tv, v, kPfD, rows_kv, 64, kPfBN))
      return PLX_ERR_CUDA;
    constexpr int smem = BqLayout::kBytes;
    if (set_smem(prefill_bwd_dq_kernel, smem) !=
        cudaSuccess)
      return PLX_ERR_CUDA;
    const long long grid = (long long)a.n_blk * a.B * a.H;
    prefill_bwd_dq_kernel<<<(unsigned)grid, kPfThreads, smem, stream>>>(tq, tr, tg, tk, tv, a);
    if (note(cudaGetLastError()) != cudaSuccess) return PLX_ERR_CUDA;
  }
  {  // dk, dv: 128-row key tiles, 64-row query tiles (and their 64-column offset slab rows)
    CUtensorMap tq, tr, tg, tk, tv, ts;
    if (!make_tmap_bf16(&tq, q, kPfD, rows_q, 64, kPfBN) || !make_tmap_bf16(&tr, rho, kPfD, rows_q, 64, kPfBN) ||
        !make_tmap_bf16(&tg, dout, kPfD, rows_q, 64, kPfBN) || !make_tmap_bf16(&tk, k, kPfD, rows_kv, 64, kPfBM) ||
        !make_tmap_bf16(&tv, v, kPfD, rows_kv, 64, kPfBM) || !make_tmap_bf16(&ts, slab, 64, rows_q, 64, kPfBN))
      return PLX_ERR_CUDA;
    constexpr int smem = BkLayout::kBytes;
    if (set_smem(prefill_bwd_dkv_kernel, smem) !=
        cudaSuccess)
      return PLX_ERR_CUDA;
    const long long grid = (long long)a.n_blk * a.B * hkv;
    prefill_bwd_dkv_kernel<<<(unsigned)grid, kPfThreads, smem, stream>>>(tq, tr, tg, tk, tv, ts, a);
    if (note(cudaGetLastError()) != cudaSuccess) return PLX_ERR_CUDA;
  }
  return PLX_OK;
}

// ---------------------------------------------- decode without allocation
// Scratch for parallax_decode_noalloc: split partials and their counters
// live in this file-scope device array instead of a caller workspace.  Every
// GPU that loads the library holds PARALLAX_NOALLOC_SCRATCH_BYTES of it
// until the process exits.  In host code `g_noalloc_scratch` only names a
// host-side stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[PARALLAX_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices];

plx_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLX_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return PLX_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return PLX_OK;
}

// ------------------------------------------------ LLA with the solved probe
plx_status validate_lla(const plx_decode_params* p, float ridge) {
  plx_status st = validate_decode(p);
  if (st != PLX_OK) return st;
  if (!std::isfinite(ridge) || ridge < 0.f) return PLX_ERR_INVALID_ARG;
  if (p->in_dtype != PLX_BF16 || p->head_dim != kLlaD) return PLX_ERR_UNSUPPORTED;
  if ((int64_t)p->batch * p->num_q_heads * kLlaMaxPieces >= (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  return PLX_OK;
}

// Pieces each query head's keys are cut into: enough CTAs to fill the SMs
// (or num_ctas of them), at least four tiles per piece.
int lla_pieces(const plx_decode_params* p, int num_sms) {
  const int64_t heads = (int64_t)p->batch * p->num_q_heads;
  const int64_t want = p->num_ctas > 0 ? p->num_ctas : num_sms;
  int64_t k = want / heads;
  const int64_t tiles = ((int64_t)p->kv_len + kTile - 1) / kTile;
  if (k > tiles / 4) k = tiles / 4;
  if (k > kLlaMaxPieces) k = kLlaMaxPieces;
  if (k < 1) k = 1;
  return (int)k;
}

size_t lla_workspace_bytes(const plx_decode_params* p, int pieces) {
  return (size_t)p->batch * p->num_q_heads * pieces * kLlaRecFloats * sizeof(float);
}

}  // namespace

// A validated decode call whose kernel arguments and tensor maps are kept
// for repeated launches (parallax_decode_plan_*).
struct plx_decode_plan {
  DecodeLaunch L;
  plx_decode_params p;
  int device;
};

extern "C" {

int32_t parallax_abi_version(void) { return PARALLAX_ABI_VERSION; }

const char* parallax_status_string(plx_status s) {
  switch (s) {
    case PLX_OK: return "PLX_OK";
    case PLX_ERR_INVALID_ARG: return "PLX_ERR_INVALID_ARG";
    case PLX_ERR_UNSUPPORTED: return "PLX_ERR_UNSUPPORTED";
    case PLX_ERR_WORKSPACE: return "PLX_ERR_WORKSPACE";
    case PLX_ERR_CUDA: return "PLX_ERR_CUDA";
    case PLX_ERR_DEVICE_FAULT: return "PLX_ERR_DEVICE_FAULT";
    case PLX_ERR_TIMEOUT: return "PLX_ERR_TIMEOUT";
  }
  return "PLX_UNKNOWN_STATUS";
}

int32_t parallax_decode_num_ctas(const plx_decode_params* p, int32_t num_sms) {
  if (validate_decode(p) != PLX_OK) return -1;
  if (num_sms <= 0) num_sms = current_device_sms();
  if (num_sms <= 0) return -1;
  return plan_decode(p, num_sms).ctas;
}

size_t parallax_decode_workspace_size(const plx_decode_params* p, int32_t num_sms) {
  if (validate_decode(p) != PLX_OK) return (size_t)-1;
  if (num_sms <= 0) num_sms = current_device_sms();
  if (num_sms <= 0) return (size_t)-1;
  const DecodePlan pl = plan_decode(p, num_sms);
  return pl.counter_bytes + pl.slot_bytes;
}

plx_status parallax_decode(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                           const int32_t* page_table, const int32_t* seq_lens, void* out, void* workspace,
                           size_t workspace_bytes, const plx_decode_params* p, cudaStream_t stream) {
  DecodeLaunch L;
  const plx_status st =
      prepare_decode(q, rho, k_cache, v_cache, page_table, seq_lens, out, workspace, workspace_bytes, p, &L);
  if (st != PLX_OK) return st;
  return launch_decode(L, p, stream, kPdlAll);
}

plx_status parallax_decode_plan_create(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                                      const int32_t* page_table, const int32_t* seq_lens, void* out,
                                      void* workspace, size_t workspace_bytes, const plx_decode_params* p,
                                      plx_decode_plan** plan) {
  if (plan == nullptr) return PLX_ERR_INVALID_ARG;
  *plan = nullptr;
  plx_decode_plan* P = new (std::nothrow) plx_decode_plan;
  if (P == nullptr) return PLX_ERR_CUDA;
  plx_status st =
      prepare_decode(q, rho, k_cache, v_cache, page_table, seq_lens, out, workspace, workspace_bytes, p, &P->L);
  if (st == PLX_OK && cudaGetDevice(&P->device) != cudaSuccess) st = PLX_ERR_CUDA;
  if (st == PLX_OK) st = set_decode_attr(P->L, p);
  if (st != PLX_OK) {
    delete P;
    return st;
  }
  P->p = *p;
  *plan = P;
  return PLX_OK;
}

plx_status parallax_decode_plan_run(const plx_decode_plan* plan, cudaStream_t stream) {
  if (plan == nullptr) return PLX_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLX_ERR_CUDA;
  if (dev != plan->device) return PLX_ERR_INVALID_ARG;
  return launch_decode(plan->L, &plan->p, stream, kPdlAll, false);
}

plx_status parallax_decode_plan_run_io(const plx_decode_plan* plan, const void* host_q, const void* host_rho,
                                      void* host_out, cudaStream_t stream) {
  if (plan == nullptr || host_q == nullptr || host_rho == nullptr || host_out == nullptr) return PLX_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLX_ERR_CUDA;
  if (dev != plan->device) return PLX_ERR_INVALID_ARG;
  const plx_decode_params& p = plan->p;
  const size_t heads = (size_t)p.batch * p.num_q_heads * p.head_dim;
  const size_t in_bytes = heads * (p.in_dtype == PLX_BF16 ? 2 : 4);
  const size_t out_bytes = heads * (p.out_dtype == PLX_BF16 ? 2 : 4);
  // Page-locked host buffers mapped into the device's address space (pinned
  // memory under unified addressing): the kernel reads q, rho and writes the
  // output across PCIe itself, with no copy operations around it.
  auto mapped = [](const void* h, void** dptr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, h) != cudaSuccess) {
      cudaGetLastError();   // an unregistered pointer is an answer here, not an error
      return false;
    }
    *dptr = at.devicePointer;
    return at.type == cudaMemoryTypeHost && *dptr != nullptr && aligned(*dptr, 16);
  };
  void *dq = nullptr, *dr = nullptr, *dout = nullptr;
  if (mapped(host_q, &dq) && mapped(host_rho, &dr) && mapped(host_out, &dout)) {
    DecodeLaunch L = plan->L;
    L.a.q = dq;
    L.a.rho = dr;
    L.a.out = dout;
    L.a.qr_early = 1;   // the host supplies q and rho: they are read before the previous grid ends
    return launch_decode(L, &plan->p, stream, kPdlAll, false);
  }
  const DecodeArgs& a = plan->L.a;
  if (note(cudaMemcpyAsync(const_cast<void*>(a.q), host_q, in_bytes, cudaMemcpyHostToDevice, stream)) != cudaSuccess ||
      note(cudaMemcpyAsync(const_cast<void*>(a.rho), host_rho, in_bytes, cudaMemcpyHostToDevice, stream)) !=
          cudaSuccess)
    return PLX_ERR_CUDA;
  const plx_status st = launch_decode(plan->L, &plan->p, stream, kPdlAll, false);
  if (st != PLX_OK) return st;
  return note(cudaMemcpyAsync(host_out, a.out, out_bytes, cudaMemcpyDeviceToHost, stream)) == cudaSuccess
             ? PLX_OK
             : PLX_ERR_CUDA;
}

void parallax_decode_plan_destroy(plx_decode_plan* plan) { delete plan; }

plx_status parallax_decode_projected(const void* x, const void* w_q, const void* w_rho, int32_t hidden,
                                     const void* k_cache, const void* v_cache, const int32_t* page_table,
                                     const int32_t* seq_lens, void* q, void* rho, void* out, void* workspace,
                                     size_t workspace_bytes, const plx_decode_params* p, cudaStream_t stream) {
  plx_status st = validate_decode(p);
  if (st != PLX_OK) return st;
  if (!x || !w_q || !w_rho || hidden <= 0) return PLX_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_q, 16) || !aligned(w_rho, 16)) return PLX_ERR_INVALID_ARG;
  if (p->in_dtype != PLX_BF16 || hidden % 32 != 0) return PLX_ERR_UNSUPPORTED;
  const int64_t n1 = (int64_t)p->num_q_heads * p->head_dim;
  if (2 * n1 > (int64_t)INT32_MAX) return PLX_ERR_UNSUPPORTED;
  // The projection writes q and rho while other CTAs still read x and the
  // weights: the outputs must not overlap the inputs or each other.
  const size_t qr_bytes = (size_t)p->batch * n1 * 2, x_bytes = (size_t)p->batch * hidden * 2,
               w_bytes = (size_t)n1 * hidden * 2;
  for (const void* o : {q, rho}) {
    if (o == nullptr) return PLX_ERR_INVALID_ARG;
    if (overlaps(o, qr_bytes, x, x_bytes) || overlaps(o, qr_bytes, w_q, w_bytes) ||
        overlaps(o, qr_bytes, w_rho, w_bytes))
      return PLX_ERR_INVALID_ARG;
  }
  if (overlaps(q, qr_bytes, rho, qr_bytes)) return PLX_ERR_INVALID_ARG;
  DecodeLaunch L;
  if ((st = prepare_decode(q, rho, k_cache, v_cache, page_table, seq_lens, out, workspace, workspace_bytes, p,
                           &L)) != PLX_OK)
    return st;
  ProjArgs pa{};
  pa.x = static_cast<const __nv_bfloat16*>(x);
  pa.wq = static_cast<const __nv_bfloat16*>(w_q);
  pa.wr = static_cast<const __nv_bfloat16*>(w_rho);
  pa.q = static_cast<__nv_bfloat16*>(q);
  pa.rho = static_cast<__nv_bfloat16*>(rho);
  pa.B = p->batch;
  pa.n1 = (int)n1;
  pa.hidden = hidden;
  if ((st = launch_project(pa, stream)) != PLX_OK) return st;
  return launch_decode(L, p, stream, kPdlQR);
}

plx_status parallax_prefill(const void* q, const void* rho, const void* k, const void* v, void* out,
                            const plx_prefill_params* p, cudaStream_t stream) {
  plx_status st = validate_prefill(p);
  if (st != PLX_OK) return st;
  if (!q || !rho || !k || !v || !out) return PLX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(rho, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return PLX_ERR_INVALID_ARG;
  return launch_prefill(q, rho, k, v, out, p, stream);
}

plx_status parallax_prefill_train(const void* q, const void* rho, const void* k, const void* v, void* out,
                                  float* vbar, float* stats, const plx_prefill_params* p, cudaStream_t stream) {
  plx_status st = validate_prefill(p);
  if (st != PLX_OK) return st;
  if (!q || !rho || !k || !v || !out || !vbar || !stats) return PLX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(rho, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(vbar, 16) || !aligned(stats, 8))
    return PLX_ERR_INVALID_ARG;
  return launch_prefill(q, rho, k, v, out, p, stream, vbar, reinterpret_cast<float2*>(stats));
}

size_t parallax_prefill_backward_workspace_size(const plx_prefill_params* p) {
  if (validate_prefill(p) != PLX_OK) return SIZE_MAX;
  return backward_rows_bytes(p);
}

plx_status parallax_prefill_backward(const void* q, const void* rho, const void* k, const void* v,
                                     const void* out, const float* vbar, const float* stats, const void* dout,
                                     void* dq, void* drho, void* dk, void* dv, void* workspace,
                                     size_t workspace_bytes, const plx_prefill_params* p, cudaStream_t stream) {
  plx_status st = validate_prefill(p);
  if (st != PLX_OK) return st;
  const void* in[] = {q, rho, k, v, out, vbar, dout, dq, drho, dk, dv, workspace};
  for (const void* x : in)
    if (x == nullptr || !aligned(x, 16)) return PLX_ERR_INVALID_ARG;
  if (stats == nullptr || !aligned(stats, 8)) return PLX_ERR_INVALID_ARG;
  if (workspace_bytes < backward_rows_bytes(p)) return PLX_ERR_WORKSPACE;
  return launch_prefill_backward(q, rho, k, v, out, vbar, reinterpret_cast<const float2*>(stats), dout, dq, drho,
                                 dk, dv, static_cast<float4*>(workspace), p, stream);
}

plx_status parallax_prefill_paged(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                                  const int32_t* page_table, const int32_t* cu_seqlens_q, const int32_t* seq_lens,
                                  void* out, const plx_prefill_paged_params* p, cudaStream_t stream) {
  plx_status st = validate_prefill_paged(p);
  if (st != PLX_OK) return st;
  if (p->total_q == 0 || p->max_q_len == 0) return PLX_OK;   // no query rows: nothing to do
  if (!q || !rho || !k_cache || !v_cache || !page_table || !cu_seqlens_q || !seq_lens || !out)
    return PLX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(rho, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(out, 16) || !aligned(page_table, 4) || !aligned(cu_seqlens_q, 4) || !aligned(seq_lens, 4))
    return PLX_ERR_INVALID_ARG;
  const uint64_t pool_rows = (uint64_t)p->num_pages * p->num_kv_heads * kPfBN;
  CUtensorMap tq, tr, tk, tv;
  if (!make_tmap_bf16_heads(&tq, q, kPfD, p->num_heads, p->total_q, 64, kPfBM) ||
      !make_tmap_bf16_heads(&tr, rho, kPfD, p->num_heads, p->total_q, 64, kPfBM) ||
      !make_tmap_bf16(&tk, k_cache, kPfD, pool_rows, 64, kPfBN) ||
      !make_tmap_bf16(&tv, v_cache, kPfD, pool_rows, 64, kPfBN))
    return PLX_ERR_CUDA;
  PrefillArgs a{};
  a.B = p->batch;
  a.H = p->num_heads;
  a.Hkv = p->num_kv_heads;
  a.T = 0;
  a.group = p->num_heads / p->num_kv_heads;
  a.n_mblk = (p->max_q_len + kPfBM - 1) / kPfBM;
  a.causal = p->causal;
  a.out_bf16 = p->out_dtype == PLX_BF16 ? 1 : 0;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.out = out;
  a.wait_ns = current_wait_ns();
  a.cu_q = cu_seqlens_q;
  a.seq_lens = seq_lens;
  a.page_table = page_table;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.total_q = p->total_q;
  a.max_q = p->max_q_len;
  return launch_prefill_kernel<true>(tq, tr, tk, tv, a, stream);
}

plx_status parallax_decode_noalloc(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                                   const int32_t* page_table, const int32_t* seq_lens, void* out,
                                   const plx_decode_params* p, cudaStream_t stream) {
  plx_status st = validate_decode(p);
  if (st != PLX_OK) return st;
  const int num_sms = current_device_sms();
  if (num_sms <= 0) return PLX_ERR_CUDA;
  const DecodePlan pl = plan_decode(p, num_sms);
  if (pl.counter_bytes + pl.slot_bytes > (size_t)PARALLAX_NOALLOC_SCRATCH_BYTES) return PLX_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != PLX_OK) return st;
  // Every check runs before anything is queued on the stream.
  DecodeLaunch L;
  if ((st = prepare_decode(q, rho, k_cache, v_cache, page_table, seq_lens, out, scratch,
                           (size_t)PARALLAX_NOALLOC_SCRATCH_BYTES, p, &L)) != PLX_OK)
    return st;
  // The counters must start at zero; the array keeps whatever the last call left.
  if (cudaMemsetAsync(scratch, 0, L.pl.counter_bytes, stream) != cudaSuccess) return PLX_ERR_CUDA;
  return launch_decode(L, p, stream, kPdlAll);
}

plx_status parallax_set_wait_limit_ns(uint64_t limit_ns, uint64_t* previous) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PLX_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (previous != nullptr) *previous = g_wait_set[dev] ? g_wait_ns[dev] : kDefaultWaitNs;
  g_wait_ns[dev] = limit_ns;
  g_wait_set[dev] = true;
  return PLX_OK;
}

size_t parallax_lla_decode_workspace_size(const plx_decode_params* p, float ridge, int32_t num_sms) {
  if (validate_lla(p, ridge) != PLX_OK) return (size_t)-1;
  if (num_sms <= 0) num_sms = current_device_sms();
  if (num_sms <= 0) return (size_t)-1;
  return lla_workspace_bytes(p, lla_pieces(p, num_sms));
}

plx_status parallax_lla_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* page_table,
                               const int32_t* seq_lens, float ridge, float* rho, void* out, void* workspace,
                               size_t workspace_bytes, const plx_decode_params* p, cudaStream_t stream) {
  plx_status st = validate_lla(p, ridge);
  if (st != PLX_OK) return st;
  if (!q || !k_cache || !v_cache || !out) return PLX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      (rho && !aligned(rho, 16)))
    return PLX_ERR_INVALID_ARG;
  const bool paged = p->page_size != 0;
  if (paged && (page_table == nullptr || seq_lens == nullptr)) return PLX_ERR_INVALID_ARG;
  if (!paged && page_table != nullptr) return PLX_ERR_INVALID_ARG;
  if ((page_table && !aligned(page_table, 4)) || (seq_lens && !aligned(seq_lens, 4))) return PLX_ERR_INVALID_ARG;
  // The solve writes out and rho while other CTAs still read q.
  const size_t heads = (size_t)p->batch * p->num_q_heads;
  const size_t q_bytes = heads * kLlaD * 2, out_bytes = heads * kLlaD * (p->out_dtype == PLX_BF16 ? 2 : 4),
               rho_bytes = heads * kLlaD * 4;
  if (overlaps(out, out_bytes, q, q_bytes)) return PLX_ERR_INVALID_ARG;
  if (rho && (overlaps(rho, rho_bytes, q, q_bytes) || overlaps(rho, rho_bytes, out, out_bytes)))
    return PLX_ERR_INVALID_ARG;
  const int num_sms = current_device_sms();
  if (num_sms <= 0) return PLX_ERR_CUDA;
  const int pieces = lla_pieces(p, num_sms);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < lla_workspace_bytes(p, pieces))
    return PLX_ERR_WORKSPACE;

  LlaArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.rec = static_cast<float*>(workspace);
  a.out = out;
  a.rho = rho;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.group = p->num_q_heads / p->num_kv_heads;
  a.kv_len = p->kv_len;
  a.paged = paged ? 1 : 0;
  a.num_pages = paged ? p->num_pages : 0;
  a.max_pages = paged ? p->max_pages_per_seq : 0;
  a.pieces = pieces;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.ridge = ridge;
  a.out_bf16 = p->out_dtype == PLX_BF16 ? 1 : 0;
  a.wait_ns = current_wait_ns();
  // One piece per head: the moments kernel solves in place (its D_KK and
  // D_KV never leave tensor memory) and no solve grid is launched.
  a.fused = pieces == 1 && p->kv_len > 0 ? 1 : 0;
  if (p->kv_len > 0) {   // kv_len 0: every sequence is empty and the solve writes zeros
    const uint64_t rows = paged ? (uint64_t)p->num_pages * p->num_kv_heads * kTile
                                : (uint64_t)p->batch * p->num_kv_heads * p->kv_len;
    CUtensorMap tk, tv;
    if (!make_tmap_bf16(&tk, k_cache, kLlaD, rows, 64, kTile) || !make_tmap_bf16(&tv, v_cache, kLlaD, rows, 64, kTile))
      return PLX_ERR_CUDA;
    constexpr int smem = LlaLayout::kBytes;
    if (set_smem(lla_moments_kernel, smem) != cudaSuccess)
      return PLX_ERR_CUDA;
    if (launch_pdl(lla_moments_kernel, dim3((unsigned)(heads * pieces)), dim3(kLlaThreads), smem, stream, tk, tv, a) !=
        cudaSuccess)
      return PLX_ERR_CUDA;
  }
  if (a.fused) return PLX_OK;
  constexpr int ssmem = lla_solve_smem_bytes();
  if (set_smem(lla_solve_kernel, ssmem) != cudaSuccess)
    return PLX_ERR_CUDA;
  return launch_pdl(lla_solve_kernel, dim3((unsigned)heads), dim3(kLlaSolveThreads), ssmem, stream, a) == cudaSuccess
             ? PLX_OK
             : PLX_ERR_CUDA;
}

int32_t parallax_last_cuda_error(void) {
  const int e = g_last_cuda_error;
  g_last_cuda_error = 0;
  return e;
}

const char* parallax_cuda_error_string(int32_t code) { return cudaGetErrorString((cudaError_t)code); }

plx_status parallax_last_device_error(cudaStream_t stream, int32_t* code) {
  if (code == nullptr) return PLX_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PLX_ERR_CUDA;
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, plx::g_device_error, sizeof(v)) != cudaSuccess) return PLX_ERR_CUDA;
  if (cudaMemcpyToSymbol(plx::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return PLX_ERR_CUDA;
  *code = v;
  return PLX_OK;
}

}  // extern "C"
