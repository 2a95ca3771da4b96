/*
 * parallax.h -- C ABI of libparallax.so: Parallax attention forward on B200.
 *
 * Parallax is a parameterized Local Linear Attention.  For one query q with
 * probe rho over keys k_i and values v_i (sources: the newx.sg page
 * "Parallax: Parameterized Local Linear Attention for Language Modeling",
 * section "Abstract"; the wispaper.ai blog "Parallax: Breaking the Boundary
 * Bias with Parameterized Local Linear Attention", sections "The Core
 * Insight: Covariance Correction" and "Hardware Efficiency"):
 *
 *     w_i  = softmax_i(scale * q.k_i)
 *     vbar = sum_i w_i v_i,  kbar = sum_i w_i k_i
 *     S_KV = sum_i w_i (k_i - kbar)(v_i - vbar)^T        (d x d)
 *     out  = vbar - S_KV^T rho
 *
 * computed in one pass over the KV stream (the covariance matrix is never
 * formed): with e_i = exp(scale q.k_i - m), a_i = rho.k_i,
 *     out = (O1/l) (1 + c/l) - O2/l,
 *     l = sum e_i, c = sum e_i a_i, O1 = sum e_i v_i, O2 = sum e_i a_i v_i.
 *
 * Conventions shared by every entry point
 *   - Pointers named as device pointers are CUDA device memory of the
 *     current device, owned by the caller, dense row-major with the last
 *     dimension contiguous and 16-byte aligned.  The library keeps no
 *     pointer after a call returns and allocates no device memory.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).  They
 *     validate on the host first and launch nothing when validation fails.
 *   - Return values: plx_status.  Faults found by a kernel while it runs
 *     (an out-of-range page id, a pipeline wait that ran out of time) set a
 *     per-device error word read by parallax_last_device_error(); kernels
 *     never trap.
 *   - Not thread-safe across concurrent calls that share a workspace.
 */
#ifndef PARALLAX_H
#define PARALLAX_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PARALLAX_ABI_VERSION 10

typedef enum plx_status {
  PLX_OK = 0,
  PLX_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer      */
  PLX_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96)    */
  PLX_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required      */
  PLX_ERR_CUDA = 4,          /* a CUDA runtime / driver call or launch failed   */
  PLX_ERR_DEVICE_FAULT = 5,  /* a kernel reported bad input (see error word)    */
  PLX_ERR_TIMEOUT = 6        /* a kernel wait ran out of time (see error word)  */
} plx_status;

typedef enum plx_dtype { PLX_F32 = 0, PLX_BF16 = 1 } plx_dtype;

/* Device error word codes (bit flags; several may be set). */
#define PLX_DEVERR_BAD_PAGE   1   /* page_table entry outside [0, num_pages)     */
#define PLX_DEVERR_TIMEOUT    2   /* an mbarrier / pipeline wait gave up         */
#define PLX_DEVERR_BAD_LENGTH 4   /* a sequence length outside its allowed range */
#define PLX_DEVERR_SINGULAR   8   /* LLA: S_KK + ridge I not positive definite     */

/* ------------------------------------------------------------------------
 * Decode: one new query per (sequence, query head) over its KV cache.
 * Defined by the single-pass decode of the "Hardware Efficiency" section of
 * the wispaper.ai blog (softmax and covariance branches fused in one pass
 * over the KV stream), on the definition above.
 * ---------------------------------------------------------------------- */
typedef struct plx_decode_params {
  int32_t batch;              /* 1 <= B <= 8192                                */
  int32_t num_q_heads;        /* Hq, a multiple of num_kv_heads                */
  int32_t num_kv_heads;       /* Hkv; query head h reads KV head h / (Hq/Hkv)  */
  int32_t head_dim;           /* d: 64 or 128                                  */
  int32_t kv_len;             /* contiguous: rows per sequence in the cache, L;
                                 paged: upper bound of every seq_lens[b]       */
  int32_t page_size;          /* 0: contiguous cache; 64: paged cache          */
  int32_t num_pages;          /* paged: pages in the pool, P                   */
  int32_t max_pages_per_seq;  /* paged: row stride of page_table (>= ceil(kv_len/64)) */
  int32_t in_dtype;           /* plx_dtype of q, rho and the caches            */
  int32_t out_dtype;          /* plx_dtype of out                              */
  float scale;                /* softmax scale on q.k (e.g. 1/sqrt(d))         */
  int32_t num_ctas;           /* persistent CTAs; 0 = one per SM (bf16), or
                                 one per SM and at most one per four 64-token
                                 tiles (fp32); never more than the tiles    */
} plx_decode_params;

/* Work decomposition.  The 64-token KV tiles of every (sequence, KV head)
 * unit (bf16 caches; (sequence, query head) for fp32 caches) are laid end to
 * end and cut into num_ctas equal contiguous chunks, one per persistent CTA
 * (at most one CTA per tile).  A unit cut by chunk boundaries is finished by
 * the last CTA to complete one of its pieces, in the same launch. */

/* CTAs a decode call with these parameters launches on a device with
 * `num_sms` SMs (num_sms <= 0: the current device).  Host-only; makes no
 * CUDA call when num_sms > 0.  Returns -1 for invalid parameters. */
int32_t parallax_decode_num_ctas(const plx_decode_params* p, int32_t num_sms);

/* Workspace bytes parallax_decode needs, for `num_sms` as above; it does not
 * grow with the sequence lengths.  Returns (size_t)-1 for invalid
 * parameters.  Layout: a counter region (one int32 per unit, padded to
 * 256 B) followed by two fp32 partial slots per CTA.  The counter region
 * must be zero before the workspace is first used (e.g. cudaMemsetAsync);
 * every call that completes leaves it zero again, so one zeroing lasts for
 * the workspace's lifetime -- as long as nothing else writes it: memory
 * lent to another call in between (parallax_lla_decode's workspace, say)
 * must be zeroed again. */
size_t parallax_decode_workspace_size(const plx_decode_params* p, int32_t num_sms);

/* Parallax decode.
 *   q, rho      device, [B, Hq, d] of in_dtype: query and probe per head.
 *   k_cache,    device, in_dtype.  Contiguous (page_size 0): [B, Hkv, L, d].
 *   v_cache     Paged (page_size 64): pools [P, Hkv, 64, d]; logical token t
 *               of sequence b is row t % 64 of page page_table[b][t / 64].
 *   page_table  device int32 [B, max_pages_per_seq]; NULL when contiguous.
 *               Entries past a sequence's last page are not read.
 *   seq_lens    device int32 [B], 0 <= seq_lens[b] <= kv_len; NULL means
 *               every sequence has kv_len tokens (required when paged).
 *               A sequence of length 0 gets a zero output.
 *   out         device, [B, Hq, d] of out_dtype (bf16 output is rounded to
 *               nearest even from fp32).
 *   workspace   device, >= parallax_decode_workspace_size() bytes, 256-byte
 *               aligned.
 * Rows of the cache past a sequence's length are never used in arithmetic
 * (they may hold anything, NaN included). */
plx_status parallax_decode(const void* q, const void* rho,
                           const void* k_cache, const void* v_cache,
                           const int32_t* page_table, const int32_t* seq_lens,
                           void* out, void* workspace, size_t workspace_bytes,
                           const plx_decode_params* p, cudaStream_t stream);

/* Prepared decode: the validation, work plan, kernel arguments and TMA
 * descriptors of one parallax_decode call, kept for repeated launches on
 * the same buffers (a serving loop that decodes into fixed q / rho / out
 * buffers over a resident cache pays the host-side preparation once).
 *
 * parallax_decode_plan_create takes exactly the arguments of
 * parallax_decode, minus the stream, checks them as parallax_decode does
 * and returns a host-allocated plan in *plan (NULL on error).  The plan
 * keeps the pointers, not the data: every buffer must stay allocated, at the
 * same address, for the plan's lifetime, and the contents (q, rho, the
 * cache, page_table, seq_lens) are read at each run.  The workspace follows
 * parallax_decode's rule (counter region zero before the first run; every
 * completed run leaves it zero); runs that share a workspace must not
 * overlap on the GPU.  The plan is bound to the device current at creation
 * (PLX_ERR_INVALID_ARG if another device is current at a run) and to the
 * pipeline wait limit in force then.
 *
 * parallax_decode_plan_run launches the decode on `stream` (one launch,
 * asynchronous); parallax_decode_plan_destroy frees the plan (NULL is a
 * no-op).  Host-only otherwise: no CUDA allocation. */
typedef struct plx_decode_plan plx_decode_plan;

plx_status parallax_decode_plan_create(const void* q, const void* rho,
                                      const void* k_cache, const void* v_cache,
                                      const int32_t* page_table, const int32_t* seq_lens,
                                      void* out, void* workspace, size_t workspace_bytes,
                                      const plx_decode_params* p, plx_decode_plan** plan);
plx_status parallax_decode_plan_run(const plx_decode_plan* plan, cudaStream_t stream);

/* One serving step from host memory: host_q and host_rho ([B, Hq, d] of
 * in_dtype) in, host_out ([B, Hq, d] of out_dtype) out, on `stream`,
 * asynchronous; the host buffers must stay valid (and host_out unread)
 * until the stream reaches the step.  When all three are page-locked and
 * mapped into the device's address space (cudaHostAlloc / pinned memory
 * under unified addressing, 16-byte aligned), the one launch reads q and rho
 * and writes the output across PCIe directly, and the plan's own q, rho and
 * out buffers are not touched.  In that case q and rho are read as the
 * launch starts, which may be before the kernel queued just ahead of it on
 * the stream has finished (programmatic dependent launch; the KV cache and
 * the output wait for it): host_q and host_rho must be written by the host
 * before the call, not by device work queued on the stream.  Otherwise it copies host_q and host_rho into
 * the plan's q and rho, runs the decode and copies the plan's out into
 * host_out: three copies and one launch (page-locked buffers let the copies
 * overlap other work).  Errors as parallax_decode_plan_run;
 * PLX_ERR_INVALID_ARG for a null host pointer. */
plx_status parallax_decode_plan_run_io(const plx_decode_plan* plan, const void* host_q, const void* host_rho,
                                      void* host_out, cudaStream_t stream);
void parallax_decode_plan_destroy(plx_decode_plan* plan);

/* Decode whose query and probe are projected from the new token's layer
 * input in the same call.
 *
 * Parallax learns the probe as a linear projection of the input (wispaper
 * blog, "The Core Insight: Covariance Correction"; the newx.sg "Abstract"
 * calls it an extra query-like projector).  For every sequence b and query
 * head h, with d = head_dim and n = h*d + j:
 *     q[b, h, j]   = bf16( sum_c w_q[n, c]   x[b, c] )
 *     rho[b, h, j] = bf16( sum_c w_rho[n, c] x[b, c] )
 * (fp32 sums, rounded to nearest even), then parallax_decode(q, rho, ...).
 *
 *   x            device bf16 [B, hidden]: the new token's layer input.
 *   w_q, w_rho   device bf16 [Hq * d, hidden]: output feature by input
 *                feature (row n belongs to head n / d, component n % d).
 *   hidden       > 0 and a multiple of 32 (else PLX_ERR_UNSUPPORTED).
 *   q, rho       device bf16 [B, Hq, d]: written with the projections, then
 *                read by the decode.  Neither may overlap x, the weights or
 *                the other (PLX_ERR_INVALID_ARG); out may be q itself.
 *   the rest     as parallax_decode; in_dtype must be PLX_BF16 (the cache
 *                is bf16), else PLX_ERR_UNSUPPORTED.  Workspace size: as
 *                parallax_decode_workspace_size().
 *
 * Two launches on `stream`: the projection kernel, then the decode kernel
 * with a programmatic dependency on it, so that the decode's set-up and its
 * first K/V loads overlap the projection; the decode reads q and rho only
 * after the projection grid has completed.  Every check of parallax_decode
 * runs before the first launch; if the second launch fails, q and rho are
 * written and out is not (PLX_ERR_CUDA). */
plx_status parallax_decode_projected(const void* x, const void* w_q, const void* w_rho, int32_t hidden,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* page_table, const int32_t* seq_lens,
                                     void* q, void* rho, void* out,
                                     void* workspace, size_t workspace_bytes,
                                     const plx_decode_params* p, cudaStream_t stream);

/* Decode that allocates nothing and takes no workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory or own a workspace: a plugin running
 * inside a host application that budgets all GPU memory itself, a binding
 * from a language runtime that has no CUDA allocator of its own, or a
 * latency-critical path that must not pay for cudaMalloc and the
 * synchronisation it can imply.
 *
 * Same arguments and results as parallax_decode, minus the workspace.  The
 * split partials live in a library-owned device array of
 * PARALLAX_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library
 * holds until the process exits.  The first call on a device looks up that
 * array's device address (cudaGetSymbolAddress, with the device current);
 * make that first call before any stream capture.  Each call clears the
 * counter region of the array on `stream` before launching.  Calls share
 * the one array: calls that overlap on the GPU (other streams, other host
 * threads) race and give wrong results; serialise them.  Parameters whose
 * parallax_decode_workspace_size() exceeds the array return
 * PLX_ERR_WORKSPACE before any launch.  No cudaMalloc, cudaFree or
 * allocating library routine is called. */
#define PARALLAX_NOALLOC_SCRATCH_BYTES (8u << 20)

plx_status parallax_decode_noalloc(const void* q, const void* rho,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* page_table, const int32_t* seq_lens,
                                   void* out, const plx_decode_params* p, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Local Linear Attention (LLA) with the solved probe, decode form.
 *
 * LLA is the local linear estimate at the query: the intercept of the
 * softmax-weighted least-squares fit v ~ a + M^T (k - q) (newx.sg page,
 * section "Abstract": softmax attention's local constant estimate upgraded
 * to a local linear one; wispaper.ai blog, section "Context: Why Softmax is
 * Not Enough": LLA solves a linear system for every token).  It is Parallax
 * with the probe solved instead of learned:
 *     (S_KK + ridge I) rho* = kbar - q,     out = vbar - S_KV^T rho*,
 *     S_KK = sum_i w_i (k_i - kbar)(k_i - kbar)^T,
 * with w, kbar, vbar and S_KV as in the definition at the top.  `ridge`
 * (>= 0, finite) penalises the slope M; the pages name no regularisation,
 * and 0 is plain LLA, which needs more effectively weighted keys than d.
 * The pages solve by conjugate gradients; here each query head's system is
 * formed in fp32 and solved exactly by a Cholesky factorisation.
 *
 * On `stream`: a single pass over each query head's K and V that
 * accumulates sum w k k^T and sum w k v^T on the tensor cores (with the
 * first moments), and one solve per query head that also writes out.  When
 * each query head's keys are one piece (num_ctas, or for 0 the SM count,
 * below twice the number of (sequence, query head) pairs, or kv_len below
 * 512) that is one launch: the pass's kernel
 * solves in place, its sums never leaving tensor memory, and the workspace
 * is not touched.  Otherwise the pieces' sums go to the workspace and a
 * second launch merges them and solves.
 *
 *   q            device bf16 [B, Hq, 128].
 *   k_cache,     device bf16, contiguous [B, Hkv, L, 128] or paged pools
 *   v_cache      [P, Hkv, 64, 128], with page_table / seq_lens exactly as
 *                for parallax_decode (a sequence of length 0 gets out = 0
 *                and rho* = 0).
 *   rho          device float32 [B, Hq, 128]: the solved probe, or NULL.
 *   out          device [B, Hq, 128] of out_dtype.  Neither out nor rho may
 *                overlap q or each other (PLX_ERR_INVALID_ARG).
 *   workspace    device, >= parallax_lla_decode_workspace_size() bytes,
 *                256-byte aligned; no initialisation needed.
 *   p            as parallax_decode; in_dtype PLX_BF16 and head_dim 128
 *                (else PLX_ERR_UNSUPPORTED).  num_ctas 0 picks how many
 *                pieces each query head's keys are cut into (one CTA each);
 *                num_ctas > 0 asks for about that many CTAs in total.
 * A query head whose factorisation meets a pivot that is not positive
 * (S_KK + ridge I not numerically positive definite, e.g. ridge 0 and one
 * key) sets PLX_DEVERR_SINGULAR and gets rho* = 0, out = vbar.  With ridge 0
 * and fewer effectively weighted keys than d the system is ill-posed even
 * when every pivot is positive: pass ridge > 0 for short sequences.  Other
 * errors as parallax_decode. */

/* Workspace bytes of parallax_lla_decode for these parameters on a device
 * with `num_sms` SMs (<= 0: the current device), or (size_t)-1 for invalid
 * ones: 132 KB per (query head, piece) -- the two d x d sums, the first
 * moments, the running max and the normaliser. */
size_t parallax_lla_decode_workspace_size(const plx_decode_params* p, float ridge, int32_t num_sms);

plx_status parallax_lla_decode(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* page_table, const int32_t* seq_lens, float ridge,
                               float* rho, void* out, void* workspace, size_t workspace_bytes,
                               const plx_decode_params* p, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Prefill: every position of a sequence is a query; causal (key i visible
 * to query t iff i <= t) or full.  The same definition per row; the dense
 * contractions (q.K^T, rho.K^T, P.V, (P o A).V) run on tcgen05 tensor cores.
 * ---------------------------------------------------------------------- */
typedef struct plx_prefill_params {
  int32_t batch;          /* B                                                */
  int32_t num_heads;      /* H (query heads)                                  */
  int32_t num_kv_heads;   /* Hkv, divides H; 0 means H                        */
  int32_t seq_len;        /* T >= 1                                           */
  int32_t head_dim;       /* d: 128                                           */
  int32_t in_dtype;       /* PLX_BF16                                         */
  int32_t out_dtype;      /* PLX_BF16 or PLX_F32                              */
  float scale;            /* softmax scale on q.k, > 0                        */
  int32_t causal;         /* 1: causal mask (diagonal included); 0: none      */
  int32_t cta_pair;       /* 0: one CTA (one SM) per 128 query rows; 1: a
                             cluster of two CTAs per 256 rows, one tcgen05
                             instruction (cta_group::2) for both, each SM
                             loading half of every K and V tile.  Same
                             results; 0 is the faster one as measured.      */
} plx_prefill_params;

/* Parallax prefill.
 *   q, rho   device, [B, H, T, d] bf16.
 *   k, v     device, [B, Hkv, T, d] bf16.
 *   out      device, [B, H, T, d] of out_dtype. */
plx_status parallax_prefill(const void* q, const void* rho, const void* k, const void* v,
                            void* out, const plx_prefill_params* p, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Training: the prefill forward with the per-row quantities its backward
 * reads, and the backward.  For a row with weights w_i, probe values
 * a_i = rho.k_i, abar = sum w_i a_i and vbar = sum w_i v_i the output is
 * out = sum_i w_i (1 + abar - a_i) v_i (the covariance correction of the
 * wispaper.ai blog "Parallax: Breaking the Boundary Bias with Parameterized
 * Local Linear Attention", section "The Core Insight: Covariance Correction");
 * the backward differentiates that expression (the pages print no
 * gradient).
 * ---------------------------------------------------------------------- */

/* parallax_prefill, plus:
 *   vbar    device float32 [B, H, T, d]: sum_i w_i v_i of every row.
 *   stats   device float32 [B, H, T, 2]: (x, abar) per row, where
 *           w_i = 2^(scale * log2(e) * q.k_i - x) (x = log2 of the softmax
 *           normaliser of the scaled scores).
 * out is written in out_dtype as by parallax_prefill.  Same errors. */
plx_status parallax_prefill_train(const void* q, const void* rho, const void* k, const void* v,
                                  void* out, float* vbar, float* stats,
                                  const plx_prefill_params* p, cudaStream_t stream);

/* Bytes of workspace parallax_prefill_backward needs, or SIZE_MAX for
 * invalid parameters: per row (B * H * T rows) a 16-byte record (rounded up
 * to 256 bytes in total) and a 128-byte row of bf16 offsets. */
size_t parallax_prefill_backward_workspace_size(const plx_prefill_params* p);

/* Gradients of L through one prefill, given dout = dL/dout.
 *   q, rho, k, v    the forward's inputs (bf16, layouts as parallax_prefill).
 *   out, vbar, stats  the outputs of parallax_prefill_train for them (out
 *                   in out_dtype).
 *   dout            device bf16 [B, H, T, d].
 *   dq, drho        device [B, H, T, d] of out_dtype.
 *   dk, dv          device [B, Hkv, T, d] of out_dtype (summed over the
 *                   query heads that share each KV head).
 *   workspace       device, >= parallax_prefill_backward_workspace_size.
 * Every output element is written exactly once (no atomics, deterministic).
 * Three launches on `stream`.  Errors: PLX_ERR_INVALID_ARG (null or
 * misaligned pointer, bad parameters), PLX_ERR_UNSUPPORTED (as
 * parallax_prefill), PLX_ERR_WORKSPACE, PLX_ERR_CUDA. */
plx_status parallax_prefill_backward(const void* q, const void* rho, const void* k, const void* v,
                                     const void* out, const float* vbar, const float* stats,
                                     const void* dout, void* dq, void* drho, void* dk, void* dv,
                                     void* workspace, size_t workspace_bytes,
                                     const plx_prefill_params* p, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Chunked (append) prefill over the paged cache: the step between a prompt
 * chunk and decode in a serving loop.  The same per-query definition as
 * decode and prefill (out = vbar - S_KV^T rho over the query's visible keys;
 * wispaper.ai blog "Parallax: Breaking the Boundary Bias with Parameterized
 * Local Linear Attention", section "The Core Insight: Covariance Correction").
 *
 * Sequence b holds L_b = seq_lens[b] keys in 64-token pages, laid out as in
 * paged decode.  Its q_len_b = cu_seqlens_q[b+1] - cu_seqlens_q[b] queries
 * are the sequence's LAST q_len_b positions, L_b - q_len_b .. L_b - 1, so
 * their own keys and values must already be in the cache.  Query i of
 * sequence b sees keys 0 .. L_b - q_len_b + i (causal) or all L_b keys.
 * A one-token chunk is a decode step; parallax_decode is the faster kernel
 * for it.
 * ---------------------------------------------------------------------- */
typedef struct plx_prefill_paged_params {
  int32_t batch;              /* B sequences                                  */
  int32_t num_heads;          /* H query heads                                */
  int32_t num_kv_heads;       /* Hkv, divides H                               */
  int32_t head_dim;           /* d: 128                                       */
  int32_t total_q;            /* rows of q, rho and out (= cu_seqlens_q[B])   */
  int32_t max_q_len;          /* >= every q_len_b; sets the grid             */
  int32_t page_size;          /* 64                                           */
  int32_t num_pages;          /* P, pages in each pool                        */
  int32_t max_pages_per_seq;  /* page_table row stride                        */
  int32_t in_dtype;           /* PLX_BF16                                     */
  int32_t out_dtype;          /* PLX_BF16 or PLX_F32                          */
  float scale;                /* softmax scale on q.k, > 0                    */
  int32_t causal;             /* 1: causal (diagonal included); 0: none       */
} plx_prefill_paged_params;

/* Paged chunked prefill.
 *   q, rho        device, [total_q, H, d] bf16; sequence b's rows start at
 *                 cu_seqlens_q[b].
 *   k_cache,      device, pools [P, Hkv, 64, d] bf16.  Slots past L_b in a
 *   v_cache       sequence's last page may hold anything, NaN included.
 *   page_table    device int32 [B, max_pages_per_seq]; entries 0 ..
 *                 ceil(L_b/64)-1 of row b are read.
 *   cu_seqlens_q  device int32 [B + 1], non-decreasing, cu_seqlens_q[B] <= total_q.
 *   seq_lens      device int32 [B], q_len_b <= L_b <= 64 * max_pages_per_seq.
 *   out           device, [total_q, H, d] of out_dtype; rows that belong to
 *                 no sequence are left untouched.
 * All buffers are caller-owned; nothing is allocated.  Asynchronous on
 * `stream`.  total_q == 0 or max_q_len == 0 returns PLX_OK without a launch.
 * Errors: host checks give PLX_ERR_INVALID_ARG / PLX_ERR_UNSUPPORTED before
 * any launch.  On the device, a sequence whose lengths break the rules
 * above (or exceed max_q_len) sets PLX_DEVERR_BAD_LENGTH, one whose pages
 * fall outside [0, P) sets PLX_DEVERR_BAD_PAGE; its rows are not written. */
plx_status parallax_prefill_paged(const void* q, const void* rho,
                                  const void* k_cache, const void* v_cache,
                                  const int32_t* page_table, const int32_t* cu_seqlens_q,
                                  const int32_t* seq_lens, void* out,
                                  const plx_prefill_paged_params* p, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Errors and introspection.
 * ---------------------------------------------------------------------- */

/* Synchronises `stream`, then reads and clears the current device's error
 * word into *code (0 = no fault, else PLX_DEVERR_* bits).  Returns PLX_OK,
 * or PLX_ERR_CUDA if the synchronisation or the read failed. */
plx_status parallax_last_device_error(cudaStream_t stream, int32_t* code);

/* Sets the limit of one pipeline wait in the kernels launched afterwards on
 * the current device, in nanoseconds, and returns the previous limit in
 * *previous (if not NULL).  A pipeline wait is one role of a CTA waiting for
 * another's data or buffer (a TMA load to land, tensor-core results, a freed
 * stage); the default limit is 2 s, far above any healthy wait.  When a wait
 * runs out, the kernel sets PLX_DEVERR_TIMEOUT in the error word, abandons
 * its work, waits for its own copies and tensor-core operations still in
 * flight (those waits keep a fixed 2 s limit) and exits; its outputs are
 * then undefined.  0 makes every wait give up unless its phase is already
 * complete, which exercises that path deliberately.  A serving loop may set
 * a shorter limit to learn sooner that a kernel is stuck.  Host-only; takes
 * effect at the next launch.  Errors: PLX_ERR_CUDA (no current device). */
plx_status parallax_set_wait_limit_ns(uint64_t limit_ns, uint64_t* previous);

/* The CUDA error (a cudaError_t value) behind the last PLX_ERR_CUDA that a
 * call on this host thread returned, or 0; reading it clears it. */
int32_t parallax_last_cuda_error(void);

/* CUDA's description of a cudaError_t value. */
const char* parallax_cuda_error_string(int32_t code);

/* Static string naming a status. */
const char* parallax_status_string(plx_status s);

/* PARALLAX_ABI_VERSION of the loaded library. */
int32_t parallax_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PARALLAX_H */
