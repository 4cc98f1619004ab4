/*
 * apr.h -- C ABI of libapr: token-level pre-gated mixture-of-LoRA with a
 * segmented gather product (SGMM), for NVIDIA B200 (sm_100a).
 *
 * The operations follow the AdaFuse summary ("AdaFuse: Accelerating Dynamic
 * Adapter Inference via Token-Level Pre-Gating and Fused Kernel
 * Optimization", gist.science, Resumen tecnico):
 *   - section 2.A: one light router, run once per token at the first adapted
 *     layer, fixes the adapters of every later layer of that token;
 *   - section 2.B, decoding steps 1-2: one router pass, top-K selection;
 *   - section 2.B, SGMM: one batched product over the tokens gathered per
 *     adapter applies (fuses) the selected adapters in a single kernel call;
 *   - section 2.B, steps 3-5: merge the selected adapters into the backbone,
 *     run the base model, unmerge for the next token.
 *
 * Conventions (all entry points):
 *   - Every buffer belongs to the caller.  The library never allocates or
 *     frees device memory.  Pointers named "device" must be device (or
 *     managed) memory of the current device; "host" pointers are read before
 *     the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  Host-side argument checks happen
 *     before anything is launched and return an error status with nothing
 *     enqueued.  Faults the device detects (an adapter index out of range, a
 *     rank above the declared maximum) set an error word in the workspace
 *     and the offending rows are skipped; they never trap.  Read and clear
 *     that word with apr_stream_status().
 *   - Kernels are launched with programmatic dependent launch allowed: each
 *     waits for its predecessor on the stream before touching activations,
 *     routing, outputs or the workspace, so stream order is kept and
 *     consecutive calls may overlap their launch.  Adapter weights (A, B) and
 *     ranks, which no kernel of this library writes, may be read before that
 *     wait; a caller that rewrites them with its own kernel just before a call
 *     on the same stream must not let that kernel signal its dependents early
 *     (griddepcontrol.launch_dependents).
 *   - Layouts are row-major and dense.  Element type is given by `dtype`
 *     (APR_F32 or APR_BF16) for activations and adapter weights; router
 *     logits are accumulated and gates are produced in fp32.
 *   - Device pointers to activations and weights must be 16-byte aligned and
 *     every row length a multiple of 8 elements.
 *   - No C++ exception crosses this boundary.  apr_last_error() returns a
 *     thread-local description of the last failure.
 */
#ifndef APR_H_
#define APR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum apr_status {
  APR_OK = 0,
  APR_ERR_INVALID_ARG = 1,  /* a host-checkable argument is wrong            */
  APR_ERR_UNSUPPORTED = 2,  /* valid but outside this build's limits         */
  APR_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small    */
  APR_ERR_CUDA = 4,         /* a CUDA runtime call failed                     */
  APR_ERR_DEVICE_INDEX = 5, /* device saw an adapter index/rank out of range */
  APR_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up            */
} apr_status;

typedef enum apr_dtype { APR_F32 = 0, APR_BF16 = 1 } apr_dtype;

/* Limits of this build. */
#define APR_MAX_E 1024        /* adapters                                   */
#define APR_MAX_K 8           /* adapters per token                         */
#define APR_MAX_RANK 128      /* LoRA rank, a multiple of 8                 */
#define APR_MAX_PROJ 4        /* projections sharing one input per SGMM call */

/* Kernel choice for apr_sgmm_shrink_expand. */
typedef enum apr_sgmm_kernel {
  APR_SGMM_AUTO = 0,    /* by T, E, the ranks and the mean segment size T*k/E */
  APR_SGMM_SKINNY = 1,  /* CUDA-core kernel for few tokens per adapter        */
  APR_SGMM_TENSOR = 2,  /* tcgen05 tensor-core kernel for long segments       */
  APR_SGMM_DENSE = 3,   /* tcgen05 over the whole adapter bank, small batches */
  APR_SGMM_BANK = 4     /* tcgen05 in token order over the whole bank: few
                           adapters, many tokens (contiguous y tiles by TMA) */
} apr_sgmm_kernel;

/* ------------------------------------------------------------------------
 * Workspace.  One device buffer of apr_workspace_size() bytes, 256-byte
 * aligned, serves a whole step: apr_pregate_route uses it as scratch,
 * apr_segment_tokens writes the routing plan into it, and every
 * apr_sgmm_shrink_expand of the step reads that plan (so it must be the same
 * buffer, untouched in between).  It starts with an error word: zero it once
 * with apr_workspace_init() before first use.  Calls that share a workspace
 * must be ordered on one stream.
 *   T, k, E      : largest token count, top-k and adapter count of the step
 *   max_rank     : largest adapter rank
 *   max_d_in     : largest SGMM input width
 * Returns 0 when an argument is out of range.
 * ---------------------------------------------------------------------- */
size_t apr_workspace_size(int T, int k, int E, int max_rank, int max_d_in);
apr_status apr_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Token-level pre-gate (section 2.A; section 2.B steps 1-2).
 *   L[t,e]   = sum_i h[t,i] * Wr[e,i]           (fp32 accumulation)
 *   idx[t,:] = the k adapters with the largest L[t,.], in descending order;
 *              equal logits go to the lower adapter index
 *   gate[t,j]= exp(L[t,idx[t,j]] - L[t,idx[t,0]]) / sum_j' exp(...)
 * h        device [T, d]  dtype     router input (hidden state of the token)
 * Wr       device [E, d]  dtype     router weight
 * idx      device [T, k]  int32     out
 * gate     device [T, k]  fp32      out
 * ws       device workspace (scratch for split-K partial logits)
 * Limits: 1 <= k <= min(E, APR_MAX_K), E <= APR_MAX_E, d % 8 == 0.  T == 0
 * is a no-op.  Logits must be finite; sums of products stay exact when the
 * inputs are small integers scaled by powers of two.
 * ---------------------------------------------------------------------- */
apr_status apr_pregate_route(const void* h, const void* Wr, int dtype, int T, int d, int E,
                             int k, int32_t* idx, float* gate, void* ws, size_t ws_bytes,
                             void* stream);

/* ------------------------------------------------------------------------
 * apr_pregate_route with no workspace: the paper has no counterpart; this is
 * a convenience of this library.  It exists for callers that cannot allocate
 * device memory for a workspace -- code without an allocator of its own (a
 * plug-in whose host application owns every byte of device memory) or a
 * latency-critical loop in which cudaMalloc and the device-wide
 * synchronisation it can trigger are not acceptable.
 * Same arguments (minus the workspace), same results as apr_pregate_route.
 * Its scratch is one fixed 8 MiB array inside libapr, which every GPU that
 * loads the library keeps until the process exits; it holds the split-K
 * partial logits, so T*E must not exceed 2,097,088, else the call returns
 * APR_ERR_UNSUPPORTED with nothing enqueued.  The first call on a device
 * looks the array up on that device (cudaGetSymbolAddress); make that first
 * call before any stream capture.  The address is kept for the life of the
 * process: after cudaDeviceReset (or a primary context that is released and
 * created again) the array moves, and this entry point must not be used on
 * that device again without restarting the process.  Every call uses the same array and leaves
 * its contents behind, so calls that overlap on the GPU (for example on two
 * streams with no ordering between them) race with each other.  Nothing is
 * allocated or freed.  A token whose logits are all NaN gets adapter 0; there
 * is no workspace in which to report that.
 * ---------------------------------------------------------------------- */
apr_status apr_pregate_route_noalloc(const void* h, const void* Wr, int dtype, int T, int d, int E,
                                     int k, int32_t* idx, float* gate, void* stream);

/* ------------------------------------------------------------------------
 * Segments (the "segmented gather" of section 2.B's SGMM).
 * Pair q = t*k + j belongs to adapter idx[t,j].
 *   seg_off  device [E+1] int32  out: seg_off[0] = 0, seg_off[e+1]-seg_off[e] =
 *                                pairs of adapter e (exclusive prefix sum)
 *   perm     device [T*k] int32  out: pair ids grouped by adapter, ascending
 *                                q inside each segment (a stable counting sort)
 * Also writes the routing plan that apr_sgmm_shrink_expand reads from `ws`
 * (inverse permutation, tokens ordered by adapter set, tile lists).
 * An index outside [0, E) sets APR_ERR_DEVICE_INDEX in the workspace and
 * leaves every segment empty.  Deterministic; bit-exact.
 * ---------------------------------------------------------------------- */
apr_status apr_segment_tokens(const int32_t* idx, int T, int k, int E, int32_t* seg_off,
                              int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/* One projection of a shared-input group. */
typedef struct apr_proj {
  void* y;                /* device [T, d_out] out; may equal y_base (in place)   */
  const void* y_base;     /* device [T, d_out] base projection output             */
  int d_out;              /* output width, a multiple of 8                        */
  const void* const* A;   /* device array [E] of device pointers, A[e] -> [r_e, d_in] */
  const void* const* B;   /* device array [E] of device pointers, B[e] -> [d_out, r_e] */
} apr_proj;

/* ------------------------------------------------------------------------
 * SGMM shrink/expand fused into the add onto the base output (section 2.B).
 * For every projection p of the group and every token t:
 *   y_p[t] = y_base_p[t] + sum_j gate[t,j] * B_e (A_e x[t]),  e = idx[t,j]
 * with fp32 accumulation and one rounding to dtype per output element.
 * x        device [T, d_in] dtype, shared by the nproj projections
 * projs    host   [nproj] (1 <= nproj <= APR_MAX_PROJ)
 * ranks    device [E] int32, r_e in [8, max_rank], multiples of 8
 * max_rank host   bound on ranks (multiple of 8, <= APR_MAX_RANK)
 * idx,gate device [T,k]: the outputs of apr_pregate_route (the same routing
 *          is reused by every layer, section 2.A)
 * seg_off,perm device: the outputs of apr_segment_tokens for this idx; `ws`
 *          must be the workspace that call wrote.
 * kernel   APR_SGMM_AUTO, or a forced kernel class.  With R16 = max_rank
 *          rounded up to 16: the tensor-core kernel needs dtype == APR_BF16
 *          and d_in % 64 == 0, and for k = 2 also k * R16 <= 64 and
 *          d_out % 16 == 0 (k = 1 takes every rank up to APR_MAX_RANK: the
 *          adapters of up to 16 short segments share one 128-token tile,
 *          the Chameleon page's many tenants of ranks 8-128); the
 *          dense kernel needs dtype == APR_BF16, T <= 64, E <= 16 and
 *          E * R16 <= 256; the bank kernel needs dtype == APR_BF16, R16 in
 *          {16, 32, 64}, k <= 4, k * R16 <= 64, E * R16 <= 256 and
 *          d_in % 64 == 0.  A forced kernel returns APR_ERR_UNSUPPORTED
 *          outside its range.  AUTO takes the dense kernel where it applies,
 *          else the bank kernel where it applies, else the tensor-core kernel
 *          where T*k/E >= 256 or T*k >= 2048, and the CUDA-core kernel
 *          otherwise.
 * T == 0 is a no-op.  Empty segments are legal.
 * ---------------------------------------------------------------------- */
apr_status apr_sgmm_shrink_expand(const void* x, int d_in, const apr_proj* projs, int nproj,
                                  int dtype, int T, int k, int E, const int32_t* ranks,
                                  int max_rank, const int32_t* idx, const float* gate,
                                  const int32_t* seg_off, const int32_t* perm, void* ws,
                                  size_t ws_bytes, int kernel, void* stream);

/* One projection of a fused base + adapter group. */
typedef struct apr_linear_proj {
  const void* W;          /* device [d_out, d_in] bf16 base weight (never written)    */
  void* y;                /* device [T, d_out] bf16 out (written once, never read)     */
  int d_out;              /* output width, a multiple of 8                             */
  const void* const* A;   /* device array [E] of device pointers, A[e] -> [r_e, d_in]  */
  const void* const* B;   /* device array [E] of device pointers, B[e] -> [d_out, r_e] */
} apr_linear_proj;

/* ------------------------------------------------------------------------
 * Base projection and adapters in one contraction (section 2.B: the selected
 * experts are fused into the backbone in a single pass).  For every
 * projection p of the group and every token t:
 *   y_p[t] = x[t] W_p^T + sum_j gate[t,j] * B_e (A_e x[t]),  e = idx[t,j]
 * with fp32 accumulation of both terms in one accumulator and one rounding to
 * bf16 per output element; y is written once and never read (no base output
 * is read back and rewritten).
 * Inputs as for apr_sgmm_shrink_expand (x shared by the group, the routing of
 * apr_pregate_route, the segments of apr_segment_tokens written into the same
 * `ws`).  bf16 only.  Needs, with R16 = max_rank rounded up to 16: R16 in
 * {16, 32, 64}, k <= 4, k * R16 <= 64, E * R16 <= 256, d_in % 64 == 0, and
 * every W, y and x 16-byte aligned; APR_ERR_UNSUPPORTED otherwise.
 * ws must hold apr_linear_workspace_size(...) bytes for this group.
 * T == 0 is a no-op.  Device faults (an index >= E, a bad rank, a wait that
 * expires) are recorded in ws and reported by apr_stream_status.
 * ---------------------------------------------------------------------- */
apr_status apr_linear_lora(const void* x, int d_in, const apr_linear_proj* projs, int nproj, int T,
                           int k, int E, const int32_t* ranks, int max_rank, const int32_t* idx,
                           const float* gate, const int32_t* seg_off, const int32_t* perm, void* ws,
                           size_t ws_bytes, void* stream);

/* Workspace bytes for apr_linear_lora on up to T tokens with nproj projections
 * whose output widths add up to at most sum_d_out (also enough for every other
 * call on these maxima).  0 if an argument is out of range. */
size_t apr_linear_workspace_size(int T, int k, int E, int max_rank, int max_d_in, int nproj,
                                 long sum_d_out);

/* ------------------------------------------------------------------------
 * Adapter paging (the Chameleon page: adapters loaded on demand, the popular
 * ones kept resident in an adaptive cache, as in S-LoRA).  n_adapters adapters
 * live in pinned host memory, each one contiguous buffer of adapter_bytes
 * holding its A and B matrices of every (layer, projection) at fixed offsets;
 * n_slots device slots (a caller-owned pool of n_slots * adapter_bytes) hold
 * the ones a step selects.  The SGMM calls keep taking device tables of A and
 * B pointers indexed by adapter id (E = n_adapters); paging rewrites the
 * entries of the adapters it brings in.
 * apr_adapter_pool_state_bytes  device bytes of the pool's state (0 if an
 *      argument is outside [1, APR_MAX_E]).
 * apr_adapter_pool_init  host_src: HOST array [n_adapters] of the adapters'
 *      buffers, each 16-byte aligned pinned host memory that the device reads
 *      at the same address (checked: APR_ERR_INVALID_ARG otherwise);
 *      host_src_table: device array [n_adapters] the call fills with them.
 *      Empties every slot, zeroes the pool and points every entry of every
 *      table at slot 0's copy: the dense and bank SGMM kernels read the whole
 *      adapter bank (a zero gate removes the adapters a token did not
 *      select), so an entry must always point at finite data in the pool.
 *      offsets: device array [ntab], read once here (multiples of 16 below
 *      adapter_bytes).  Synchronises `stream` (set-up call).
 * apr_adapter_pool_page_in  after the router, before the step's SGMM calls:
 *      every adapter idx [T, k] selects becomes resident (empty slots first,
 *      then the least recently used slots this step does not need), copied
 *      from its host buffer by a kernel, and for each of the ntab tables
 *      (device array `tables`, each a device array [n_adapters] of pointers)
 *      its entry becomes pool + slot * adapter_bytes + offsets[t] (device
 *      array [ntab], multiples of 16 below adapter_bytes).  Asynchronous, no
 *      host round trip.  More distinct adapters in idx than slots:
 *      APR_ERR_WORKSPACE from apr_stream_status and nothing changes.  The
 *      entries of adapters not resident keep pointing at a copy in the pool
 *      (another adapter's or zeros): kernels that read the whole bank get
 *      finite data, which the zero gates of those adapters remove.  Nothing
 *      after the copy starts before it is complete (the copy kernel does not
 *      release its dependents early), since the SGMM kernels may read
 *      adapter weights before their own dependency wait.
 * ---------------------------------------------------------------------- */
size_t apr_adapter_pool_state_bytes(int n_adapters, int n_slots);
apr_status apr_adapter_pool_init(void* state, size_t state_bytes, int n_adapters, int n_slots,
                                 const void* const* host_src, size_t adapter_bytes,
                                 void* host_src_table, void* pool, size_t pool_bytes,
                                 const uint64_t* offsets, void* const* tables, int ntab,
                                 void* stream);
apr_status apr_adapter_pool_page_in(void* state, size_t state_bytes, int n_adapters, int n_slots,
                                    const int32_t* idx, int T, int k,
                                    const void* const* host_src_table, size_t adapter_bytes,
                                    void* pool, size_t pool_bytes, const uint64_t* offsets,
                                    void* const* tables, int ntab, void* ws, size_t ws_bytes,
                                    void* stream);

/* One weight of the merge step. */
typedef struct apr_merge_proj {
  const void* W;          /* device [d_out, d_in] bf16 base weight (never written) */
  void* Wp;               /* device [d_out, d_in] bf16 merged weight, out         */
  int d_in, d_out;        /* multiples of 8                                       */
  const void* const* A;   /* device array [E] of device pointers, A[e] -> [r, d_in]  */
  const void* const* B;   /* device array [E] of device pointers, B[e] -> [d_out, r] */
} apr_merge_proj;

/* ------------------------------------------------------------------------
 * Batch-1 merge (section 2.B steps 3 and 5), all weights in ONE launch:
 *   Wp = W + sum_j gate[j] * B_{idx[j]} A_{idx[j]}
 * written out of place, so W is never modified and unmerging is free.
 * projs    device [nproj] apr_merge_proj
 * r        rank shared by the merged adapters (multiple of 8, <= 64)
 * idx,gate device [k]: one token's pre-gate (row 0 of apr_pregate_route)
 * fp32 accumulation, one rounding to bf16 per element.
 * ---------------------------------------------------------------------- */
apr_status apr_merge_adapters(const apr_merge_proj* projs, int nproj, int E, int r,
                              const int32_t* idx, const float* gate, int k, void* ws,
                              size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * In-place merge and exact unmerge (section 2.B steps 3 and 5: merge the
 * token's adapters, run the base model, unmerge for the next token), all
 * weights in one launch each, without a second copy of W.
 * apr_merge_adapters_inplace  W <- rn(W + sum_j gate[j] B_{idx[j]} A_{idx[j]}),
 *      the same values as apr_merge_adapters writes to Wp, bit for bit.  For
 *      this call projs[p].Wp is NOT a weight: it receives the residual codes
 *      that make the unmerge exact, one byte per element in a tiled layout of
 *      its own (device, caller-owned, 16-byte aligned,
 *      apr_merge_residual_bytes(d_out, d_in) bytes).
 * apr_unmerge_adapters_inplace  restores every W bit for bit from W', the
 *      residual codes and `escapes`, recomputing the same delta: idx and gate
 *      must be the merge's (checked on the device: APR_ERR_INVALID_ARG from
 *      apr_stream_status, and no weight is touched, otherwise).
 * escapes  device, caller-owned, 16-byte aligned, apr_merge_escape_bytes(c)
 *      bytes for c escapes: elements whose restoring distance does not fit a
 *      code (typically |W| far below the delta) keep their exact bits there.
 *      When more than c are needed, the excess elements are left unmerged (so
 *      the unmerge is still exact) and the merge reports APR_ERR_WORKSPACE.
 * Needs k * round16(r) <= 64 (APR_ERR_UNSUPPORTED otherwise).  Between the
 * two calls neither W nor the codes nor `escapes` may change.
 * ---------------------------------------------------------------------- */
size_t apr_merge_escape_bytes(long capacity);
size_t apr_merge_residual_bytes(int d_out, int d_in);
apr_status apr_merge_adapters_inplace(const apr_merge_proj* projs, int nproj, int E, int r,
                                      const int32_t* idx, const float* gate, int k, void* escapes,
                                      size_t escape_bytes, void* ws, size_t ws_bytes, void* stream);
apr_status apr_unmerge_adapters_inplace(const apr_merge_proj* projs, int nproj, int E, int r,
                                        const int32_t* idx, const float* gate, int k, void* escapes,
                                        size_t escape_bytes, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Merge plan: TMA descriptors of every weight pair (W, Wp).  The weights'
 * addresses and shapes do not change from one token to the next, so a plan is
 * built once for a set of weights and then used by every
 * apr_merge_adapters_planned, which streams W in and Wp out with TMA copies
 * (the same result as apr_merge_adapters, bit for bit).
 * apr_merge_plan_size  device bytes of a plan for nproj weights (0 if nproj is
 *                      outside [1, 4096])
 * apr_merge_plan_init  projs: HOST array [nproj], the same entries as the device
 *                      table later given to the merge; plan: device memory of
 *                      apr_merge_plan_size(nproj) bytes, 128-byte aligned, owned by
 *                      the caller.  W and Wp must be 16-byte aligned and d_in a
 *                      multiple of 8.  A set-up call: it encodes on the host and
 *                      copies synchronously (no stream).
 * apr_merge_adapters_planned  as apr_merge_adapters, with the plan of the same
 *                      weights in the same order; needs k * round16(r) <= 64
 *                      (APR_ERR_UNSUPPORTED otherwise).
 * ---------------------------------------------------------------------- */
size_t apr_merge_plan_size(int nproj);
apr_status apr_merge_plan_init(const apr_merge_proj* projs, int nproj, void* plan, size_t plan_bytes);
apr_status apr_merge_adapters_planned(const apr_merge_proj* projs, const void* plan, int nproj, int E, int r,
                                      const int32_t* idx, const float* gate, int k, void* ws, size_t ws_bytes,
                                      void* stream);

/* ------------------------------------------------------------------------
 * Base inference on the merged weight (section 2.B step 4): y = W x.
 * W device [d_out, d_in] bf16, x device [d_in] bf16, y device [d_out] bf16.
 * fp32 accumulation, one rounding per output.
 * ---------------------------------------------------------------------- */
apr_status apr_gemv(const void* W, const void* x, void* y, int d_in, int d_out, void* stream);

/* ------------------------------------------------------------------------
 * Status plumbing.
 * apr_stream_status: synchronizes `stream`, then reads and clears the device
 *   error word of `ws`; returns APR_OK, the first device-side error recorded
 *   since the last call, or APR_ERR_CUDA if the stream itself failed.
 * apr_last_error: thread-local text of the last non-OK status of this thread.
 * apr_status_string: fixed name of a status code.
 * apr_kernel_launches: number of kernels this library has launched in the
 *   process (all threads), for accounting.
 * ---------------------------------------------------------------------- */
apr_status apr_stream_status(void* ws, void* stream);
const char* apr_last_error(void);
const char* apr_status_string(int status);
uint64_t apr_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* APR_H_ */
