// Internal definitions shared by the libapr translation units: workspace
// layout, device error reporting, launch helpers and element conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "../../include/apr.h"

namespace apr {

// ---------------------------------------------------------------- workspace

constexpr size_t kAlign = 256;
constexpr int kPairTile = 32;       // pairs per shrink tile of the skinny kernel
constexpr int kSetTile = 128;       // tokens per tensor-core tile (one adapter set)
constexpr int kShrinkKC = 2048;     // input columns per skinny shrink item (256 threads x 8)
constexpr int kRouteKC = 256;       // minimum router split-K chunk

struct WsHeader {
  int err;          // first device-side apr_status recorded (0 = none)
  int err_info;     // detail (kernel id << 24 | value)
  int n_ptiles;     // shrink pair tiles written by the segment kernel
  int n_stiles;     // tensor-core set tiles written by the segment kernel
  int n_qtiles;     // tensor-core pair tiles (<= 128 pairs of one adapter)
  int n_mtiles;     // tensor-core mixed tiles (<= 128 tokens, <= 4 adapters in all)
  unsigned sched;   // work counter of the tensor-core shrink (reset by the segment kernel and every expand)
  int T, k, E;      // routing the plan was built for
  int gplan;        // set and mixed tiles of the current plan built (the gathered expand's tiles)
  int pad[53];
};
static_assert(sizeof(WsHeader) == 256, "header is one alignment unit");

struct PairTile {   // a run of <= kPairTile consecutive sorted pairs of one adapter
  int e, start, len, pad;
};
struct SetTile {    // a run of <= kSetTile tokens (in set order) sharing one adapter set
  int start, len;
};
constexpr int kMixAdapters = 4;
struct MixTile {    // a run of <= kSetTile tokens (in set order) whose adapters number <= kMixAdapters
  int start, len, nu, pad;
  int u[kMixAdapters];   // the adapters, ascending
};

__host__ __device__ inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

__host__ __device__ inline int max_ptiles(int T, int k, int E) {
  long n = (long)T * k;
  long m = n < E ? n : E;
  return (int)((n + kPairTile - 1) / kPairTile + m + 1);
}

__host__ __device__ inline int max_qtiles(int T, int k, int E) {
  long n = (long)T * k;
  long m = n < E ? n : E;
  return (int)((n + kSetTile - 1) / kSetTile + m + 1);
}

struct WsLayout {
  size_t inv, tok_order, tok_tmp, ptiles, stiles, qtiles, mtiles, scratch;
};

__host__ __device__ inline WsLayout ws_layout(int T, int k, int E) {
  WsLayout L;
  size_t o = align_up(sizeof(WsHeader));
  L.inv = o;       o = align_up(o + sizeof(int) * (size_t)T * k);
  L.tok_order = o; o = align_up(o + sizeof(int) * (size_t)T);
  L.tok_tmp = o;   o = align_up(o + sizeof(int) * (size_t)T);
  L.ptiles = o;    o = align_up(o + sizeof(PairTile) * (size_t)max_ptiles(T, k, E));
  L.stiles = o;    o = align_up(o + sizeof(SetTile) * (size_t)(T + 1));
  L.qtiles = o;    o = align_up(o + sizeof(PairTile) * (size_t)max_qtiles(T, k, E));
  L.mtiles = o;    o = align_up(o + sizeof(MixTile) * (size_t)(T + 2 * (T / kSetTile) + 2));
  L.scratch = o;
  (void)E;
  return L;
}

inline int route_max_chunks(int T, int E) {
  long te = (long)T * E;
  long cap = te > 0 ? (1L << 18) / te : 16;
  if (cap < 1) cap = 1;
  if (cap > 16) cap = 16;
  return (int)cap;
}

inline size_t route_scratch_bytes(int T, int E) {
  return sizeof(float) * (size_t)route_max_chunks(T, E) * T * E;
}

inline int shrink_kchunks(int d_in) { return (d_in + kShrinkKC - 1) / kShrinkKC; }

// Dense small-batch path: up to 64 tokens and an adapter bank of at most 16
// adapters whose rank slots (max rank rounded up to 16) add up to <= 256 rows;
// d_in is split over clusters of 8 (or 16) CTAs x 256 columns.  Limits and
// scratch are sized for clusters of 8, the larger count of partials.
constexpr int kDenseMaxT = 64;
constexpr int kDenseMaxRows = 256;
constexpr int kDenseClusterCols = 8 * 256;
inline int round16i(int v) { return (v + 15) / 16 * 16; }
inline int dense_clusters(int d_in) { return (d_in + kDenseClusterCols - 1) / kDenseClusterCols; }
inline bool dense_dims_ok(int T, int E, int max_rank, int d_in = 0) {
  return T >= 1 && T <= kDenseMaxT && E <= 16 && E * round16i(max_rank) <= kDenseMaxRows &&
         dense_clusters(d_in) <= 8;
}

// Tensor-core path: gated v rows [projection][pair position][2 * R16] bf16
// (hi | lo); k <= 2, k * R16 <= 64.
// After the rows, each shrink CTA's A tensor maps ([CTA][projection], <= 256 CTAs).
constexpr int kTensorMaxK2 = 64;
constexpr int kShrinkMaxCtas = 256;
constexpr size_t kShrinkMapBytes = (size_t)kShrinkMaxCtas * APR_MAX_PROJ * 128;
inline size_t tc_vc_bytes(int T, int k, int max_rank) {
  return align_up((size_t)APR_MAX_PROJ * T * k * 4 * round16i(max_rank));
}
inline size_t tc_scratch_bytes(int T, int k, int max_rank) {
  if (k < 1 || k > 2) return 0;
  const int R16 = round16i(max_rank);
  if (k * R16 > kTensorMaxK2) return 0;
  return tc_vc_bytes(T, k, max_rank) + kShrinkMapBytes;
}

// Bank path (token order over the whole adapter bank): gated v per pair
// [projection][pair q][R16] bf16; R16 in {16, 32, 64}, k <= 4, k * R16 <= 64,
// E * R16 <= 256.
constexpr int kBankMaxKR = 64;
constexpr int kBankMaxRows = 256;
inline size_t bank_vc_bytes(int T, int k, int max_rank) {
  return align_up((size_t)APR_MAX_PROJ * T * k * round16i(max_rank) * 2);
}
inline size_t bank_scratch_bytes(int T, int k, int E, int max_rank) {
  const int R16 = round16i(max_rank);
  if (R16 != 16 && R16 != 32 && R16 != 64) return 0;
  if (k < 1 || k > 4 || k * R16 > kBankMaxKR || E * R16 > kBankMaxRows) return 0;
  return bank_vc_bytes(T, k, max_rank) + kShrinkMapBytes;
}

// Many-tenant path (top-1 routing): ragged tiles of <= kSetTile consecutive plan tokens whose
// adapters number <= kRgSlots and whose rank slots (each rank rounded up to 16) add up to
// <= kRgKmax; an adapter with more tokens than fit goes on in the next tile.  Scratch: gated v
// by plan position [projection][position][R16] bf16, then the tile count and the tiles.
constexpr int kRgSlots = 16;
constexpr int kRgKmax = 256;
struct RgTile {
  int start, len, nu, kt;     // plan positions [start, start + len); adapters; rank rows in all
  short u[kRgSlots];          // the adapters, ascending
  short koff[kRgSlots];       // first rank row of each adapter's slot (multiples of 16)
};
static_assert(sizeof(RgTile) == 80, "ragged tile record");
// A tile closes when it is full (<= ceil(T / 128) times) or when the next adapter does not fit
// (such a tile holds an adapter that starts in it: <= min(E, T) times), plus the last one.
__host__ __device__ inline int rg_max_tiles(int T, int E) {
  return (T + kSetTile - 1) / kSetTile + (E < T ? E : T) + 1;
}
inline bool rg_dims_ok(int k, int max_rank) { return k == 1 && round16i(max_rank) <= 128; }
inline size_t rg_vc_bytes(int T, int max_rank) {
  return align_up((size_t)APR_MAX_PROJ * T * round16i(max_rank) * 2);
}
// After the tiles: each shrink CTA's ring of A tensor maps ([CTA][stage][projection]), then one
// B tensor map per (projection, adapter) for the expand.
constexpr int kRgMaxCtas = 256;
constexpr int kRgMaxStages = 8;
inline size_t rg_amaps_off(int T, int E, int max_rank) {
  return align_up(rg_vc_bytes(T, max_rank) + 16 + 80 * (size_t)rg_max_tiles(T, E));
}
inline size_t rg_bmaps_off(int T, int E, int max_rank) {
  return rg_amaps_off(T, E, max_rank) + (size_t)kRgMaxCtas * kRgMaxStages * APR_MAX_PROJ * 128;
}
inline size_t rg_scratch_bytes(int T, int k, int E, int max_rank) {
  if (!rg_dims_ok(k, max_rank)) return 0;
  return rg_bmaps_off(T, E, max_rank) + (size_t)APR_MAX_PROJ * E * 128;
}

// Shrink partial sums.  Gather paths: [projection][column chunk][sorted pair][rank]
// fp32; dense path: [projection][cluster][token (padded to 16)][adapter * rank slot].
inline size_t sgmm_scratch_bytes(int T, int k, int E, int max_rank, int d_in) {
  size_t b = sizeof(float) * APR_MAX_PROJ * (size_t)shrink_kchunks(d_in) * T * k * max_rank;
  if (dense_dims_ok(T, E, max_rank, d_in)) {
    const size_t d = sizeof(float) * APR_MAX_PROJ * (size_t)dense_clusters(d_in) * round16i(T) * E *
                     round16i(max_rank);
    if (d > b) b = d;
  }
  const size_t t = tc_scratch_bytes(T, k, max_rank);
  if (t > b) b = t;
  const size_t bk = bank_scratch_bytes(T, k, E, max_rank);
  if (bk > b) b = bk;
  const size_t rg = rg_scratch_bytes(T, k, E, max_rank);
  if (rg > b) b = rg;
  return b;
}

// Fused base projection + adapters: gated v per pair [proj][pair][R16] bf16, the bank rows
// V [proj][T][E * R16] bf16, then each projection's Bcat [d_out][E * R16] bf16 (aligned blocks).
struct LinearScratch {
  size_t vc, abank, v, bcat;
};
inline LinearScratch linear_scratch(int T, int k, int E, int max_rank, int nproj, int d_in) {
  const size_t R16 = (size_t)round16i(max_rank);
  LinearScratch L;
  L.vc = 0;
  L.abank = align_up((size_t)nproj * T * k * R16 * 2);
  L.v = L.abank + align_up((size_t)nproj * E * R16 * d_in * 2);
  L.bcat = L.v + align_up((size_t)nproj * T * E * R16 * 2);
  return L;
}
// Bytes for nproj projections whose output widths add up to sum_d_out.
inline size_t linear_scratch_bytes(int T, int k, int E, int max_rank, int nproj, long sum_d_out, int d_in) {
  const LinearScratch L = linear_scratch(T, k, E, max_rank, nproj, d_in);
  return L.bcat + align_up((size_t)sum_d_out * E * round16i(max_rank) * 2) + (size_t)nproj * kAlign;
}

template <typename P>
__host__ __device__ inline P* ws_at(void* ws, size_t off) {
  return reinterpret_cast<P*>(reinterpret_cast<char*>(ws) + off);
}

// ---------------------------------------------------------------- device helpers

// Record the first device-side fault; later ones keep the first code.
__device__ inline void report(void* ws, int code, int kernel_id, int value) {
  WsHeader* h = reinterpret_cast<WsHeader*>(ws);
  if (atomicCAS(&h->err, 0, code) == 0) {
    atomicExch(&h->err_info, (kernel_id << 24) | (value & 0xFFFFFF));
  }
}

// Programmatic dependent launch: wait for the preceding grid on the stream
// (and its memory) before reading inputs; then let the next grid launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Unpack 8 consecutive elements starting at a 16-byte aligned address.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Streaming (evict-first) variant for data read once per step.
__device__ __forceinline__ void load8_stream(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8_stream(const float* p, float (&f)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// Asynchronous 16-byte global -> shared copies (L2 only), grouped and awaited.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Every copy this thread issued has landed, committed to a group or not (cp.async.wait_all;
// "wait_group 0" alone would skip copies not yet committed).
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Kernel ids used in WsHeader::err_info.
enum KernelId { K_ROUTE = 1, K_TOPK = 2, K_SEGMENT = 3, K_SHRINK = 4, K_EXPAND = 5, K_MERGE = 6, K_TC = 7, K_LINEAR = 8, K_POOL = 9 };

}  // namespace apr

// ---------------------------------------------------------------- launchers (host)
namespace apr {

void count_launch();
void set_error(const char* fmt, ...);

// Kernel attributes and device properties are per device, and a process may
// drive several devices from several threads: each record below is kept per
// device ordinal under a lock.
constexpr int kMaxDevices = 64;

// A kernel's raised dynamic shared-memory limit, per device.
struct SmemLimit {
  std::mutex mu;
  size_t done[kMaxDevices] = {};
  // Raise `func`'s limit to at least `bytes` on the current device (once per
  // device and size; devices past kMaxDevices are set on every call).
  cudaError_t ensure(const void* func, size_t bytes);
};

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Launch with programmatic stream serialization allowed (PDL).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Host-side launchers implemented in the kernel translation units.
cudaError_t launch_route(const void* h, const void* Wr, int dtype, int T, int d, int E, int k,
                         int32_t* idx, float* gate, void* ws, size_t scratch_off, cudaStream_t s);
cudaError_t launch_route_noalloc(const void* h, const void* Wr, int dtype, int T, int d, int E, int k,
                                 int32_t* idx, float* gate, cudaStream_t s);
size_t route_noalloc_capacity_floats();
cudaError_t launch_segment(const int32_t* idx, int T, int k, int E, int32_t* seg_off,
                           int32_t* perm, void* ws, cudaStream_t s);
struct ProjArgs {
  void* y;
  const void* y_base;
  int d_out;
  const void* const* A;
  const void* const* B;
};
struct SgmmArgs {
  const void* x;
  int d_in;
  ProjArgs proj[APR_MAX_PROJ];
  int nproj;
  int T, k, E;
  const int32_t* ranks;
  int max_rank;
  const int32_t* idx;
  const float* gate;
  const int32_t* seg_off;
  const int32_t* perm;
  void* ws;
};
cudaError_t launch_sgmm_skinny(const SgmmArgs& a, int dtype, size_t scratch_off, cudaStream_t s);
cudaError_t launch_sgmm_tensor(const SgmmArgs& a, size_t scratch_off, cudaStream_t s);
cudaError_t launch_gather_plan(const int32_t* idx, int T, int k, int E, void* ws, cudaStream_t s);
bool sgmm_ragged_supported(const SgmmArgs& a, int dtype);
cudaError_t launch_sgmm_ragged(const SgmmArgs& a, size_t scratch_off, cudaStream_t s);

cudaError_t launch_sgmm_dense(const SgmmArgs& a, size_t scratch_off, cudaStream_t s);
cudaError_t launch_sgmm_bank(const SgmmArgs& a, size_t scratch_off, cudaStream_t s);
bool sgmm_bank_supported(const SgmmArgs& a, int dtype);
bool linear_lora_supported(const SgmmArgs& a);
bool route_tc_supported(int dtype, int d, int E, const void* h, const void* Wr);
cudaError_t launch_route_tc(const void* h, const void* Wr, int T, int d, int E, int k, int32_t* idx, float* gate,
                            void* ws, cudaStream_t s);
size_t adapter_pool_state_bytes(int n_adapters, int n_slots);
cudaError_t launch_pool_init(void* state, int n_adapters, int n_slots, void* pool, size_t pool_bytes,
                             const unsigned long long* offsets, void* const* tables, int ntab, cudaStream_t s);
cudaError_t launch_pool_page_in(void* state, int n_adapters, int n_slots, const int32_t* idx, int nq,
                                const void* const* host_src, size_t adapter_bytes, void* pool,
                                const unsigned long long* offsets, void* const* tables, int ntab, void* ws,
                                cudaStream_t s);
cudaError_t launch_linear_lora(const SgmmArgs& a, const void* const* W, size_t scratch_off, cudaStream_t s);
// The bank shrink of the fused call: gated v per pair [proj][t * k + j][R16] at vc_off from one
// GEMM of x with each projection's adapter bank, packed at abank_off.
cudaError_t launch_bank_shrink(const SgmmArgs& a, size_t vc_off, size_t abank_off, cudaStream_t s);
bool sgmm_dense_supported(const SgmmArgs& a, int dtype);
bool sgmm_tensor_supported(const SgmmArgs& a, int dtype);
cudaError_t launch_merge(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                         const float* gate, int k, void* ws, cudaStream_t s);
bool merge_tensor_supported(int k, int r, int nproj);
size_t merge_escape_bytes(long capacity);
size_t merge_residual_bytes(int d_out, int d_in);
cudaError_t launch_merge_inplace(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                 const float* gate, int k, void* escapes, long capacity, bool unmerge, void* ws,
                                 cudaStream_t s);
cudaError_t launch_merge_tensor(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                const float* gate, int k, void* ws, cudaStream_t s);
size_t merge_plan_bytes(int nproj);
cudaError_t merge_plan_build(const apr_merge_proj* projs, int nproj, void* plan);
cudaError_t launch_merge_tma(const apr_merge_proj* projs, const void* plan, int nproj, int E, int r,
                             const int32_t* idx, const float* gate, int k, void* ws, cudaStream_t s);
cudaError_t launch_gemv(const void* W, const void* x, void* y, int d_in, int d_out, cudaStream_t s);

}  // namespace apr
