// Host side of the C ABI declared in include/apr.h: argument checks, workspace
// layout, dispatch to the kernel launchers, status plumbing.  Nothing here
// allocates device memory.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include <vector>

#include "apr_internal.cuh"

namespace apr {

static thread_local char g_err[512] = "";
static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

cudaError_t SmemLimit::ensure(const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices)
    return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  std::lock_guard<std::mutex> lock(mu);
  if (bytes <= done[dev]) return cudaSuccess;
  err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (err == cudaSuccess) done[dev] = bytes;
  return err;
}

int device_sm_count() {
  static std::mutex mu;
  static int cached[kMaxDevices] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] > 0) return cached[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
    return n;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  return n;
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

bool merge_supported(int k, int r, int nproj);

static apr_status fail(apr_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

static apr_status cuda_fail(cudaError_t e, const char* where) {
  return fail(APR_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static apr_status check_ws(void* ws, size_t ws_bytes, size_t need, const char* who) {
  if (ws == nullptr) return fail(APR_ERR_WORKSPACE, "%s: workspace is NULL", who);
  if (reinterpret_cast<uintptr_t>(ws) % kAlign)
    return fail(APR_ERR_WORKSPACE, "%s: workspace must be %zu-byte aligned", who, kAlign);
  if (ws_bytes < need)
    return fail(APR_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", who, ws_bytes, need);
  return APR_OK;
}

static apr_status check_route_dims(int T, int k, int E, const char* who) {
  if (T < 0) return fail(APR_ERR_INVALID_ARG, "%s: T=%d < 0", who, T);
  if (E < 1 || E > APR_MAX_E) return fail(APR_ERR_INVALID_ARG, "%s: E=%d outside [1, %d]", who, E, APR_MAX_E);
  if (k < 1 || k > E || k > APR_MAX_K)
    return fail(APR_ERR_INVALID_ARG, "%s: k=%d outside [1, min(E, %d)]", who, k, APR_MAX_K);
  if ((long)T * k > (1L << 30)) return fail(APR_ERR_UNSUPPORTED, "%s: T*k too large", who);
  return APR_OK;
}

}  // namespace apr

using namespace apr;

extern "C" {

size_t apr_workspace_size(int T, int k, int E, int max_rank, int max_d_in) {
  if (T < 0 || k < 1 || k > APR_MAX_K || E < 1 || E > APR_MAX_E || max_rank < 8 ||
      max_rank > APR_MAX_RANK || (max_rank & 7) || max_d_in < 8 || (max_d_in & 7))
    return 0;
  const WsLayout L = ws_layout(T, k, E);
  size_t scratch = route_scratch_bytes(T, E);
  const size_t sg = sgmm_scratch_bytes(T, k, E, max_rank, max_d_in);
  if (sg > scratch) scratch = sg;
  return L.scratch + align_up(scratch) + kAlign;
}

size_t apr_linear_workspace_size(int T, int k, int E, int max_rank, int max_d_in, int nproj, long sum_d_out) {
  const size_t base = apr_workspace_size(T, k, E, max_rank, max_d_in);
  if (base == 0 || nproj < 1 || nproj > APR_MAX_PROJ || sum_d_out < 8 || sum_d_out > (1L << 30)) return 0;
  const WsLayout L = ws_layout(T, k, E);
  const size_t lin = L.scratch + align_up(linear_scratch_bytes(T, k, E, max_rank, nproj, sum_d_out, max_d_in)) + kAlign;
  return lin > base ? lin : base;
}

apr_status apr_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < sizeof(WsHeader)) return fail(APR_ERR_WORKSPACE, "workspace_init: too small");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(APR_ERR_WORKSPACE, "workspace_init: misaligned");
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "workspace_init");
  return APR_OK;
}

apr_status apr_pregate_route(const void* h, const void* Wr, int dtype, int T, int d, int E, int k,
                             int32_t* idx, float* gate, void* ws, size_t ws_bytes, void* stream) {
  apr_status st = check_route_dims(T, k, E, "pregate_route");
  if (st) return st;
  if (dtype != APR_F32 && dtype != APR_BF16) return fail(APR_ERR_INVALID_ARG, "pregate_route: bad dtype %d", dtype);
  if (d < 8 || (d & 7)) return fail(APR_ERR_INVALID_ARG, "pregate_route: d=%d must be a positive multiple of 8", d);
  if (T == 0) return APR_OK;
  if (!h || !Wr || !idx || !gate) return fail(APR_ERR_INVALID_ARG, "pregate_route: NULL pointer");
  if (!aligned16(h) || !aligned16(Wr)) return fail(APR_ERR_INVALID_ARG, "pregate_route: h/Wr not 16-byte aligned");
  const WsLayout L = ws_layout(T, k, E);
  st = check_ws(ws, ws_bytes, L.scratch + route_scratch_bytes(T, E), "pregate_route");
  if (st) return st;
  cudaError_t e = launch_route(h, Wr, dtype, T, d, E, k, idx, gate, ws, L.scratch, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "pregate_route launch");
  return APR_OK;
}

apr_status apr_pregate_route_noalloc(const void* h, const void* Wr, int dtype, int T, int d, int E,
                                     int k, int32_t* idx, float* gate, void* stream) {
  apr_status st = check_route_dims(T, k, E, "pregate_route_noalloc");
  if (st) return st;
  if (dtype != APR_F32 && dtype != APR_BF16) return fail(APR_ERR_INVALID_ARG, "pregate_route_noalloc: bad dtype %d", dtype);
  if (d < 8 || (d & 7)) return fail(APR_ERR_INVALID_ARG, "pregate_route_noalloc: d=%d must be a positive multiple of 8", d);
  if (T == 0) return APR_OK;
  if (!h || !Wr || !idx || !gate) return fail(APR_ERR_INVALID_ARG, "pregate_route_noalloc: NULL pointer");
  if (!aligned16(h) || !aligned16(Wr)) return fail(APR_ERR_INVALID_ARG, "pregate_route_noalloc: h/Wr not 16-byte aligned");
  if ((size_t)T * E > route_noalloc_capacity_floats())
    return fail(APR_ERR_UNSUPPORTED, "pregate_route_noalloc: T*E=%zu exceeds the fixed scratch (%zu)",
                (size_t)T * E, route_noalloc_capacity_floats());
  cudaError_t e = launch_route_noalloc(h, Wr, dtype, T, d, E, k, idx, gate, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "pregate_route_noalloc launch");
  return APR_OK;
}

apr_status apr_segment_tokens(const int32_t* idx, int T, int k, int E, int32_t* seg_off,
                              int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  apr_status st = check_route_dims(T, k, E, "segment_tokens");
  if (st) return st;
  if (!seg_off) return fail(APR_ERR_INVALID_ARG, "segment_tokens: NULL seg_off");
  const WsLayout L = ws_layout(T, k, E);
  st = check_ws(ws, ws_bytes, L.scratch, "segment_tokens");
  if (st) return st;
  if (T > 0 && (!idx || !perm)) return fail(APR_ERR_INVALID_ARG, "segment_tokens: NULL pointer");
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(seg_off, 0, sizeof(int32_t) * (E + 1), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "segment_tokens");
    return APR_OK;
  }
  cudaError_t e = launch_segment(idx, T, k, E, seg_off, perm, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "segment_tokens launch");
  return APR_OK;
}

apr_status apr_sgmm_shrink_expand(const void* x, int d_in, const apr_proj* projs, int nproj,
                                  int dtype, int T, int k, int E, const int32_t* ranks,
                                  int max_rank, const int32_t* idx, const float* gate,
                                  const int32_t* seg_off, const int32_t* perm, void* ws,
                                  size_t ws_bytes, int kernel, void* stream) {
  apr_status st = check_route_dims(T, k, E, "sgmm");
  if (st) return st;
  if (dtype != APR_F32 && dtype != APR_BF16) return fail(APR_ERR_INVALID_ARG, "sgmm: bad dtype %d", dtype);
  if (nproj < 1 || nproj > APR_MAX_PROJ) return fail(APR_ERR_INVALID_ARG, "sgmm: nproj=%d outside [1, %d]", nproj, APR_MAX_PROJ);
  if (!projs) return fail(APR_ERR_INVALID_ARG, "sgmm: NULL projs");
  if (d_in < 8 || (d_in & 7)) return fail(APR_ERR_INVALID_ARG, "sgmm: d_in=%d must be a positive multiple of 8", d_in);
  if (max_rank < 8 || max_rank > APR_MAX_RANK || (max_rank & 7))
    return fail(APR_ERR_INVALID_ARG, "sgmm: max_rank=%d must be a multiple of 8 in [8, %d]", max_rank, APR_MAX_RANK);
  if (kernel < APR_SGMM_AUTO || kernel > APR_SGMM_BANK) return fail(APR_ERR_INVALID_ARG, "sgmm: bad kernel %d", kernel);
  for (int p = 0; p < nproj; ++p) {
    const apr_proj& pj = projs[p];
    if (pj.d_out < 8 || (pj.d_out & 7)) return fail(APR_ERR_INVALID_ARG, "sgmm: proj %d d_out=%d must be a positive multiple of 8", p, pj.d_out);
    if (T > 0 && (!pj.y || !pj.y_base || !pj.A || !pj.B)) return fail(APR_ERR_INVALID_ARG, "sgmm: proj %d has a NULL pointer", p);
    if (T > 0 && (!aligned16(pj.y) || !aligned16(pj.y_base))) return fail(APR_ERR_INVALID_ARG, "sgmm: proj %d y/y_base not 16-byte aligned", p);
  }
  if (T == 0) return APR_OK;
  if (!x || !ranks || !idx || !gate || !seg_off || !perm) return fail(APR_ERR_INVALID_ARG, "sgmm: NULL pointer");
  if (!aligned16(x)) return fail(APR_ERR_INVALID_ARG, "sgmm: x not 16-byte aligned");
  const WsLayout L = ws_layout(T, k, E);
  st = check_ws(ws, ws_bytes, L.scratch + sgmm_scratch_bytes(T, k, E, max_rank, d_in), "sgmm");
  if (st) return st;

  SgmmArgs a;
  memset(&a, 0, sizeof(a));
  a.x = x;
  a.d_in = d_in;
  a.nproj = nproj;
  for (int p = 0; p < nproj; ++p) {
    a.proj[p].y = projs[p].y;
    a.proj[p].y_base = projs[p].y_base;
    a.proj[p].d_out = projs[p].d_out;
    a.proj[p].A = projs[p].A;
    a.proj[p].B = projs[p].B;
  }
  a.T = T;
  a.k = k;
  a.E = E;
  a.ranks = ranks;
  a.max_rank = max_rank;
  a.idx = idx;
  a.gate = gate;
  a.seg_off = seg_off;
  a.perm = perm;
  a.ws = ws;

  int use = kernel;
  if (use == APR_SGMM_AUTO) {
    // by the shapes and the mean pairs per adapter, known on the host without reading the routing
    const double mean_seg = (double)T * k / E;
    if (sgmm_dense_supported(a, dtype)) use = APR_SGMM_DENSE;
    else if (sgmm_bank_supported(a, dtype)) use = APR_SGMM_BANK;
    else if ((mean_seg >= 256.0 || (long)T * k >= 2048) && sgmm_tensor_supported(a, dtype)) use = APR_SGMM_TENSOR;
    else use = APR_SGMM_SKINNY;
  }
  cudaError_t e;
  if (use == APR_SGMM_DENSE) {
    if (!sgmm_dense_supported(a, dtype))
      return fail(APR_ERR_UNSUPPORTED, "sgmm: dense kernel needs bf16, T<=64, E<=16, E*round16(max_rank)<=256");
    e = launch_sgmm_dense(a, L.scratch, (cudaStream_t)stream);
  } else if (use == APR_SGMM_BANK) {
    if (!sgmm_bank_supported(a, dtype))
      return fail(APR_ERR_UNSUPPORTED, "sgmm: bank kernel needs bf16, rank slots of 16/32/64, k<=4, k*R16<=64, "
                                       "E*R16<=256, d_in%%64==0");
    e = launch_sgmm_bank(a, L.scratch, (cudaStream_t)stream);
  } else if (use == APR_SGMM_TENSOR) {
    if (!sgmm_tensor_supported(a, dtype))
      return fail(APR_ERR_UNSUPPORTED, "sgmm: tensor-core kernel needs bf16 and d_in%%64==0, and for k=2 "
                                       "max_rank<=32 and d_out%%16==0");
    e = sgmm_ragged_supported(a, dtype) ? launch_sgmm_ragged(a, L.scratch, (cudaStream_t)stream)
                                        : launch_sgmm_tensor(a, L.scratch, (cudaStream_t)stream);
  } else {
    e = launch_sgmm_skinny(a, dtype, L.scratch, (cudaStream_t)stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "sgmm launch");
  return APR_OK;
}

size_t apr_merge_plan_size(int nproj) {
  if (nproj < 1 || nproj > 4096) return 0;
  return merge_plan_bytes(nproj);
}

apr_status apr_merge_plan_init(const apr_merge_proj* projs, int nproj, void* plan, size_t plan_bytes) {
  if (nproj < 1 || nproj > 4096) return fail(APR_ERR_INVALID_ARG, "merge_plan_init: nproj=%d outside [1, 4096]", nproj);
  if (!projs || !plan) return fail(APR_ERR_INVALID_ARG, "merge_plan_init: NULL pointer");
  if (reinterpret_cast<uintptr_t>(plan) & 127) return fail(APR_ERR_INVALID_ARG, "merge_plan_init: plan not 128-byte aligned");
  if (plan_bytes < merge_plan_bytes(nproj))
    return fail(APR_ERR_WORKSPACE, "merge_plan_init: %zu bytes < %zu needed", plan_bytes, merge_plan_bytes(nproj));
  for (int p = 0; p < nproj; ++p) {
    const apr_merge_proj& m = projs[p];
    if (!m.W || !m.Wp) return fail(APR_ERR_INVALID_ARG, "merge_plan_init: weight %d has a NULL pointer", p);
    if (!aligned16(m.W) || !aligned16(m.Wp)) return fail(APR_ERR_INVALID_ARG, "merge_plan_init: weight %d not 16-byte aligned", p);
    if (m.d_in < 8 || (m.d_in & 7) || m.d_out < 1)
      return fail(APR_ERR_INVALID_ARG, "merge_plan_init: weight %d shape %d x %d (d_in must be a multiple of 8)", p, m.d_out, m.d_in);
  }
  cudaError_t e = merge_plan_build(projs, nproj, plan);
  if (e != cudaSuccess) return cuda_fail(e, "merge_plan_init");
  return APR_OK;
}

apr_status apr_merge_adapters_planned(const apr_merge_proj* projs, const void* plan, int nproj, int E, int r,
                                      const int32_t* idx, const float* gate, int k, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (nproj < 1) return fail(APR_ERR_INVALID_ARG, "merge: nproj=%d < 1", nproj);
  if (E < 1 || E > APR_MAX_E) return fail(APR_ERR_INVALID_ARG, "merge: E=%d outside [1, %d]", E, APR_MAX_E);
  if (k < 1 || k > E || k > APR_MAX_K) return fail(APR_ERR_INVALID_ARG, "merge: k=%d outside [1, min(E, %d)]", k, APR_MAX_K);
  if (r < 8 || (r & 7) || r > APR_MAX_RANK) return fail(APR_ERR_INVALID_ARG, "merge: r=%d must be a multiple of 8 in [8, %d]", r, APR_MAX_RANK);
  if (!merge_tensor_supported(k, r, nproj))
    return fail(APR_ERR_UNSUPPORTED, "merge (planned): needs k * round16(r) <= 64 and nproj <= 4096");
  if (!projs || !plan || !idx || !gate) return fail(APR_ERR_INVALID_ARG, "merge: NULL pointer");
  if (reinterpret_cast<uintptr_t>(plan) & 127) return fail(APR_ERR_INVALID_ARG, "merge: plan not 128-byte aligned");
  apr_status st = check_ws(ws, ws_bytes, sizeof(WsHeader), "merge");
  if (st) return st;
  cudaError_t e = launch_merge_tma(projs, plan, nproj, E, r, idx, gate, k, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return APR_OK;
}

apr_status apr_linear_lora(const void* x, int d_in, const apr_linear_proj* projs, int nproj, int T,
                           int k, int E, const int32_t* ranks, int max_rank, const int32_t* idx,
                           const float* gate, const int32_t* seg_off, const int32_t* perm, void* ws,
                           size_t ws_bytes, void* stream) {
  apr_status st = check_route_dims(T, k, E, "linear_lora");
  if (st) return st;
  if (nproj < 1 || nproj > APR_MAX_PROJ)
    return fail(APR_ERR_INVALID_ARG, "linear_lora: nproj=%d outside [1, %d]", nproj, APR_MAX_PROJ);
  if (!projs) return fail(APR_ERR_INVALID_ARG, "linear_lora: NULL projs");
  if (d_in < 8 || (d_in & 7)) return fail(APR_ERR_INVALID_ARG, "linear_lora: d_in=%d must be a positive multiple of 8", d_in);
  if (max_rank < 8 || max_rank > APR_MAX_RANK || (max_rank & 7))
    return fail(APR_ERR_INVALID_ARG, "linear_lora: max_rank=%d must be a multiple of 8 in [8, %d]", max_rank, APR_MAX_RANK);
  long sum_d_out = 0;
  for (int p = 0; p < nproj; ++p) {
    const apr_linear_proj& pj = projs[p];
    if (pj.d_out < 8 || (pj.d_out & 7))
      return fail(APR_ERR_INVALID_ARG, "linear_lora: proj %d d_out=%d must be a positive multiple of 8", p, pj.d_out);
    if (T > 0 && (!pj.W || !pj.y || !pj.A || !pj.B))
      return fail(APR_ERR_INVALID_ARG, "linear_lora: proj %d has a NULL pointer", p);
    if (T > 0 && (!aligned16(pj.W) || !aligned16(pj.y)))
      return fail(APR_ERR_INVALID_ARG, "linear_lora: proj %d W/y not 16-byte aligned", p);
    sum_d_out += pj.d_out;
  }
  if (T == 0) return APR_OK;
  if (!x || !ranks || !idx || !gate || !seg_off || !perm) return fail(APR_ERR_INVALID_ARG, "linear_lora: NULL pointer");
  if (!aligned16(x)) return fail(APR_ERR_INVALID_ARG, "linear_lora: x not 16-byte aligned");
  const WsLayout L = ws_layout(T, k, E);
  st = check_ws(ws, ws_bytes, L.scratch + linear_scratch_bytes(T, k, E, max_rank, nproj, sum_d_out, d_in), "linear_lora");
  if (st) return st;

  SgmmArgs a;
  memset(&a, 0, sizeof(a));
  const void* W[APR_MAX_PROJ] = {};
  a.x = x;
  a.d_in = d_in;
  a.nproj = nproj;
  for (int p = 0; p < nproj; ++p) {
    a.proj[p].y = projs[p].y;
    a.proj[p].y_base = nullptr;
    a.proj[p].d_out = projs[p].d_out;
    a.proj[p].A = projs[p].A;
    a.proj[p].B = projs[p].B;
    W[p] = projs[p].W;
  }
  a.T = T;
  a.k = k;
  a.E = E;
  a.ranks = ranks;
  a.max_rank = max_rank;
  a.idx = idx;
  a.gate = gate;
  a.seg_off = seg_off;
  a.perm = perm;
  a.ws = ws;
  if (!linear_lora_supported(a))
    return fail(APR_ERR_UNSUPPORTED, "linear_lora: needs rank slots of 16/32/64, k<=4, k*R16<=64, E*R16<=256, "
                                     "d_in%%64==0");
  cudaError_t e = launch_linear_lora(a, W, L.scratch, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "linear_lora launch");
  return APR_OK;
}

apr_status apr_merge_adapters(const apr_merge_proj* projs, int nproj, int E, int r,
                              const int32_t* idx, const float* gate, int k, void* ws,
                              size_t ws_bytes, void* stream) {
  if (nproj < 1) return fail(APR_ERR_INVALID_ARG, "merge: nproj=%d < 1", nproj);
  if (E < 1 || E > APR_MAX_E) return fail(APR_ERR_INVALID_ARG, "merge: E=%d outside [1, %d]", E, APR_MAX_E);
  if (k < 1 || k > E || k > APR_MAX_K) return fail(APR_ERR_INVALID_ARG, "merge: k=%d outside [1, min(E, %d)]", k, APR_MAX_K);
  if (r < 8 || (r & 7) || r > APR_MAX_RANK) return fail(APR_ERR_INVALID_ARG, "merge: r=%d must be a multiple of 8 in [8, %d]", r, APR_MAX_RANK);
  const bool on_tensor = merge_tensor_supported(k, r, nproj);
  if (!on_tensor && !merge_supported(k, r, nproj))
    return fail(APR_ERR_UNSUPPORTED, "merge: k*r=%d > 64 or nproj=%d > 4096", k * r, nproj);
  if (!projs || !idx || !gate) return fail(APR_ERR_INVALID_ARG, "merge: NULL pointer");
  apr_status st = check_ws(ws, ws_bytes, sizeof(WsHeader), "merge");
  if (st) return st;
  cudaError_t e = on_tensor ? launch_merge_tensor(projs, nproj, E, r, idx, gate, k, ws, (cudaStream_t)stream)
                            : launch_merge(projs, nproj, E, r, idx, gate, k, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return APR_OK;
}

size_t apr_merge_escape_bytes(long capacity) { return capacity < 0 ? 0 : merge_escape_bytes(capacity); }
size_t apr_merge_residual_bytes(int d_out, int d_in) {
  return (d_out < 1 || d_in < 8 || (d_in & 7)) ? 0 : merge_residual_bytes(d_out, d_in);
}

static apr_status merge_inplace_call(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                     const float* gate, int k, void* escapes, size_t escape_bytes, void* ws,
                                     size_t ws_bytes, void* stream, bool unmerge) {
  const char* who = unmerge ? "unmerge_inplace" : "merge_inplace";
  if (nproj < 1) return fail(APR_ERR_INVALID_ARG, "%s: nproj=%d < 1", who, nproj);
  if (E < 1 || E > APR_MAX_E) return fail(APR_ERR_INVALID_ARG, "%s: E=%d outside [1, %d]", who, E, APR_MAX_E);
  if (k < 1 || k > E || k > APR_MAX_K) return fail(APR_ERR_INVALID_ARG, "%s: k=%d outside [1, min(E, %d)]", who, k, APR_MAX_K);
  if (r < 8 || (r & 7) || r > APR_MAX_RANK)
    return fail(APR_ERR_INVALID_ARG, "%s: r=%d must be a multiple of 8 in [8, %d]", who, r, APR_MAX_RANK);
  if (!merge_tensor_supported(k, r, nproj))
    return fail(APR_ERR_UNSUPPORTED, "%s: needs k * round16(r) <= 64 and nproj <= 4096", who);
  if (!projs || !idx || !gate || !escapes) return fail(APR_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (escape_bytes < merge_escape_bytes(0) || reinterpret_cast<uintptr_t>(escapes) % 16)
    return fail(APR_ERR_INVALID_ARG, "%s: escape buffer below %zu bytes or not 16-byte aligned", who,
                merge_escape_bytes(0));
  apr_status st = check_ws(ws, ws_bytes, sizeof(WsHeader), who);
  if (st) return st;
  const long capacity = (long)((escape_bytes - merge_escape_bytes(0)) / 12);
  cudaError_t e = launch_merge_inplace(projs, nproj, E, r, idx, gate, k, escapes, capacity, unmerge, ws,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, unmerge ? "unmerge_inplace launch" : "merge_inplace launch");
  return APR_OK;
}

apr_status apr_merge_adapters_inplace(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                      const float* gate, int k, void* escapes, size_t escape_bytes, void* ws,
                                      size_t ws_bytes, void* stream) {
  return merge_inplace_call(projs, nproj, E, r, idx, gate, k, escapes, escape_bytes, ws, ws_bytes, stream, false);
}

apr_status apr_unmerge_adapters_inplace(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                        const float* gate, int k, void* escapes, size_t escape_bytes, void* ws,
                                        size_t ws_bytes, void* stream) {
  return merge_inplace_call(projs, nproj, E, r, idx, gate, k, escapes, escape_bytes, ws, ws_bytes, stream, true);
}

size_t apr_adapter_pool_state_bytes(int n_adapters, int n_slots) {
  if (n_adapters < 1 || n_adapters > APR_MAX_E || n_slots < 1 || n_slots > APR_MAX_E) return 0;
  return adapter_pool_state_bytes(n_adapters, n_slots);
}

apr_status apr_adapter_pool_init(void* state, size_t state_bytes, int n_adapters, int n_slots,
                                 const void* const* host_src, size_t adapter_bytes, void* host_src_table,
                                 void* pool, size_t pool_bytes, const uint64_t* offsets, void* const* tables,
                                 int ntab, void* stream) {
  const size_t need = apr_adapter_pool_state_bytes(n_adapters, n_slots);
  if (need == 0) return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: n_adapters=%d, n_slots=%d outside [1, %d]",
                             n_adapters, n_slots, APR_MAX_E);
  if (!state || state_bytes < need || !aligned16(state))
    return fail(APR_ERR_WORKSPACE, "adapter_pool_init: state NULL, unaligned or below %zu bytes", need);
  if (!host_src || !host_src_table) return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: NULL pointer");
  if (adapter_bytes < 16 || adapter_bytes % 16)
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: adapter_bytes=%zu must be a positive multiple of 16", adapter_bytes);
  if (!pool || !aligned16(pool) || pool_bytes / adapter_bytes < (size_t)n_slots)
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: pool NULL, unaligned or below n_slots * adapter_bytes");
  if (ntab < 0 || (ntab > 0 && (!offsets || !tables)))
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: NULL tables/offsets or ntab=%d < 0", ntab);
  if (ntab > 0) {
    // offsets are read on the host here once (the kernels trust them afterwards)
    std::vector<uint64_t> off((size_t)ntab);
    cudaError_t e = cudaMemcpy(off.data(), offsets, sizeof(uint64_t) * (size_t)ntab, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "adapter_pool_init: reading offsets");
    for (int t = 0; t < ntab; ++t)
      if (off[t] % 16 || off[t] >= adapter_bytes)
        return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: offsets[%d]=%llu not a multiple of 16 below adapter_bytes",
                    t, (unsigned long long)off[t]);
  }
  // every source must be pinned host memory the device reads at the same address
  for (int i = 0; i < n_adapters; ++i) {
    cudaPointerAttributes at;
    if (!host_src[i] || !aligned16(host_src[i]) || cudaPointerGetAttributes(&at, host_src[i]) != cudaSuccess ||
        at.type != cudaMemoryTypeHost || at.devicePointer != host_src[i]) {
      (void)cudaGetLastError();
      return fail(APR_ERR_INVALID_ARG, "adapter_pool_init: host_src[%d] is not 16-byte aligned pinned, mapped host memory", i);
    }
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(host_src_table, host_src, sizeof(void*) * (size_t)n_adapters, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);     // the host array may go once this returns
  if (e == cudaSuccess)
    e = launch_pool_init(state, n_adapters, n_slots, pool, pool_bytes,
                         reinterpret_cast<const unsigned long long*>(offsets), tables, ntab, s);
  if (e != cudaSuccess) return cuda_fail(e, "adapter_pool_init");
  return APR_OK;
}

apr_status apr_adapter_pool_page_in(void* state, size_t state_bytes, int n_adapters, int n_slots,
                                    const int32_t* idx, int T, int k, const void* const* host_src_table,
                                    size_t adapter_bytes, void* pool, size_t pool_bytes,
                                    const uint64_t* offsets, void* const* tables, int ntab, void* ws,
                                    size_t ws_bytes, void* stream) {
  const size_t need = apr_adapter_pool_state_bytes(n_adapters, n_slots);
  if (need == 0) return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: n_adapters=%d, n_slots=%d outside [1, %d]",
                             n_adapters, n_slots, APR_MAX_E);
  if (!state || state_bytes < need || !aligned16(state))
    return fail(APR_ERR_WORKSPACE, "adapter_pool_page_in: state NULL, unaligned or below %zu bytes", need);
  if (T < 0 || k < 1 || k > APR_MAX_K) return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: T=%d, k=%d", T, k);
  if (adapter_bytes < 16 || adapter_bytes % 16)
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: adapter_bytes=%zu must be a positive multiple of 16", adapter_bytes);
  if (!pool || !aligned16(pool) || pool_bytes / adapter_bytes < (size_t)n_slots)
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: pool NULL, unaligned or below n_slots * adapter_bytes");
  if (ntab < 0 || (ntab > 0 && (!offsets || !tables)) || !host_src_table)
    return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: NULL pointer or ntab=%d < 0", ntab);
  if (T > 0 && !idx) return fail(APR_ERR_INVALID_ARG, "adapter_pool_page_in: NULL idx");
  apr_status st = check_ws(ws, ws_bytes, sizeof(WsHeader), "adapter_pool_page_in");
  if (st) return st;
  cudaError_t e = launch_pool_page_in(state, n_adapters, n_slots, idx, T * k, host_src_table, adapter_bytes, pool,
                                      reinterpret_cast<const unsigned long long*>(offsets), tables, ntab, ws,
                                      (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "adapter_pool_page_in launch");
  return APR_OK;
}

apr_status apr_gemv(const void* W, const void* x, void* y, int d_in, int d_out, void* stream) {
  if (d_in < 8 || (d_in & 7)) return fail(APR_ERR_INVALID_ARG, "gemv: d_in=%d must be a positive multiple of 8", d_in);
  if (d_in > 48 * 1024) return fail(APR_ERR_UNSUPPORTED, "gemv: d_in=%d > 49152", d_in);
  if (d_out < 0) return fail(APR_ERR_INVALID_ARG, "gemv: d_out=%d < 0", d_out);
  if (d_out == 0) return APR_OK;
  if (!W || !x || !y) return fail(APR_ERR_INVALID_ARG, "gemv: NULL pointer");
  if (!aligned16(W) || !aligned16(x)) return fail(APR_ERR_INVALID_ARG, "gemv: W/x not 16-byte aligned");
  cudaError_t e = launch_gemv(W, x, y, d_in, d_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
  return APR_OK;
}

apr_status apr_stream_status(void* ws, void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream_status");
  if (ws == nullptr) return APR_OK;
  int words[2] = {0, 0};
  e = cudaMemcpy(words, ws, sizeof(words), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "stream_status read");
  if (words[0] != 0) {
    // clear the error word and its detail
    e = cudaMemset(ws, 0, 2 * sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "stream_status clear");
    return fail((apr_status)words[0], "device reported %s (kernel %d, value %d)",
                apr_status_string(words[0]), (words[1] >> 24) & 0xFF, words[1] & 0xFFFFFF);
  }
  return APR_OK;
}

const char* apr_last_error(void) { return g_err; }

const char* apr_status_string(int s) {
  switch (s) {
    case APR_OK: return "APR_OK";
    case APR_ERR_INVALID_ARG: return "APR_ERR_INVALID_ARG";
    case APR_ERR_UNSUPPORTED: return "APR_ERR_UNSUPPORTED";
    case APR_ERR_WORKSPACE: return "APR_ERR_WORKSPACE";
    case APR_ERR_CUDA: return "APR_ERR_CUDA";
    case APR_ERR_DEVICE_INDEX: return "APR_ERR_DEVICE_INDEX";
    case APR_ERR_TIMEOUT: return "APR_ERR_TIMEOUT";
    default: return "APR_ERR_UNKNOWN";
  }
}

uint64_t apr_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
