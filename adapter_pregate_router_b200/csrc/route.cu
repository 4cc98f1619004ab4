// Token-level pre-gate: router logits, warp-level top-k and gates.
//
// AdaFuse summary (gist.science), Resumen tecnico §2.A: a single light router
// at the first adapted layer fixes each token's adapters for all later
// layers; §2.B steps 1-2: one router pass per token, then Top-K selection.
//
// bf16 inputs and at most 256 adapters: one launch on the tensor cores
// (launch_route_tc: the tile GEMM of h and Wr, with top-k and gates in its
// epilogue; the logits of bf16 inputs are exact in fp32 accumulation whatever
// the summation order, for the integer-valued inputs the checks use).
// Otherwise two launches:
//   route_logits_kernel  split-K tiled product L = h Wr^T in fp32 (CUDA cores;
//                        partial sums per K chunk, no atomics, so the result
//                        does not depend on scheduling).  The router is tiny
//                        next to the per-layer SGMM; exactness of integer-valued
//                        inputs matters more here than tensor-core speed.
//   route_topk_kernel    one warp per token: sums the chunk partials in a fixed
//                        order, k rounds of warp-shuffle argmax with the
//                        lower index winning ties, softmax over the k winners.
#include <math.h>

#include <mutex>

#include "apr_internal.cuh"

namespace apr {

constexpr int RT_M = 64;   // tokens per tile
constexpr int RT_N = 64;   // adapters per tile
constexpr int RT_K = 32;   // k step

template <typename In>
__global__ void __launch_bounds__(256) route_logits_kernel(const In* __restrict__ h,
                                                           const In* __restrict__ Wr, int T, int d,
                                                           int E, int chunk,
                                                           float* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float hs[RT_K][RT_M + 4];
  __shared__ __align__(16) float wsm[RT_K][RT_N + 4];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * RT_M, e0 = blockIdx.y * RT_N, c = blockIdx.z;
  const int kbeg = c * chunk;
  const int kend = min(d, kbeg + chunk);
  const int tx = tid & 15, ty = tid >> 4;     // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int lrow = tid >> 2, lcol = (tid & 3) * 8;  // loader: 64 rows x 4 vectors of 8
  for (int k0 = kbeg; k0 < kend; k0 += RT_K) {
    float f[8];
    const int kc = k0 + lcol;
    if (t0 + lrow < T && kc < kend) {
      load8(h + (size_t)(t0 + lrow) * d + kc, f);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) hs[lcol + i][lrow] = f[i];
    if (e0 + lrow < E && kc < kend) {
      load8(Wr + (size_t)(e0 + lrow) * d + kc, f);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) wsm[lcol + i][lrow] = f[i];
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < RT_K; ++kk) {
      float4 a = *reinterpret_cast<const float4*>(&hs[kk][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&wsm[kk][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = part + (size_t)c * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j];
    }
  }
}

constexpr int TOPK_PER_LANE = APR_MAX_E / 32;

__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ part, int nch,
                                                         int T, int E, int k,
                                                         int32_t* __restrict__ idx,
                                                         float* __restrict__ gate, void* ws) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[TOPK_PER_LANE];
#pragma unroll
  for (int i = 0; i < TOPK_PER_LANE; ++i) {
    const int e = lane + 32 * i;
    float s = 0.f;
    if (e < E) {
      for (int c = 0; c < nch; ++c) s += part[((size_t)c * T + t) * E + e];
    }
    v[i] = s;
  }
  unsigned chosen = 0u;  // bit i: element lane + 32 i already selected
  float sel_v[APR_MAX_K];
  int sel_e[APR_MAX_K];
#pragma unroll
  for (int j = 0; j < APR_MAX_K; ++j) {
    if (j >= k) break;
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < TOPK_PER_LANE; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((chosen >> i) & 1u)) {
        if (v[i] > bv || (v[i] == bv && e < be)) {
          bv = v[i];
          be = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be == 0x7FFFFFFF) {  // only NaN logits left
      if (lane == 0) report(ws, APR_ERR_DEVICE_INDEX, K_TOPK, t);
      be = 0;
      bv = 0.f;
    }
    if ((be & 31) == lane) chosen |= 1u << (be >> 5);
    sel_v[j] = bv;
    sel_e[j] = be;
  }
  // gates: softmax over the selected logits (the first one is the largest)
  float w[APR_MAX_K];
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < APR_MAX_K; ++j) {
    if (j >= k) break;
    w[j] = expf(sel_v[j] - sel_v[0]);
    sum += w[j];
  }
#pragma unroll
  for (int j = 0; j < APR_MAX_K; ++j) {
    if (j >= k) break;
    if (lane == j) {
      idx[(size_t)t * k + j] = sel_e[j];
      gate[(size_t)t * k + j] = w[j] / sum;
    }
  }
}

cudaError_t launch_route(const void* h, const void* Wr, int dtype, int T, int d, int E, int k,
                         int32_t* idx, float* gate, void* ws, size_t scratch_off, cudaStream_t s) {
  // bf16 banks of up to 256 adapters: logits, top-k and gates in one tensor-core launch
  if (route_tc_supported(dtype, d, E, h, Wr)) return launch_route_tc(h, Wr, T, d, E, k, idx, gate, ws, s);
  const int tiles_t = (T + RT_M - 1) / RT_M;
  const int tiles_e = (E + RT_N - 1) / RT_N;
  const int tiles = tiles_t * tiles_e;
  int nch = (2 * 148 + tiles - 1) / tiles;
  int by_k = d / kRouteKC;
  if (by_k < 1) by_k = 1;
  if (nch > by_k) nch = by_k;
  if (nch > route_max_chunks(T, E)) nch = route_max_chunks(T, E);
  if (nch < 1) nch = 1;
  int chunk = (d + nch - 1) / nch;
  chunk = (chunk + RT_K - 1) / RT_K * RT_K;
  nch = (d + chunk - 1) / chunk;
  float* part = ws_at<float>(ws, scratch_off);
  cudaError_t err;
  dim3 grid(tiles_t, tiles_e, nch);
  if (dtype == APR_BF16) {
    err = launch_pdl(route_logits_kernel<__nv_bfloat16>, grid, dim3(256), 0, s,
                     (const __nv_bfloat16*)h, (const __nv_bfloat16*)Wr, T, d, E, chunk, part);
  } else {
    err = launch_pdl(route_logits_kernel<float>, grid, dim3(256), 0, s, (const float*)h,
                     (const float*)Wr, T, d, E, chunk, part);
  }
  if (err != cudaSuccess) return err;
  const int warps_per_block = 8;
  dim3 g2((T + warps_per_block - 1) / warps_per_block);
  return launch_pdl(route_topk_kernel, g2, dim3(32 * warps_per_block), 0, s, (const float*)part,
                    nch, T, E, k, idx, gate, ws);
}


// ---------------------------------------------------------------- no-allocation variant
//
// apr_pregate_route_noalloc serves callers that cannot hand the library a
// workspace: code with no device allocator of its own (a plug-in whose host
// application owns every byte of device memory, or a latency-critical loop in
// which cudaMalloc and the device-wide synchronisation it can cause are not
// acceptable).  Its scratch is the file-scope array below: a 256-byte header
// (the device error word) followed by the split-K partial logits of one call.
// Every GPU that loads the library keeps these 8 MiB until the process exits.
// All calls share the array, so calls that overlap on the GPU (different
// streams without ordering) race on it.

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr size_t kNoAllocHeaderBytes = 256;
static __device__ __align__(256) unsigned char g_route_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  Looked up once
// per device (with that device current) on the first call there.
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

size_t route_noalloc_capacity_floats() { return (kNoAllocScratchBytes - kNoAllocHeaderBytes) / sizeof(float); }

cudaError_t launch_route_noalloc(const void* h, const void* Wr, int dtype, int T, int d, int E, int k,
                                 int32_t* idx, float* gate, cudaStream_t s) {
  void* base = nullptr;
  cudaError_t err = noalloc_scratch(&base);
  if (err != cudaSuccess) return err;
  const size_t cap = route_noalloc_capacity_floats();
  const size_t te = (size_t)T * E;
  // the error word must start at zero; the partial sums are fully overwritten
  err = cudaMemsetAsync(base, 0, kNoAllocHeaderBytes, s);
  if (err != cudaSuccess) return err;
  const int tiles_t = (T + RT_M - 1) / RT_M;
  const int tiles_e = (E + RT_N - 1) / RT_N;
  const int tiles = tiles_t * tiles_e;
  int nch = (2 * 148 + tiles - 1) / tiles;
  int by_k = d / kRouteKC;
  if (by_k < 1) by_k = 1;
  if (nch > by_k) nch = by_k;
  if (nch > route_max_chunks(T, E)) nch = route_max_chunks(T, E);
  if ((size_t)nch * te > cap) nch = (int)(cap / te);
  if (nch < 1) nch = 1;
  int chunk = (d + nch - 1) / nch;
  chunk = (chunk + RT_K - 1) / RT_K * RT_K;
  nch = (d + chunk - 1) / chunk;
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kNoAllocHeaderBytes);
  dim3 grid(tiles_t, tiles_e, nch);
  if (dtype == APR_BF16) {
    err = launch_pdl(route_logits_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, (const __nv_bfloat16*)h,
                     (const __nv_bfloat16*)Wr, T, d, E, chunk, part);
  } else {
    err = launch_pdl(route_logits_kernel<float>, grid, dim3(256), 0, s, (const float*)h, (const float*)Wr, T,
                     d, E, chunk, part);
  }
  if (err != cudaSuccess) return err;
  const int warps_per_block = 8;
  dim3 g2((T + warps_per_block - 1) / warps_per_block);
  return launch_pdl(route_topk_kernel, g2, dim3(32 * warps_per_block), 0, s, (const float*)part, nch, T, E, k,
                    idx, gate, base);
}

}  // namespace apr
