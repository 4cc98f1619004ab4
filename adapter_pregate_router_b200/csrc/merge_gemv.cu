// Batch-1 merge path.  AdaFuse summary (gist.science), Resumen tecnico §2.B
// decoding steps 3-5: the selected adapters are fused into the backbone in
// one pass, the base model runs, and the adapters are unfused for the next
// token.  Here the merged weight is written out of place
//   Wp = W + sum_j g_j B_{e_j} A_{e_j}
// for every weight of the model in ONE launch (a persistent grid walks all
// (weight, 32 x 256 tile) items), so W is never modified and unmerging is
// free.  The rank-(k*r) update is accumulated in fp32 on CUDA cores with the
// gate-scaled B rows broadcast from shared memory; W and Wp stream with
// 4-byte-per-lane coalesced accesses.
//
// apr_gemv: y = W x for the merged weight, a streaming HBM-bound kernel: each
// warp owns one row with eight 128-bit evict-first loads of W in flight per
// lane, x staged in shared memory, warp-shuffle reduction.
#include "apr_internal.cuh"

namespace apr {

constexpr int MG_THREADS = 128;
constexpr int MG_ROWS = 32;
constexpr int MG_COLS = 2 * MG_THREADS;   // two columns per thread
constexpr int MG_MAXKR = 64;              // k * r handled per launch
constexpr int MG_MAXPROJ = 4096;

__global__ void __launch_bounds__(MG_THREADS) merge_kernel(const apr_merge_proj* __restrict__ projs,
                                                           int nproj, int E, int r,
                                                           const int32_t* __restrict__ idx,
                                                           const float* __restrict__ gate, int k,
                                                           void* ws) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_pref[];                 // [nproj + 1] tile prefix
  __shared__ __align__(16) float s_gb[MG_ROWS][MG_MAXKR + 4];
  __shared__ int s_e[APR_MAX_K];
  __shared__ float s_g[APR_MAX_K];
  __shared__ int s_bad;
  __shared__ int s_carry;
  const int tid = threadIdx.x;
  const int kr = k * r;
  if (tid == 0) {
    s_bad = 0;
    s_carry = 0;
  }
  __syncthreads();
  if (tid < k) {
    const int e = idx[tid];
    if (e < 0 || e >= E) s_bad = 1;
    s_e[tid] = e;
    s_g[tid] = gate[tid];
  }
  // tiles per weight, prefix over the weights (chunks of MG_THREADS)
  for (int base = 0; base < nproj; base += MG_THREADS) {
    const int p = base + tid;
    int nt = 0;
    if (p < nproj) {
      const int di = projs[p].d_in, dout = projs[p].d_out;
      nt = ((dout + MG_ROWS - 1) / MG_ROWS) * ((di + MG_COLS - 1) / MG_COLS);
    }
    // inclusive warp scan, then across the 4 warps
    int x = nt;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    __shared__ int wsum[MG_THREADS / 32];
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = s_carry;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (p < nproj) s_pref[p + 1] = before + x;
    __syncthreads();
    if (tid == MG_THREADS - 1) s_carry = before + x;
    __syncthreads();
  }
  if (tid == 0) s_pref[0] = 0;
  __syncthreads();
  if (s_bad) {
    if (tid == 0 && blockIdx.x == 0) report(ws, APR_ERR_DEVICE_INDEX, K_MERGE, 0);
    return;
  }
  const int total = s_pref[nproj];
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = nproj;          // find p with s_pref[p] <= item < s_pref[p+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pref[mid] <= item) lo = mid; else hi = mid;
    }
    const int p = lo;
    const apr_merge_proj pj = projs[p];
    const int lt = item - s_pref[p];
    const int nct = (pj.d_in + MG_COLS - 1) / MG_COLS;
    const int row0 = (lt / nct) * MG_ROWS, col0 = (lt % nct) * MG_COLS;
    // gate-scaled B rows of this tile: s_gb[row][j*r + i] = g_j * B_{e_j}[row0+row, i]
    for (int w = tid; w < MG_ROWS * kr; w += MG_THREADS) {
      const int row = w / kr, kk = w % kr;
      const int j = kk / r, i = kk % r;
      const int n = row0 + row;
      float v = 0.f;
      if (n < pj.d_out) {
        const __nv_bfloat16* B = reinterpret_cast<const __nv_bfloat16*>(pj.B[s_e[j]]);
        v = s_g[j] * __bfloat162float(B[(size_t)n * r + i]);
      }
      s_gb[row][kk] = v;
    }
    // this thread's two columns of every selected A
    const int c = col0 + 2 * tid;
    const bool active = c < pj.d_in;
    float a0[MG_MAXKR], a1[MG_MAXKR];
#pragma unroll
    for (int kk = 0; kk < MG_MAXKR; ++kk) {
      a0[kk] = 0.f;
      a1[kk] = 0.f;
      if (kk < kr && active) {
        const int j = kk / r, i = kk % r;
        const __nv_bfloat16* A = reinterpret_cast<const __nv_bfloat16*>(pj.A[s_e[j]]);
        const float2 f = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(A + (size_t)i * pj.d_in + c));
        a0[kk] = f.x;
        a1[kk] = f.y;
      }
    }
    __syncthreads();
    const int nrows = min(MG_ROWS, pj.d_out - row0);
    const __nv_bfloat16* W = reinterpret_cast<const __nv_bfloat16*>(pj.W);
    __nv_bfloat16* Wp = reinterpret_cast<__nv_bfloat16*>(pj.Wp);
    if (active) {
#pragma unroll 4
      for (int row = 0; row < nrows; ++row) {
        const size_t off = (size_t)(row0 + row) * pj.d_in + c;
        const float2 w = __bfloat1622float2(__ldcs(reinterpret_cast<const __nv_bfloat162*>(W + off)));
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int kk = 0; kk < MG_MAXKR; kk += 4) {
          if (kk >= kr) break;
          const float4 g = *reinterpret_cast<const float4*>(&s_gb[row][kk]);
          d0 = fmaf(g.x, a0[kk], d0); d1 = fmaf(g.x, a1[kk], d1);
          d0 = fmaf(g.y, a0[kk + 1], d0); d1 = fmaf(g.y, a1[kk + 1], d1);
          d0 = fmaf(g.z, a0[kk + 2], d0); d1 = fmaf(g.z, a1[kk + 2], d1);
          d0 = fmaf(g.w, a0[kk + 3], d0); d1 = fmaf(g.w, a1[kk + 3], d1);
        }
        __stcs(reinterpret_cast<__nv_bfloat162*>(Wp + off), __floats2bfloat162_rn(w.x + d0, w.y + d1));
      }
    }
    __syncthreads();
  }
}

constexpr int GV_THREADS = 256;
constexpr int GV_UNROLL = 8;     // 16-byte loads of W in flight per lane

// One warp per output row: 8 x 128-bit evict-first loads of W in flight per
// lane, x from shared memory, warp-shuffle reduction.
__global__ void __launch_bounds__(GV_THREADS) gemv_kernel(const __nv_bfloat16* __restrict__ W,
                                                          const __nv_bfloat16* __restrict__ x,
                                                          __nv_bfloat16* __restrict__ y, int d_in,
                                                          int d_out) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) __nv_bfloat16 xs[];
  for (int c = threadIdx.x * 8; c < d_in; c += GV_THREADS * 8)
    *reinterpret_cast<uint4*>(xs + c) = *reinterpret_cast<const uint4*>(x + c);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * (GV_THREADS / 32) + warp;
  if (row >= d_out) return;
  const __nv_bfloat16* __restrict__ wr = W + (size_t)row * d_in;
  float acc = 0.f;
  for (int c0 = lane * 8; c0 < d_in; c0 += 256 * GV_UNROLL) {
    uint4 wv[GV_UNROLL];
#pragma unroll
    for (int u = 0; u < GV_UNROLL; ++u) {
      const int c = c0 + u * 256;
      wv[u] = c < d_in ? __ldcs(reinterpret_cast<const uint4*>(wr + c)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < GV_UNROLL; ++u) {
      const int c = c0 + u * 256;
      if (c < d_in) {
        float xv[8];
        load8(xs + c, xv);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&wv[u]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h[i]);
          acc = fmaf(f.x, xv[2 * i], acc);
          acc = fmaf(f.y, xv[2 * i + 1], acc);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) y[row] = __float2bfloat16_rn(acc);
}

cudaError_t launch_merge(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                         const float* gate, int k, void* ws, cudaStream_t s) {
  const int nsm = device_sm_count();
  const size_t smem = sizeof(int) * ((size_t)nproj + 1);
  return launch_pdl(merge_kernel, dim3(nsm * 8), dim3(MG_THREADS), smem, s, projs, nproj, E, r, idx,
                    gate, k, ws);
}

cudaError_t launch_gemv(const void* W, const void* x, void* y, int d_in, int d_out, cudaStream_t s) {
  const int rows_per_block = GV_THREADS / 32;
  const size_t smem = sizeof(__nv_bfloat16) * (size_t)d_in;
  static SmemLimit limit;
  if (smem > 48 * 1024) {
    cudaError_t err = limit.ensure((const void*)gemv_kernel, smem);
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(gemv_kernel, dim3((d_out + rows_per_block - 1) / rows_per_block),
                    dim3(GV_THREADS), smem, s, (const __nv_bfloat16*)W, (const __nv_bfloat16*)x,
                    (__nv_bfloat16*)y, d_in, d_out);
}

bool merge_supported(int k, int r, int nproj) { return k * r <= MG_MAXKR && nproj <= MG_MAXPROJ; }

}  // namespace apr
