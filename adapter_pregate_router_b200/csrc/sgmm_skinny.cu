// SGMM for few tokens per adapter (decode, many tenants): a memory-bound
// skinny product on CUDA cores.  AdaFuse summary (gist.science), Resumen
// tecnico §2.B: the segmented gather product applies the selected low-rank
// adapters to the tokens gathered per adapter, fused into the add onto the
// base projection output, with prefetching and tiling to hide global-memory
// latency.
//
//   y_p[t] = y_base_p[t] + sum_j gate[t,j] * B_e (A_e x[t]),  e = idx[t,j]
//
// Two launches per shared-input group (programmatic dependent launch lets the
// second one start while the first drains):
//
// shrink  items (projection, pair tile of one adapter, 2048-column chunk,
//         16-row chunk of A_e).  Each thread keeps an 8-column slice of 16
//         rows of A_e in registers (128-bit loads, read once), streams the
//         gathered x rows of the tile's pairs, and reduces the 16 partial dot
//         products across the warp with a transposing shuffle reduction
//         (16 shuffles for 16 values) and across warps through shared memory.
//         Partial sums go to the workspace per column chunk (no atomics).
// expand  CTA per (projection, token tile, 128 output columns).  Token tiles
//         follow the adapter-set order built by the segment kernel, so a
//         tile touches few adapters.  The CTA sums the column-chunk partials
//         of its tokens' pairs, applies the gates, stages the B_e rows of the
//         distinct adapters of the tile in shared memory, accumulates in fp32
//         and finally streams y_base -> y with 128-bit accesses, one rounding
//         per element.  Each output element has one owner: no atomics, y may
//         alias y_base.
#include "apr_internal.cuh"

namespace apr {

constexpr int SH_THREADS = 256;
constexpr int SH_RC = 16;          // rows of A_e per shrink item
constexpr int SH_BATCH = 4;        // x rows in flight per thread

constexpr int EX_THREADS = 128;
constexpr int EX_NT = 128;         // output columns per expand CTA
constexpr int EX_BBUDGET = 48 * 1024;

// Sum 16 values over the 32 lanes of a warp.  On return, even lanes hold the
// total of value (lane >> 1) in v[0].
__device__ __forceinline__ void warp_transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 16;
    const float send = up ? v[i] : v[i + 8];
    const float keep = up ? v[i + 8] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 8;
    const float send = up ? v[i] : v[i + 4];
    const float keep = up ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 4;
    const float send = up ? v[i] : v[i + 2];
    const float keep = up ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool up = lane & 2;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

template <typename In>
struct Vec8 {
  In v[8];
};

template <typename In>
__device__ __forceinline__ void raw_load8(const In* p, Vec8<In>& r) {
  if constexpr (sizeof(In) == 2) {
    *reinterpret_cast<uint4*>(&r) = *reinterpret_cast<const uint4*>(p);
  } else {
    reinterpret_cast<float4*>(&r)[0] = reinterpret_cast<const float4*>(p)[0];
    reinterpret_cast<float4*>(&r)[1] = reinterpret_cast<const float4*>(p)[1];
  }
}

template <typename In>
__global__ void __launch_bounds__(SH_THREADS) sgmm_shrink_kernel(SgmmArgs a, size_t scratch_off,
                                                                 int nkc, int nrc) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[SH_THREADS / 32][kPairTile][SH_RC + 1];
  __shared__ int s_tok[kPairTile];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const WsLayout L = ws_layout(a.T, a.k, a.E);
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const PairTile* tiles = ws_at<PairTile>(a.ws, L.ptiles);
  float* vpart = ws_at<float>(a.ws, scratch_off);
  const int ntiles = hdr->n_ptiles;
  const int npairs = a.T * a.k;
  const long nitems = (long)a.nproj * ntiles * nkc * nrc;
  const In* __restrict__ x = reinterpret_cast<const In*>(a.x);
  const int d_in = a.d_in;

  for (long it = blockIdx.x; it < nitems; it += gridDim.x) {
    const int rc = (int)(it % nrc);
    long rest = it / nrc;
    const int kc = (int)(rest % nkc);
    rest /= nkc;
    const int tile = (int)(rest % ntiles);
    const int p = (int)(rest / ntiles);
    const PairTile pt = tiles[tile];
    const int e = pt.e;
    const int r_e = a.ranks[e];
    if (r_e <= 0 || r_e > a.max_rank || (r_e & 7)) {
      if (tid == 0 && rc == 0 && kc == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_SHRINK, e);
      continue;
    }
    const int r0 = rc * SH_RC;
    if (r0 >= r_e) continue;
    const int nr = min(SH_RC, r_e - r0);
    const In* __restrict__ A = reinterpret_cast<const In*>(a.proj[p].A[e]);
    const int col = kc * kShrinkKC + tid * 8;
    const bool active = col < d_in;

    if (tid < pt.len) s_tok[tid] = a.perm[pt.start + tid] / a.k;
    Vec8<In> areg[SH_RC];
#pragma unroll
    for (int i = 0; i < SH_RC; ++i) {
      if (active && i < nr) {
        raw_load8(A + (size_t)(r0 + i) * d_in + col, areg[i]);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) areg[i].v[c] = from_f32<In>(0.f);
      }
    }
    __syncthreads();

    for (int s0 = 0; s0 < pt.len; s0 += SH_BATCH) {
      float xv[SH_BATCH][8];
#pragma unroll
      for (int u = 0; u < SH_BATCH; ++u) {
        if (active && s0 + u < pt.len) {
          load8(x + (size_t)s_tok[s0 + u] * d_in + col, xv[u]);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) xv[u][c] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < SH_BATCH; ++u) {
        if (s0 + u >= pt.len) break;
        float v[16];
#pragma unroll
        for (int i = 0; i < SH_RC; ++i) {
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) acc = fmaf(to_f32(areg[i].v[c]), xv[u][c], acc);
          v[i] = acc;
        }
        warp_transpose_reduce16(v, lane);
        if ((lane & 1) == 0) red[warp][s0 + u][lane >> 1] = v[0];
      }
    }
    __syncthreads();
    for (int j = tid; j < pt.len * SH_RC; j += SH_THREADS) {
      const int s = j / SH_RC, i = j % SH_RC;
      if (i < nr) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < SH_THREADS / 32; ++w) sum += red[w][s][i];
        vpart[((size_t)kc * npairs + pt.start + s) * a.max_rank + r0 + i] = sum;
      }
    }
    __syncthreads();
  }
}

template <typename In>
__global__ void __launch_bounds__(EX_THREADS) sgmm_expand_kernel(SgmmArgs a, size_t scratch_off,
                                                                 int nkc, int TT) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char smem[];
  const int p = blockIdx.z, tt = blockIdx.y;
  const int d_out = a.proj[p].d_out;
  const int n0 = blockIdx.x * EX_NT;
  if (n0 >= d_out) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = a.k, R = a.max_rank;
  const int TK = TT * K;
  const int npairs = a.T * K;
  const WsLayout L = ws_layout(a.T, a.k, a.E);
  const int* tok_order = ws_at<int>(a.ws, L.tok_order);
  const int* inv = ws_at<int>(a.ws, L.inv);
  const float* vpart = ws_at<float>(a.ws, scratch_off);

  // shared layout
  float* s_v = reinterpret_cast<float*>(smem);                 // [TK][R]
  float* s_acc = s_v + (size_t)TK * R;                         // [TT][EX_NT]
  int* s_tok = reinterpret_cast<int*>(s_acc + (size_t)TT * EX_NT);  // [TT]
  int* s_pe = s_tok + TT;                                      // [TK] adapter of each pair
  int* s_pu = s_pe + TK;                                       // [TK] slot in U
  int* s_U = s_pu + TK;                                        // [TK] distinct adapters
  int* s_Ur = s_U + TK;                                        // [TK] their ranks
  int* s_nU = s_Ur + TK;                                       // [1]
  unsigned char* s_B = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(s_nU + 1) + 15) & ~uintptr_t(15));
  const int stride_b = R * (int)sizeof(In) + 16;               // bytes per staged B row

  const int ntok = min(TT, a.T - tt * TT);
  for (int i = tid; i < TT; i += EX_THREADS) s_tok[i] = i < ntok ? tok_order[tt * TT + i] : -1;
  __syncthreads();
  for (int pi = tid; pi < TK; pi += EX_THREADS) {
    const int i = pi / K, j = pi % K;
    int e = -1;
    if (i < ntok) {
      e = a.idx[(size_t)s_tok[i] * K + j];
      if (e < 0 || e >= a.E) {
        report(a.ws, APR_ERR_DEVICE_INDEX, K_EXPAND, e);
        e = -1;
      } else {
        const int r_e = a.ranks[e];
        if (r_e <= 0 || r_e > R || (r_e & 7)) {
          report(a.ws, APR_ERR_DEVICE_INDEX, K_EXPAND, e);
          e = -1;
        }
      }
    }
    s_pe[pi] = e;
  }
  __syncthreads();
  // distinct adapters of the tile, in order of first appearance
  if (warp == 0) {
    int nu = 0;
    for (int c0 = 0; c0 < TK; c0 += 32) {
      const int pi = c0 + lane;
      int e = pi < TK ? s_pe[pi] : -1;
      bool first = e >= 0;
      for (int q = 0; first && q < pi; ++q) first = s_pe[q] != e;
      const unsigned m = __ballot_sync(0xffffffffu, first);
      if (first) {
        const int slot = nu + __popc(m & ((1u << lane) - 1u));
        s_U[slot] = e;
        s_Ur[slot] = a.ranks[e];
      }
      nu += __popc(m);
    }
    if (lane == 0) *s_nU = nu;
  }
  __syncthreads();
  const int nU = *s_nU;
  for (int pi = tid; pi < TK; pi += EX_THREADS) {
    const int e = s_pe[pi];
    int slot = -1;
    if (e >= 0)
      for (int u = 0; u < nU; ++u)
        if (s_U[u] == e) { slot = u; break; }
    s_pu[pi] = slot;
  }
  // gate-scaled v of every pair of the tile (column-chunk partials summed in order)
  for (int w = tid; w < TK * R; w += EX_THREADS) {
    const int pi = w / R, i = w % R;
    const int e = s_pe[pi];
    float val = 0.f;
    if (e >= 0 && i < a.ranks[e]) {
      const int q = s_tok[pi / K] * K + (pi % K);
      const int pos = inv[q];
      float sum = 0.f;
      for (int c = 0; c < nkc; ++c) sum += vpart[((size_t)c * npairs + pos) * R + i];
      val = a.gate[q] * sum;
    }
    s_v[w] = val;
  }
  for (int w = tid; w < TT * EX_NT; w += EX_THREADS) s_acc[w] = 0.f;
  __syncthreads();

  const int nrows = min(EX_NT, d_out - n0);
  const int ucap = max(1, EX_BBUDGET / (EX_NT * stride_b));
  const In* const* Bp = reinterpret_cast<const In* const*>(a.proj[p].B);
  for (int u0 = 0; u0 < nU; u0 += ucap) {
    const int u1 = min(nU, u0 + ucap);
    // stage B_u[n0 : n0 + nrows, 0 : r_u] for u in [u0, u1)
    for (int u = u0; u < u1; ++u) {
      const int r_u = s_Ur[u];
      const int vpr = r_u * (int)sizeof(In) / 16;
      const unsigned char* src =
          reinterpret_cast<const unsigned char*>(Bp[s_U[u]] + (size_t)n0 * r_u);
      unsigned char* dst = s_B + (size_t)(u - u0) * EX_NT * stride_b;
      for (int v = tid; v < nrows * vpr; v += EX_THREADS) {
        const int row = v / vpr, c = v % vpr;
        *reinterpret_cast<uint4*>(dst + (size_t)row * stride_b + c * 16) =
            *reinterpret_cast<const uint4*>(src + ((size_t)row * vpr + c) * 16);
      }
    }
    __syncthreads();
    if (tid < nrows) {
      for (int i = 0; i < ntok; ++i) {
        float acc = 0.f;
        for (int j = 0; j < K; ++j) {
          const int u = s_pu[i * K + j];
          if (u < u0 || u >= u1) continue;
          const int r_u = s_Ur[u];
          const In* brow =
              reinterpret_cast<const In*>(s_B + (size_t)(u - u0) * EX_NT * stride_b + (size_t)tid * stride_b);
          const float* vv = s_v + (size_t)(i * K + j) * R;
          for (int c = 0; c < r_u; c += 8) {
            float b[8];
            load8(brow + c, b);
            const float4 v0 = *reinterpret_cast<const float4*>(vv + c);
            const float4 v1 = *reinterpret_cast<const float4*>(vv + c + 4);
            acc = fmaf(b[0], v0.x, acc);
            acc = fmaf(b[1], v0.y, acc);
            acc = fmaf(b[2], v0.z, acc);
            acc = fmaf(b[3], v0.w, acc);
            acc = fmaf(b[4], v1.x, acc);
            acc = fmaf(b[5], v1.y, acc);
            acc = fmaf(b[6], v1.z, acc);
            acc = fmaf(b[7], v1.w, acc);
          }
        }
        s_acc[i * EX_NT + tid] += acc;
      }
    }
    __syncthreads();
  }
  // y = y_base + delta, 8 columns per access
  const In* __restrict__ yb = reinterpret_cast<const In*>(a.proj[p].y_base);
  In* __restrict__ y = reinterpret_cast<In*>(a.proj[p].y);
  const int vpr_out = EX_NT / 8;
  for (int w = tid; w < ntok * vpr_out; w += EX_THREADS) {
    const int i = w / vpr_out, c8 = (w % vpr_out) * 8;
    const int n = n0 + c8;
    if (n >= d_out) continue;
    const size_t off = (size_t)s_tok[i] * d_out + n;
    float f[8];
    load8(yb + off, f);
    const float4 a0 = *reinterpret_cast<const float4*>(s_acc + i * EX_NT + c8);
    const float4 a1 = *reinterpret_cast<const float4*>(s_acc + i * EX_NT + c8 + 4);
    f[0] += a0.x; f[1] += a0.y; f[2] += a0.z; f[3] += a0.w;
    f[4] += a1.x; f[5] += a1.y; f[6] += a1.z; f[7] += a1.w;
    store8(y + off, f);
  }
}

static int expand_tokens_per_tile(int k, int max_rank) {
  int tt = 8192 / (k * max_rank);
  if (tt > 32) tt = 32;
  if (tt < 1) tt = 1;
  return tt;
}

static size_t expand_smem_bytes(int TT, int k, int R, int elem) {
  const int TK = TT * k;
  size_t b = sizeof(float) * ((size_t)TK * R + (size_t)TT * EX_NT);
  b += sizeof(int) * ((size_t)TT + 4 * (size_t)TK + 1);
  b = (b + 15) / 16 * 16;
  const size_t stride_b = (size_t)R * elem + 16;
  const size_t ucap = EX_BBUDGET / (EX_NT * stride_b) > 0 ? EX_BBUDGET / (EX_NT * stride_b) : 1;
  b += ucap * EX_NT * stride_b;
  return b;
}

template <typename In>
static cudaError_t launch_skinny_typed(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  const int nkc = shrink_kchunks(a.d_in);
  const int nrc = (a.max_rank + SH_RC - 1) / SH_RC;
  const long max_items = (long)a.nproj * max_ptiles(a.T, a.k, a.E) * nkc * nrc;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const long g1 = max_items < 4L * nsm ? max_items : 4L * nsm;
  cudaError_t err = launch_pdl(sgmm_shrink_kernel<In>, dim3((unsigned)(g1 > 0 ? g1 : 1)),
                               dim3(SH_THREADS), 0, s, a, scratch_off, nkc, nrc);
  if (err != cudaSuccess) return err;
  const int TT = expand_tokens_per_tile(a.k, a.max_rank);
  const int ntt = (a.T + TT - 1) / TT;
  int ntd = 1;
  for (int p = 0; p < a.nproj; ++p) {
    const int n = (a.proj[p].d_out + EX_NT - 1) / EX_NT;
    if (n > ntd) ntd = n;
  }
  const size_t smem = expand_smem_bytes(TT, a.k, a.max_rank, (int)sizeof(In));
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    err = cudaFuncSetAttribute(sgmm_expand_kernel<In>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (err != cudaSuccess) return err;
    configured = smem;
  }
  return launch_pdl(sgmm_expand_kernel<In>, dim3(ntd, ntt, a.nproj), dim3(EX_THREADS), smem, s, a,
                    scratch_off, nkc, TT);
}

cudaError_t launch_sgmm_skinny(const SgmmArgs& a, int dtype, size_t scratch_off, cudaStream_t s) {
  if (dtype == APR_BF16) return launch_skinny_typed<__nv_bfloat16>(a, scratch_off, s);
  return launch_skinny_typed<float>(a, scratch_off, s);
}

}  // namespace apr
