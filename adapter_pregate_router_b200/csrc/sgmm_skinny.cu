// SGMM for few tokens per adapter (decode, many tenants): a memory-bound
// skinny product on CUDA cores.  AdaFuse summary (gist.science), Resumen
// tecnico §2.B: the segmented gather product applies the selected low-rank
// adapters to the tokens gathered per adapter, fused into the add onto the
// base projection output, with prefetching and tiling to hide global-memory
// latency.
//
//   y_p[t] = y_base_p[t] + sum_j gate[t,j] * B_e (A_e x[t]),  e = idx[t,j]
//
// Two launches per shared-input group.  Both are launched with programmatic
// dependent launch and read the adapter weights (static inputs) BEFORE waiting
// for the preceding kernel on the stream, so the weight stream of one call
// overlaps the tail of the previous one; everything produced by earlier
// kernels (routing plan, x, y_base, partial sums) is read after the wait.
//
// shrink  static items (projection, adapter e, 2048-column chunk, 16-row chunk
//         of A_e, split of the segment).  Each thread holds an 8-column slice
//         of 16 rows of A_e in registers (128-bit loads), streams the gathered
//         x rows of the segment's pairs 8 at a time, and reduces the 16 dot
//         products across the warp with a transposing shuffle reduction
//         (16 shuffles for 16 values) and across warps in shared memory.
//         Partial sums go to the workspace per (projection, column chunk):
//         no atomics, so results do not depend on scheduling.
// expand  CTA per (projection, token tile, 128 output columns).  Token tiles
//         follow the adapter-set order of the routing plan.  B rows of the
//         tile's adapters are staged in shared memory with cp.async (all
//         adapters before the wait when they fit), y_base rows are fetched
//         asynchronously, the column-chunk partials of the tile's pairs are
//         summed in a fixed order and gated, products accumulate in fp32, and
//         y = y_base + delta is written with 128-bit stores, one rounding per
//         element.  Each output element has one owner: y may alias y_base.
#include "apr_internal.cuh"

namespace apr {

constexpr int SH_THREADS = 128;
constexpr int SH_RC = 16;          // rows of A_e per shrink item

constexpr int EX_THREADS = 64;
constexpr int EX_NT = 64;          // output columns per expand CTA
constexpr int EX_BBUDGET = 32 * 1024;

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
__device__ __forceinline__ void zero8(Vec8<In>& r) {
#pragma unroll
  for (int c = 0; c < 8; ++c) r.v[c] = from_f32<In>(0.f);
}

__device__ __forceinline__ bool rank_ok(int r, int max_rank) { return r > 0 && r <= max_rank && !(r & 7); }

// ---------------------------------------------------------------- shrink

template <typename In>
__global__ void __launch_bounds__(SH_THREADS) sgmm_shrink_kernel(SgmmArgs a, size_t scratch_off,
                                                                    int nkc, int nrc, int nsplit) {
  constexpr int SH_BATCH = sizeof(In) == 2 ? 8 : 4;   // x rows in flight per thread
  __shared__ float red[SH_THREADS / 32][kPairTile][SH_RC + 1];
  __shared__ int s_tok[kPairTile];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int npairs = a.T * a.k;
  const long nitems = (long)a.nproj * a.E * nkc * nrc * nsplit;
  const In* __restrict__ x = reinterpret_cast<const In*>(a.x);
  const int d_in = a.d_in;
  float* vpart = ws_at<float>(a.ws, scratch_off);
  bool waited = false;

  for (long it = blockIdx.x; it < nitems; it += gridDim.x) {
    long rest = it;
    const int split = (int)(rest % nsplit); rest /= nsplit;
    const int rc = (int)(rest % nrc); rest /= nrc;
    const int kc = (int)(rest % nkc); rest /= nkc;
    const int e = (int)(rest % a.E);
    const int p = (int)(rest / a.E);
    // static inputs: rank and weights (read before waiting on the previous kernel)
    const int r_e = a.ranks[e];
    const bool bad = !rank_ok(r_e, a.max_rank);
    const int r0 = rc * SH_RC;
    const bool has_rows = !bad && r0 < r_e;
    const int nr = has_rows ? min(SH_RC, r_e - r0) : 0;
    const int col = kc * kShrinkKC + tid * 8;
    const bool active = col < d_in;
    Vec8<In> areg[SH_RC];
    if (has_rows) {
      const In* __restrict__ A = reinterpret_cast<const In*>(a.proj[p].A[e]);
#pragma unroll
      for (int i = 0; i < SH_RC; ++i) {
        if (active && i < nr) raw_load8(A + (size_t)(r0 + i) * d_in + col, areg[i]);
        else zero8(areg[i]);
      }
    }
    if (!waited) {
      pdl_wait();
      pdl_trigger();
      waited = true;
    }
    if (bad) {
      if (tid == 0 && p == 0 && rc == 0 && kc == 0 && split == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_SHRINK, e);
      continue;
    }
    if (!has_rows) continue;
    const int seg0 = a.seg_off[e], seg1 = a.seg_off[e + 1];
    for (int ts = seg0 + split * kPairTile; ts < seg1; ts += nsplit * kPairTile) {
      const int len = min(kPairTile, seg1 - ts);
      if (tid < len) s_tok[tid] = a.perm[ts + tid] / a.k;
      __syncthreads();
      for (int s0 = 0; s0 < len; s0 += SH_BATCH) {
        Vec8<In> xr[SH_BATCH];
#pragma unroll
        for (int u = 0; u < SH_BATCH; ++u) {
          if (active && s0 + u < len) raw_load8(x + (size_t)s_tok[s0 + u] * d_in + col, xr[u]);
          else zero8(xr[u]);
        }
#pragma unroll
        for (int u = 0; u < SH_BATCH; ++u) {
          if (s0 + u >= len) break;
          float xv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) xv[c] = to_f32(xr[u].v[c]);
          float v[16];
#pragma unroll
          for (int i = 0; i < SH_RC; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) acc = fmaf(to_f32(areg[i].v[c]), xv[c], acc);
            v[i] = acc;
          }
          warp_transpose_reduce16(v, lane);
          if ((lane & 1) == 0) red[warp][s0 + u][lane >> 1] = v[0];
        }
      }
      __syncthreads();
      float* out = vpart + ((size_t)(p * nkc + kc) * npairs + ts) * a.max_rank + r0;
      for (int j = tid; j < len * SH_RC; j += SH_THREADS) {
        const int s = j / SH_RC, i = j % SH_RC;
        if (i < nr) {
          float sum = 0.f;
#pragma unroll
          for (int w = 0; w < SH_THREADS / 32; ++w) sum += red[w][s][i];
          out[(size_t)s * a.max_rank + i] = sum;
        }
      }
      __syncthreads();
    }
  }
  // A CTA without items exits; that counts as its trigger for the next launch.
}

// ---------------------------------------------------------------- expand

struct ExpandSmem {      // byte offsets inside the dynamic shared memory
  size_t B, yb, v, acc, ints, total;
};

__host__ __device__ inline ExpandSmem expand_smem_layout(int TT, int k, int R, int elem, int bslots) {
  ExpandSmem L;
  const int TK = TT * k;
  size_t o = 0;
  L.B = o;    o += (size_t)bslots * EX_NT * ((size_t)R * elem + 16);
  L.yb = o;   o += (size_t)TT * EX_NT * elem;
  L.v = o;    o += sizeof(float) * (size_t)TK * R;
  L.acc = o;  o += sizeof(float) * (size_t)TT * EX_NT;
  L.ints = o; o += sizeof(int) * ((size_t)TT + 7 * (size_t)TK + 1);
  L.total = (o + 15) / 16 * 16;
  return L;
}

// Inputs of the call (weights, routing plan, y_base) are read before waiting
// for the preceding kernel, which is always this call's shrink: it only
// triggers this launch after its own wait, so everything written two or more
// launches back is complete.  Only the shrink's partial sums need the wait.
template <typename In>
__global__ void __launch_bounds__(EX_THREADS) sgmm_expand_kernel(SgmmArgs a, size_t scratch_off,
                                                                 int nkc, int TT, int bslots,
                                                                 int prefetch_all) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int p = blockIdx.z, tt = blockIdx.y;
  const int d_out = a.proj[p].d_out;
  const int n0 = blockIdx.x * EX_NT;
  if (n0 >= d_out) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = a.k, R = a.max_rank, E = a.E;
  const int TK = TT * K;
  const int npairs = a.T * K;
  const int elem = (int)sizeof(In);
  const int nrows = min(EX_NT, d_out - n0);
  const ExpandSmem Ls = expand_smem_layout(TT, K, R, elem, bslots);
  unsigned char* s_B = smem + Ls.B;
  In* s_yb = reinterpret_cast<In*>(smem + Ls.yb);
  float* s_v = reinterpret_cast<float*>(smem + Ls.v);
  float* s_acc = reinterpret_cast<float*>(smem + Ls.acc);
  int* s_tok = reinterpret_cast<int*>(smem + Ls.ints);   // [TT]
  int* s_pe = s_tok + TT;                                  // [TK] adapter of each pair (-1: none)
  int* s_pr = s_pe + TK;                                   // [TK] its rank
  int* s_pu = s_pr + TK;                                   // [TK] staging slot of that adapter
  int* s_pos = s_pu + TK;                                  // [TK] sorted position of the pair
  int* s_U = s_pos + TK;                                   // [TK] distinct adapters (dedupe path)
  int* s_Ur = s_U + TK;                                    // [TK] their ranks
  float* s_g = reinterpret_cast<float*>(s_Ur + TK);        // [TK] gate of the pair
  int* s_nU = reinterpret_cast<int*>(s_g + TK);            // [1]
  const int stride_b = R * elem + 16;
  const In* const* Bp = reinterpret_cast<const In* const*>(a.proj[p].B);

  // stage B_e[n0 : n0 + nrows, 0 : r_e] of adapter e into slot `slot`
  auto stage_B = [&](int e, int r_e, int slot) {
    const int vpr = r_e * elem / 16;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(Bp[e] + (size_t)n0 * r_e);
    unsigned char* dst = s_B + (size_t)slot * EX_NT * stride_b;
    for (int v = tid; v < nrows * vpr; v += EX_THREADS) {
      const int row = v / vpr, c = v % vpr;
      cp_async16(dst + (size_t)row * stride_b + c * 16, src + ((size_t)row * vpr + c) * 16);
    }
  };

  // ---- before the wait: weights, routing plan of the tile, y_base rows
  if (prefetch_all) {
    for (int e = 0; e < E; ++e) {
      const int r_e = a.ranks[e];
      if (rank_ok(r_e, R)) stage_B(e, r_e, e);
    }
  }
  const WsLayout L = ws_layout(a.T, a.k, a.E);
  const int* tok_order = ws_at<int>(a.ws, L.tok_order);
  const int* inv = ws_at<int>(a.ws, L.inv);
  const int ntok = min(TT, a.T - tt * TT);
  for (int i = tid; i < TT; i += EX_THREADS) s_tok[i] = i < ntok ? tok_order[tt * TT + i] : -1;
  __syncthreads();
  const In* __restrict__ yb = reinterpret_cast<const In*>(a.proj[p].y_base);
  {
    const int vpr = nrows * elem / 16;
    for (int v = tid; v < ntok * vpr; v += EX_THREADS) {
      const int i = v / vpr, c = v % vpr;
      cp_async16(reinterpret_cast<unsigned char*>(s_yb + (size_t)i * EX_NT) + c * 16,
                 reinterpret_cast<const unsigned char*>(yb + (size_t)s_tok[i] * d_out + n0) + c * 16);
    }
  }
  cp_async_commit();
  for (int pi = tid; pi < TK; pi += EX_THREADS) {
    const int i = pi / K, j = pi % K;
    int e = -1, pos = 0, r_e = 0;
    float g = 0.f;
    if (i < ntok) {
      const int q = s_tok[i] * K + j;
      e = a.idx[q];
      pos = inv[q];
      g = a.gate[q];
      r_e = (e >= 0 && e < E) ? a.ranks[e] : 0;
      if (!rank_ok(r_e, R)) {
        report(a.ws, APR_ERR_DEVICE_INDEX, K_EXPAND, e);
        e = -1;
        r_e = 0;
      }
    }
    s_pe[pi] = e;
    s_pr[pi] = r_e;
    s_pos[pi] = pos;
    s_g[pi] = g;
  }
  __syncthreads();
  int nU;
  if (prefetch_all) {
    for (int pi = tid; pi < TK; pi += EX_THREADS) s_pu[pi] = s_pe[pi];
    nU = E;
  } else {
    // distinct adapters of the tile, in order of first appearance
    if (warp == 0) {
      int nu = 0;
      for (int c0 = 0; c0 < TK; c0 += 32) {
        const int pi = c0 + lane;
        const int e = pi < TK ? s_pe[pi] : -1;
        bool first = e >= 0;
        for (int q = 0; first && q < pi; ++q) first = s_pe[q] != e;
        const unsigned m = __ballot_sync(0xffffffffu, first);
        if (first) {
          const int slot = nu + __popc(m & ((1u << lane) - 1u));
          s_U[slot] = e;
          s_Ur[slot] = s_pr[pi];
        }
        nu += __popc(m);
      }
      if (lane == 0) *s_nU = nu;
    }
    __syncthreads();
    nU = *s_nU;
    for (int pi = tid; pi < TK; pi += EX_THREADS) {
      const int e = s_pe[pi];
      int slot = -1;
      if (e >= 0)
        for (int u = 0; u < nU; ++u)
          if (s_U[u] == e) { slot = u; break; }
      s_pu[pi] = slot;
    }
  }
  for (int w = tid; w < TT * EX_NT; w += EX_THREADS) s_acc[w] = 0.f;

  // ---- after the wait: the shrink's partial sums
  pdl_wait();
  pdl_trigger();
  const float* vpart = ws_at<float>(a.ws, scratch_off) + (size_t)p * nkc * npairs * R;
  constexpr int VB = 8;                         // independent loads in flight per thread
  for (int w0 = tid * VB; w0 < TK * R; w0 += EX_THREADS * VB) {
    float part[VB];
#pragma unroll
    for (int u = 0; u < VB; ++u) part[u] = 0.f;
    for (int c = 0; c < nkc; ++c) {
      float ld[VB];
#pragma unroll
      for (int u = 0; u < VB; ++u) {
        const int w = w0 + u;
        const int pi = w / R, i = w % R;
        ld[u] = (w < TK * R && i < s_pr[pi])
                    ? vpart[((size_t)c * npairs + s_pos[pi]) * R + i] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < VB; ++u) part[u] += ld[u];
    }
#pragma unroll
    for (int u = 0; u < VB; ++u) {
      const int w = w0 + u;
      if (w < TK * R) s_v[w] = s_g[w / R] * part[u];
    }
  }
  __syncthreads();

  const int ucap = prefetch_all ? E : bslots;
  for (int u0 = 0; u0 < nU; u0 += ucap) {
    const int u1 = min(nU, u0 + ucap);
    if (!prefetch_all) {
      for (int u = u0; u < u1; ++u) stage_B(s_U[u], s_Ur[u], u - u0);
      cp_async_commit();
    }
    cp_async_wait_all();
    __syncthreads();
    if (tid < nrows) {
      for (int i = 0; i < ntok; ++i) {
        float acc = 0.f;
        for (int j = 0; j < K; ++j) {
          const int pi = i * K + j;
          const int u = s_pu[pi];
          if (u < u0 || u >= u1) continue;
          const int r_u = s_pr[pi];
          const In* brow =
              reinterpret_cast<const In*>(s_B + (size_t)(u - u0) * EX_NT * stride_b + (size_t)tid * stride_b);
          const float* vv = s_v + (size_t)pi * R;
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
  cp_async_wait_all();
  __syncthreads();
  // y = y_base + delta, 8 columns per access
  In* __restrict__ y = reinterpret_cast<In*>(a.proj[p].y);
  const int vpr_out = EX_NT / 8;
  for (int w = tid; w < ntok * vpr_out; w += EX_THREADS) {
    const int i = w / vpr_out, c8 = (w % vpr_out) * 8;
    if (c8 >= nrows) continue;
    float f[8];
    load8(s_yb + (size_t)i * EX_NT + c8, f);
    const float4 a0 = *reinterpret_cast<const float4*>(s_acc + i * EX_NT + c8);
    const float4 a1 = *reinterpret_cast<const float4*>(s_acc + i * EX_NT + c8 + 4);
    f[0] += a0.x; f[1] += a0.y; f[2] += a0.z; f[3] += a0.w;
    f[4] += a1.x; f[5] += a1.y; f[6] += a1.z; f[7] += a1.w;
    store8(y + (size_t)s_tok[i] * d_out + n0 + c8, f);
  }
}

static int expand_tokens_per_tile(int k, int max_rank) {
  int tt = 8192 / (k * max_rank);
  if (tt > 32) tt = 32;
  if (tt < 1) tt = 1;
  return tt;
}

static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <typename In>
static cudaError_t launch_skinny_typed(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  const int nkc = shrink_kchunks(a.d_in);
  const int nrc = (a.max_rank + SH_RC - 1) / SH_RC;
  // split long segments over several CTAs (mean pairs per adapter known on the host)
  const long mean_tiles = ((long)a.T * a.k / a.E + kPairTile - 1) / kPairTile;
  int nsplit = (int)((mean_tiles + 1) / 2);
  if (nsplit < 1) nsplit = 1;
  if (nsplit > 16) nsplit = 16;
  const long nitems = (long)a.nproj * a.E * nkc * nrc * nsplit;
  const long cap = 16L * sm_count();
  const long g1 = nitems < cap ? nitems : cap;
  cudaError_t err = launch_pdl(sgmm_shrink_kernel<In>, dim3((unsigned)g1), dim3(SH_THREADS), 0, s, a,
                               scratch_off, nkc, nrc, nsplit);
  if (err != cudaSuccess) return err;

  const int elem = (int)sizeof(In);
  const int TT = expand_tokens_per_tile(a.k, a.max_rank);
  const int ntt = (a.T + TT - 1) / TT;
  int ntd = 1;
  for (int p = 0; p < a.nproj; ++p) {
    const int n = (a.proj[p].d_out + EX_NT - 1) / EX_NT;
    if (n > ntd) ntd = n;
  }
  const size_t per_slot = (size_t)EX_NT * ((size_t)a.max_rank * elem + 16);
  const int prefetch_all = (size_t)a.E * per_slot <= (size_t)EX_BBUDGET ? 1 : 0;
  int bslots = prefetch_all ? a.E : (int)(EX_BBUDGET / per_slot);
  if (bslots < 1) bslots = 1;
  const size_t smem = expand_smem_layout(TT, a.k, a.max_rank, elem, bslots).total;
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    err = cudaFuncSetAttribute(sgmm_expand_kernel<In>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    configured = smem;
  }
  return launch_pdl(sgmm_expand_kernel<In>, dim3(ntd, ntt, a.nproj), dim3(EX_THREADS), smem, s, a,
                    scratch_off, nkc, TT, bslots, prefetch_all);
}

cudaError_t launch_sgmm_skinny(const SgmmArgs& a, int dtype, size_t scratch_off, cudaStream_t s) {
  if (dtype == APR_BF16) return launch_skinny_typed<__nv_bfloat16>(a, scratch_off, s);
  return launch_skinny_typed<float>(a, scratch_off, s);
}

}  // namespace apr
