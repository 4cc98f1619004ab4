// SGMM for small batches (decode) as two dense tcgen05 products over the whole
// adapter bank.  AdaFuse summary (gist.science), Resumen tecnico §2.B: the
// segmented gather product applies the pre-gated adapters of every token and
// is fused into the add onto the base projection output.
//
// With a few dozen tokens the gather buys nothing: every adapter is selected
// by some token, so all of A and B is read anyway, and the cost of a call is
// its latency.  Both products therefore run densely over the E adapters
// (rank slots padded to Rp, a multiple of 16), and the gates zero what a token
// did not select:
//
//  shrink  U[e*Rp + i, t] = (A_e x_t)_i for all e, t.  The input columns are
//          split over clusters of 8 CTAs (16 where the rank rows fit one M
//          tile and the device can place such a cluster), 256 columns per
//          CTA; each CTA stages
//          its slice of every A_e (before the PDL wait: weights never depend
//          on the preceding launch) and of x (after it) in 128B-swizzled
//          K-major tiles, and one thread issues the tcgen05 MMAs
//          D[NR x Tp] = A_slice . x_slice^T (A as the M side, tokens as N).
//          The MMAs of the two halves of the K slice are issued by two
//          threads into two accumulators.  The cluster's partial products
//          are summed in a fixed order through distributed shared memory
//          (one rank-row tile: each CTA sends every owner its rows by one
//          bulk copy that completes on the owner's own mbarrier), gated
//          V[t, e*Rp + i] = sum_j [idx[t,j] = e] g[t,j] U[e*Rp + i, t]
//          and written as fp32 partials per cluster: [proj][cluster][Tp][NR];
//          when one cluster spans all of d_in, the final V is written instead,
//          split into bf16 hi + lo in the expand's MMA operand layout.
//  expand  one CTA per 128 output columns: D[128 x Tp] = Bslice . V^T with
//          Bslice[n, e*Rp + i] = B_e[n, i] (staged before the wait, with the
//          y_base columns) and V summed over the clusters in order and split
//          into bf16 hi + lo halves (two MMA chains, issued by two threads
//          into two accumulators, keep ~16 mantissa bits of v),
//          or, with a single cluster, V fetched as is by two bulk copies.
//          Thread n reads row n of D from TMEM and writes
//          y[t, n] = y_base[t, n] + D[n, t], rounded to bf16 once.
//
// Every wait is bounded (1 s); an expired wait records APR_ERR_TIMEOUT and the
// CTA still passes every cluster barrier and frees its TMEM.
#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int DN_THREADS = 256;
constexpr int DN_KC = 256;        // input columns per shrink CTA (four 64-column swizzle atoms)
constexpr int DN_CL = 8;          // shrink CTAs per cluster (16 when the rank rows fit one M tile)
constexpr int DN_NT = 128;        // output columns per expand CTA

struct DenseArgs {
  SgmmArgs a;
  int Tp;                              // tokens rounded up to 16 (MMA N)
  int Rp;                              // rank slot per adapter (max rank rounded up to 16)
  int NR;                              // E * Rp
  int MR;                              // NR rounded up to 128 (shrink MMA M)
  int ncl;                             // clusters along d_in
  int direct;                          // ncl == 1: the shrink writes the final V (bf16 hi | lo, MMA layout)
  size_t vpart_off;                    // scratch offset of the gated partials
  int tiles_before[APR_MAX_PROJ + 1];  // expand: prefix of 128-column tiles per projection
};

static_assert(DN_KC == 4 * 64, "four swizzle atoms per shrink CTA");

__device__ __forceinline__ uint32_t tmem_cols_for(int n) {
  uint32_t c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

// A load from another CTA's shared memory; ordered by the cluster barriers
// around it, it carries no memory clobber, so several stay in flight.
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// ---------------------------------------------------------------- shrink

// TP (tokens padded to 16) and MRT (rank rows padded to 128) are compile-time,
// so the decode instantiation is short straight-line code.
template <int TP, int MRT, int CLT>
__global__ void __launch_bounds__(DN_THREADS, 1) dense_shrink_kernel(const __grid_constant__ DenseArgs args) {
  const SgmmArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = blockIdx.x;                    // rank in the cluster (cluster spans gridDim.x)
  const int cl = blockIdx.y, p = blockIdx.z;
  constexpr int Tp = TP, MR = MRT;
  const int Rp = args.Rp, NR = args.NR;
  const int T = a.T, K = a.k, E = a.E, d_in = a.d_in;
  const int k0 = (cl * CLT + rank) * DN_KC;

  // shared memory: A slice [4 atoms][MR][128 B], x slice [4 atoms][Tp][128 B];
  // after the MMAs the A area holds this CTA's partial product: P[Tp][MR] fp32, or with one
  // M tile P[MR][Tp + 4] (row-major, padded: owner o's rows form one contiguous block).
  unsigned char* sA = smem;
  unsigned char* sX = smem + (size_t)MR * 512;
  constexpr int TS = TP + 4;                        // row stride of P and red with one M tile
  constexpr int RS = MR / CLT;                      // rank rows owned per CTA (8, 16 or 32)
  // MR == 128: each source CTA's block of this CTA's rows lands here, [source rank][RS][TS] fp32
  float* red = reinterpret_cast<float*>(sX + (size_t)Tp * 512);
  unsigned char* meta = sX + (size_t)Tp * 512 + (MR == 128 ? (size_t)TS * MR * 4 : 0);
  uint64_t* bar = reinterpret_cast<uint64_t*>(meta);                                  // [0] MMAs [1] rows in
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + 16);
  const __nv_bfloat16** s_Ap = reinterpret_cast<const __nv_bfloat16**>(meta + 32);   // [E]
  int* s_rk = reinterpret_cast<int*>(meta + 32 + 8 * 16);                             // [E]
  int* s_idx = s_rk + 16;                                                              // [T*K]
  float* s_gate = reinterpret_cast<float*>(s_idx + 64 * APR_MAX_K);                   // [T*K]
  float* P = reinterpret_cast<float*>(sA);

  // one M tile: the K slice's two halves go to two accumulators, issued by two threads
  constexpr int NACC = MR == 128 ? 2 : 1;
  // let the next kernel of the stream start staging its weights now: its CTAs still wait for this
  // grid to finish before they read anything it writes (griddepcontrol.wait)
  pdl_trigger();
  const uint32_t cs = tmem_cols_for(Tp);            // TMEM columns per M tile (a power of two)
  const uint32_t ncols = (uint32_t)(NACC * MR / 128) * cs;
  constexpr uint32_t kBlockBytes = (uint32_t)(RS * TS * 4);   // one source's rows for one owner
  if (tid == 0) {
    mbar_init(smem_u32(bar), NACC);
    mbar_init(smem_u32(bar + 1), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(s_tmem), ncols);
  if (tid < E) {
    s_Ap[tid] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].A[tid]);
    const int r = a.ranks[tid];
    const bool ok = r >= 8 && r <= Rp && (r & 7) == 0;
    if (!ok) report(a.ws, APR_ERR_DEVICE_INDEX, K_SHRINK, tid);
    s_rk[tid] = ok ? r : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if constexpr (MR == 128) {
    // the CLT blocks of this CTA's rows are expected as transaction bytes; every CTA's barrier is
    // initialised before any peer's copy can target it (cluster barrier, before the PDL wait)
    if (tid == 0) mbar_arrive_expect_tx(smem_u32(bar + 1), (uint32_t)CLT * kBlockBytes);
    cluster_sync_all();
  }

  // A slice of every adapter (rows beyond a rank, or columns beyond d_in, are zeros)
  {
    const int q = tid & 31;                 // 16-byte column chunk
    const int col = k0 + q * 8;
    const bool col_ok = col < d_in;
    int r = tid >> 5;
    int e = r / Rp, i = r - e * Rp;
    const uint32_t base = smem_u32(sA) + (uint32_t)(q >> 3) * (uint32_t)(MR * 128);
    for (; r < MR; r += 8) {
      const bool valid = col_ok && e < E && i < s_rk[e];
      const void* src = valid ? (const void*)(s_Ap[e] + (size_t)i * d_in + col) : (const void*)a.x;
      cp_async16_zfill(base + (uint32_t)r * 128 + ((((uint32_t)q & 7) ^ ((uint32_t)r & 7)) << 4), src, valid);
      i += 8;
      if (i >= Rp) { i -= Rp; ++e; }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  pdl_wait();

  // x slice of the tokens, and their routing
  {
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    const int q = tid & 31;
    const int col = k0 + q * 8;
    const uint32_t base = smem_u32(sX) + (uint32_t)(q >> 3) * (uint32_t)(Tp * 128);
    for (int t = tid >> 5; t < Tp; t += 8) {
      const bool valid = t < T && col < d_in;
      const void* src = valid ? (const void*)(x + (size_t)t * d_in + col) : (const void*)a.x;
      cp_async16_zfill(base + (uint32_t)t * 128 + ((((uint32_t)q & 7) ^ ((uint32_t)t & 7)) << 4), src, valid);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int w = tid; w < T * K; w += DN_THREADS) {
      s_idx[w] = a.idx[w];
      s_gate[w] = a.gate[w];
    }
  }
  cp_async_wait_all();
  fence_proxy_async();
  __syncthreads();

  // D[MR x Tp] = A_slice . x_slice^T, one M tile of 128 rows at a time; with one M tile, thread 0
  // issues the first half of the K steps into accumulator 0 and thread 32 the second half into
  // accumulator 1 (columns cs..)
  if (tid == 0 || (NACC == 2 && tid == 32)) {
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, Tp);
    const int h = tid >> 5;
    constexpr int KS = DN_KC / 16 / NACC;            // K steps per issuing thread
    for (int mt = 0; mt < MR / 128; ++mt)
      for (int kk = h * KS; kk < (h + 1) * KS; ++kk) {
        const uint32_t aa = smem_u32(sA) + (uint32_t)(kk >> 2) * (uint32_t)(MR * 128) + (uint32_t)mt * 16384 +
                            (uint32_t)(kk & 3) * 32;
        const uint32_t bb = smem_u32(sX) + (uint32_t)(kk >> 2) * (uint32_t)(Tp * 128) + (uint32_t)(kk & 3) * 32;
        mma_bf16(tmem + (uint32_t)(h + mt) * cs, desc_k_sw128(aa), desc_k_sw128(bb), id, kk > h * KS ? 1u : 0u);
      }
    mma_commit(smem_u32(bar));
  }
  const bool done = mbar_wait(smem_u32(bar), 0);
  tc_fence_after();
  if (!done) {
    if (tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_SHRINK, (int)blockIdx.x);
  } else {
    if constexpr (MR == 128) {
      // row r of the partial product (the two accumulators summed) -> P[r][0 .. Tp) (the A slice
      // is no longer read); owner o's rows o*RS .. are then one contiguous block
      // (this warp's column groups of both accumulators are all loaded before one wait)
      const int wq = warp & 3, wg = warp >> 2;
      const int r = wq * 32 + lane;
      constexpr int NG = (TP / 8 + 1) / 2;
      const uint32_t lb = tmem + ((uint32_t)(wq * 32) << 16);
      uint32_t v0[NG][8], v1[NG][8];
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        const int c8 = wg + 2 * gi;
        if (c8 < TP / 8) {
          tmem_ld8_async(lb + (uint32_t)(c8 * 8), v0[gi]);
          tmem_ld8_async(lb + cs + (uint32_t)(c8 * 8), v1[gi]);
        }
      }
      tmem_ld_wait();
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        const int c8 = wg + 2 * gi;
        if (c8 < TP / 8) {
          tmem_ld_tie(v0[gi]);
          tmem_ld_tie(v1[gi]);
          const auto f = [&](int u) { return __uint_as_float(v0[gi][u]) + __uint_as_float(v1[gi][u]); };
          float4* dst = reinterpret_cast<float4*>(P + (size_t)r * TS + c8 * 8);
          dst[0] = make_float4(f(0), f(1), f(2), f(3));
          dst[1] = make_float4(f(4), f(5), f(6), f(7));
        }
      }
    } else {
      // TMEM -> P[t][r] (the A slice is no longer read)
      const int wq = warp & 3, wg = warp >> 2;
      const int r_in = wq * 32 + lane;
      for (int mt = 0; mt < MR / 128; ++mt) {
        if (mt != wg) continue;
        for (int c8 = 0; c8 < Tp / 8; ++c8) {
          float v[8];
          tmem_ld8(tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)mt * cs + (uint32_t)(c8 * 8), v);
#pragma unroll
          for (int u = 0; u < 8; ++u) P[(size_t)(c8 * 8 + u) * MR + mt * 128 + r_in] = v[u];
        }
      }
    }
  }
  tc_fence_before();
  bool rows_in = true;
  if constexpr (MR == 128) {
    // every owner gets its block of this CTA's rows by one bulk copy into red[rank], completing
    // as transaction bytes on the owner's barrier; then this CTA waits for its own CLT blocks
    fence_proxy_async();                     // P's generic writes are visible to the copies
    __syncthreads();
    if (tid < CLT) {
      const uint32_t src = smem_u32(P) + (uint32_t)tid * kBlockBytes;
      const uint32_t dst = cluster_map(smem_u32(red) + (uint32_t)rank * kBlockBytes, (uint32_t)tid);
      const uint32_t rb = cluster_map(smem_u32(bar + 1), (uint32_t)tid);
      asm volatile(
          "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
          "r"(src), "r"(kBlockBytes), "r"(rb)
          : "memory");
      bulk_commit();
    }
    rows_in = mbar_wait(smem_u32(bar + 1), 0);
    if (!rows_in && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_SHRINK, (int)blockIdx.x);
  } else {
    cluster_sync_all();        // every CTA's partial product is in place
  }

  // this CTA's share of the rows, summed over the cluster in rank order, gated
  if (rows_in) {
    constexpr int groups = RS / 4;
    float* vpart = ws_at<float>(a.ws, args.vpart_off) + ((size_t)(p * args.ncl + cl) * Tp) * NR;
    constexpr int PER = (groups * TP + DN_THREADS - 1) / DN_THREADS;   // float4 groups per thread (1 or 2)
    float4 part[PER][CLT];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int w = tid + u * DN_THREADS;
      if (w < groups * Tp) {
        const int t = w / groups, g4 = w % groups;
        if constexpr (MR == 128) {
#pragma unroll
          for (int c = 0; c < CLT; ++c) {
            const float* blk = red + (size_t)c * RS * TS + (size_t)(g4 * 4) * TS + t;
            part[u][c] = make_float4(blk[0], blk[TS], blk[2 * TS], blk[3 * TS]);
          }
        } else {
          const uint32_t off = smem_u32(P + (size_t)t * MR + rank * RS + g4 * 4);
#pragma unroll
          for (int c = 0; c < CLT; ++c) part[u][c] = ld_cluster_f4(cluster_map(off, (uint32_t)c));
        }
      }
    }
    if constexpr (MR != 128) cluster_arrive();   // this CTA's reads of the cluster's P are done
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int w = tid + u * DN_THREADS;
      if (w >= groups * Tp) continue;
      const int t = w / groups, r0 = rank * RS + (w % groups) * 4;
      float4 s = part[u][0];
#pragma unroll
      for (int c = 1; c < CLT; ++c) {
        s.x += part[u][c].x; s.y += part[u][c].y; s.z += part[u][c].z; s.w += part[u][c].w;
      }
      if (r0 >= NR) continue;
      const int e = r0 / Rp;
      float g = 0.f;
      if (t < T) {
        for (int j = 0; j < K; ++j) {
          const int ej = s_idx[t * K + j];
          if (ej < 0 || ej >= E) {
            if (rank == 0 && cl == 0 && r0 == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_SHRINK, ej);
          } else if (ej == e) {
            g += s_gate[t * K + j];
          }
        }
      }
      if (args.direct) {
        // the final V: bf16 hi | lo blocks in the expand's K-major core-matrix layout (K chunk r0 / 8)
        __nv_bfloat16* vh = reinterpret_cast<__nv_bfloat16*>(ws_at<unsigned char>(a.ws, args.vpart_off) +
                                                             (size_t)p * 4 * Tp * NR);
        __nv_bfloat16* vl = vh + (size_t)Tp * NR;
        const float f[4] = {g * s.x, g * s.y, g * s.z, g * s.w};
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
          const float2 hf = __bfloat1622float2(hv);
          hi[i] = *reinterpret_cast<const uint32_t*>(&hv);
          lo[i] = pack_bf16x2(f[2 * i] - hf.x, f[2 * i + 1] - hf.y);
        }
        const size_t o = ((size_t)(t >> 3) * (NR / 8) + (size_t)(r0 >> 3)) * 64 + (size_t)(t & 7) * 8 + (size_t)(r0 & 7);
        *reinterpret_cast<uint2*>(vh + o) = make_uint2(hi[0], hi[1]);
        *reinterpret_cast<uint2*>(vl + o) = make_uint2(lo[0], lo[1]);
      } else {
        *reinterpret_cast<float4*>(vpart + (size_t)t * NR + r0) = make_float4(g * s.x, g * s.y, g * s.z, g * s.w);
      }
    }
  }
  if constexpr (MR != 128) cluster_wait();   // every CTA's reads of this CTA's P are over before it leaves
  if constexpr (MR == 128) {
    if (tid < CLT) bulk_wait_read_all();     // this CTA's outgoing copies have read P
  }
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

// ---------------------------------------------------------------- expand

template <int TP>
__global__ void __launch_bounds__(DN_THREADS, 1) dense_expand_kernel(const __grid_constant__ DenseArgs args) {
  const SgmmArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int Tp = TP;
  const int Rp = args.Rp, NR = args.NR;
  const int T = a.T, E = a.E;
  int p = 0;
  while (p + 1 < a.nproj && (int)blockIdx.x >= args.tiles_before[p + 1]) ++p;
  const int n0 = ((int)blockIdx.x - args.tiles_before[p]) * DN_NT;
  const int d_out = a.proj[p].d_out;
  const uint32_t SBO = (uint32_t)(NR / 8) * 128;     // next 8-row group of a K-major no-swizzle operand

  // shared memory: Bslice [128 x NR], V hi / lo [Tp x NR] (bf16, 8x16-byte core matrices),
  // y_base columns [Tp][128] bf16
  unsigned char* sB = smem;
  unsigned char* sVH = sB + (size_t)DN_NT * NR * 2;
  unsigned char* sVL = sVH + (size_t)Tp * NR * 2;
  __nv_bfloat16* sYB = reinterpret_cast<__nv_bfloat16*>(sVL + (size_t)Tp * NR * 2);
  unsigned char* meta = reinterpret_cast<unsigned char*>(sYB + (size_t)Tp * DN_NT);
  uint64_t* bar = reinterpret_cast<uint64_t*>(meta);                                  // [2]: MMA done, V landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + 16);
  const __nv_bfloat16** s_Bp = reinterpret_cast<const __nv_bfloat16**>(meta + 32);   // [E]
  int* s_rk = reinterpret_cast<int*>(meta + 32 + 8 * 16);                             // [E]

  pdl_trigger();                                     // as in the shrink: the next kernel may stage early
  const uint32_t cs = tmem_cols_for(Tp);
  const uint32_t ncols = 2 * cs;                     // the hi and lo products in two accumulators
  if (tid == 0) {
    mbar_init(smem_u32(bar), 2);
    mbar_init(smem_u32(bar + 1), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(s_tmem), ncols);
  if (tid < E) {
    s_Bp[tid] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[tid]);
    const int r = a.ranks[tid];
    s_rk[tid] = (r >= 8 && r <= Rp && (r & 7) == 0) ? r : 0;    // a bad rank is reported by the shrink
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // B slice of every adapter and the y_base columns: before the wait
  {
    const int kq_n = NR / 8, cq_n = Rp / 8;
    for (int w = tid; w < DN_NT * kq_n; w += DN_THREADS) {
      const int n = w / kq_n, kq = w - n * kq_n;
      const int e = kq / cq_n, cq = kq - e * cq_n;
      const bool valid = n0 + n < d_out && cq * 8 < s_rk[e];
      const void* src = valid ? (const void*)(s_Bp[e] + (size_t)(n0 + n) * s_rk[e] + cq * 8) : (const void*)a.x;
      cp_async16_zfill(smem_u32(sB) + (uint32_t)(n >> 3) * SBO + (uint32_t)kq * 128 + (uint32_t)(n & 7) * 16, src,
                       valid);
    }
    const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].y_base);
    for (int w = tid; w < T * (DN_NT / 8); w += DN_THREADS) {
      const int t = w >> 4, c = (w & 15) * 8;
      const bool valid = n0 + c < d_out;
      cp_async16_zfill(smem_u32(sYB + (size_t)t * DN_NT + c),
                       valid ? (const void*)(yb + (size_t)t * d_out + n0 + c) : (const void*)a.x, valid);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  pdl_wait();

  if (args.direct) {
    // the final V, already in the MMA layout: two contiguous bulk copies on the V barrier
    if (tid == 0) {
      const unsigned char* src = ws_at<unsigned char>(a.ws, args.vpart_off) + (size_t)p * 4 * Tp * NR;
      const uint32_t bytes = (uint32_t)(Tp * NR * 2);
      mbar_arrive_expect_tx(smem_u32(bar + 1), 2 * bytes);
      bulk_load_1d(smem_u32(sVH), src, bytes, smem_u32(bar + 1));
      bulk_load_1d(smem_u32(sVL), src + bytes, bytes, smem_u32(bar + 1));
    }
  } else {
  // V = sum over the clusters' gated partials (in order), split into bf16 hi + lo
  {
    const float* vp = ws_at<float>(a.ws, args.vpart_off) + (size_t)p * args.ncl * Tp * NR;
    const int kq_n = NR / 8;
    for (int w0 = tid; w0 < Tp * kq_n; w0 += DN_THREADS * 2) {
      // two 8-value chunks per thread; the cluster partials are summed in order,
      // two clusters' loads in flight per round
      float f[2][8];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) f[h][i] = 0.f;
      for (int c0 = 0; c0 < args.ncl; c0 += 2) {
        float4 ld[2][2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int w = w0 + h * DN_THREADS;
          const int t = w / kq_n, kq = w - t * kq_n;
#pragma unroll
          for (int dc = 0; dc < 2; ++dc) {
            const int c = c0 + dc;
            if (w < Tp * kq_n && c < args.ncl) {
              const float4* src = reinterpret_cast<const float4*>(vp + ((size_t)c * Tp + t) * NR + kq * 8);
              ld[h][dc][0] = __ldcg(src);
              ld[h][dc][1] = __ldcg(src + 1);
            } else {
              ld[h][dc][0] = ld[h][dc][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int dc = 0; dc < 2; ++dc) {
            const float4 u0 = ld[h][dc][0], u1 = ld[h][dc][1];
            f[h][0] += u0.x; f[h][1] += u0.y; f[h][2] += u0.z; f[h][3] += u0.w;
            f[h][4] += u1.x; f[h][5] += u1.y; f[h][6] += u1.z; f[h][7] += u1.w;
          }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
      const int w = w0 + h * DN_THREADS;
      if (w >= Tp * kq_n) continue;
      const int t = w / kq_n, kq = w - t * kq_n;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 hv = __floats2bfloat162_rn(f[h][2 * i], f[h][2 * i + 1]);
        const float2 hf = __bfloat1622float2(hv);
        hi[i] = *reinterpret_cast<const uint32_t*>(&hv);
        lo[i] = pack_bf16x2(f[h][2 * i] - hf.x, f[h][2 * i + 1] - hf.y);
      }
      const uint32_t off = (uint32_t)(t >> 3) * SBO + (uint32_t)kq * 128 + (uint32_t)(t & 7) * 16;
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(sVH) + off), "r"(hi[0]), "r"(hi[1]),
                   "r"(hi[2]), "r"(hi[3])
                   : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(sVL) + off), "r"(lo[0]), "r"(lo[1]),
                   "r"(lo[2]), "r"(lo[3])
                   : "memory");
      }
    }
  }
  }
  cp_async_wait_all();
  fence_proxy_async();
  __syncthreads();

  bool vready = true;
  const bool issuer = tid == 0 || tid == 32;         // thread 0: B . V_hi^T, thread 32: B . V_lo^T
  if (args.direct && issuer) vready = mbar_wait(smem_u32(bar + 1), 0);
  if (issuer && vready) {
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, Tp);
    const int h = tid >> 5;
    const uint32_t sv = h ? smem_u32(sVL) : smem_u32(sVH);
    for (int kk = 0; kk < NR / 16; ++kk)
      mma_bf16(tmem + (uint32_t)h * cs, desc_k_plain(smem_u32(sB) + kk * 256, 128, SBO),
               desc_k_plain(sv + kk * 256, 128, SBO), id, kk > 0 ? 1u : 0u);
    mma_commit(smem_u32(bar));
  }
  const bool done = __syncthreads_and(vready) && mbar_wait(smem_u32(bar), 0);
  tc_fence_after();
  if (!done) {
    if (tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_EXPAND, (int)blockIdx.x);
  } else {
    // thread n holds D[n][t] for its column: y_base[t, n] + D[n, t] in place in shared memory,
    // then whole 16-byte row pieces go out
    // (all TMEM loads of the warp before one wait; each group's y_base values are read before
    // any of them is written)
    const int wq = warp & 3, wg = warp >> 2;
    const int n = wq * 32 + lane;
    constexpr int NG = (TP / 8 + 1) / 2;
    const uint32_t lb = tmem + ((uint32_t)(wq * 32) << 16);
    uint32_t vh[NG][8], vl[NG][8];
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      const int c8 = wg + 2 * gi;
      if (c8 < TP / 8) {
        tmem_ld8_async(lb + (uint32_t)(c8 * 8), vh[gi]);
        tmem_ld8_async(lb + cs + (uint32_t)(c8 * 8), vl[gi]);
      }
    }
    tmem_ld_wait();
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      const int c8 = wg + 2 * gi;
      if (c8 < TP / 8) {
        tmem_ld_tie(vh[gi]);
        tmem_ld_tie(vl[gi]);
        float yv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) yv[u] = __bfloat162float(sYB[(size_t)(c8 * 8 + u) * DN_NT + n]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = c8 * 8 + u;
          if (t < T)
            sYB[(size_t)t * DN_NT + n] =
                __float2bfloat16_rn(yv[u] + (__uint_as_float(vh[gi][u]) + __uint_as_float(vl[gi][u])));
        }
      }
    }
  }
  __syncthreads();
  if (done) {
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.proj[p].y);
    for (int w = tid; w < T * (DN_NT / 8); w += DN_THREADS) {
      const int t = w >> 4, c = (w & 15) * 8;
      if (n0 + c < d_out)
        *reinterpret_cast<uint4*>(y + (size_t)t * d_out + n0 + c) = *reinterpret_cast<const uint4*>(sYB + (size_t)t * DN_NT + c);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

// ---------------------------------------------------------------- host side

static int dn_round16(int v) { return (v + 15) / 16 * 16; }

bool sgmm_dense_supported(const SgmmArgs& a, int dtype) {
  return dtype == APR_BF16 && dense_dims_ok(a.T, a.E, a.max_rank, a.d_in) && a.k <= APR_MAX_K;
}

static size_t shrink_smem(int MR, int Tp) {
  return (size_t)MR * 512 + (size_t)Tp * 512 + (MR == 128 ? (size_t)(Tp + 4) * MR * 4 : 0) + 32 + 8 * 16 + 4 * 16 +
         8 * 64 * APR_MAX_K + 1024;
}
static size_t expand_smem(int NR, int Tp) {
  return (size_t)DN_NT * NR * 2 + 2 * (size_t)Tp * NR * 2 + (size_t)Tp * DN_NT * 2 + 32 + 8 * 16 + 4 * 16 + 128;
}

static void shrink_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[2], int cl, int ncl, int nproj,
                          size_t smem, cudaStream_t s) {
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(cl, ncl, nproj);
  cfg.blockDim = dim3(DN_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cl;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
}

cudaError_t launch_sgmm_dense(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  DenseArgs d;
  memset(&d, 0, sizeof(d));
  d.a = a;
  d.Tp = dn_round16(a.T);
  d.Rp = dn_round16(a.max_rank);
  d.NR = a.E * d.Rp;
  d.MR = d.NR <= 128 ? 128 : 256;
  d.vpart_off = scratch_off;
  d.tiles_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) d.tiles_before[p + 1] = d.tiles_before[p] + (a.proj[p].d_out + DN_NT - 1) / DN_NT;

  const size_t sm1 = shrink_smem(d.MR, d.Tp), sm2 = expand_smem(d.NR, d.Tp);
  using Kern = void (*)(DenseArgs);
  const int ti = d.Tp / 16 - 1;
  // shrink variants: [rows 128, cluster 8] [rows 256, cluster 8] [rows 128, cluster 16]
  static const Kern shrinks[4][3] = {
      {dense_shrink_kernel<16, 128, 8>, dense_shrink_kernel<16, 256, 8>, dense_shrink_kernel<16, 128, 16>},
      {dense_shrink_kernel<32, 128, 8>, dense_shrink_kernel<32, 256, 8>, dense_shrink_kernel<32, 128, 16>},
      {dense_shrink_kernel<48, 128, 8>, dense_shrink_kernel<48, 256, 8>, dense_shrink_kernel<48, 128, 16>},
      {dense_shrink_kernel<64, 128, 8>, dense_shrink_kernel<64, 256, 8>, dense_shrink_kernel<64, 128, 16>}};
  static const Kern expands[4] = {dense_expand_kernel<16>, dense_expand_kernel<32>, dense_expand_kernel<48>,
                                  dense_expand_kernel<64>};
  static SmemLimit lim1[4][3], lim2[4];
  // whether a 16-CTA cluster of each token padding fits the device: 0 unknown, 1 yes, -1 no
  static std::mutex wide_mu;
  static int wide_ok[kMaxDevices][4] = {};
  cudaError_t err;
  int vi = d.MR == 128 ? 0 : 1;
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if (d.MR == 128 && dev >= 0 && dev < kMaxDevices) {
    // one 16-CTA cluster spans 4096 input columns; kept only where the device can place one
    if ((err = lim1[ti][2].ensure((const void*)shrinks[ti][2], sm1)) != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(wide_mu);
    if (wide_ok[dev][ti] == 0) {
      int nclus = 0;
      cudaLaunchConfig_t cfg;
      cudaLaunchAttribute attr[2];
      shrink_config(cfg, attr, 16, 1, 1, sm1, s);
      const bool ok = cudaFuncSetAttribute(shrinks[ti][2], cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                          cudaSuccess &&
                      cudaOccupancyMaxActiveClusters(&nclus, shrinks[ti][2], &cfg) == cudaSuccess && nclus >= 1;
      (void)cudaGetLastError();
      wide_ok[dev][ti] = ok ? 1 : -1;
    }
    if (wide_ok[dev][ti] > 0) vi = 2;
  }
  const int cl = vi == 2 ? 16 : DN_CL;
  d.ncl = (a.d_in + cl * DN_KC - 1) / (cl * DN_KC);
  d.direct = d.ncl == 1;
  const Kern k1 = shrinks[ti][vi], k2 = expands[ti];
  if ((err = lim1[ti][vi].ensure((const void*)k1, sm1)) != cudaSuccess) return err;
  if ((err = lim2[ti].ensure((const void*)k2, sm2)) != cudaSuccess) return err;
  {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    shrink_config(cfg, attr, cl, d.ncl, a.nproj, sm1, s);
    count_launch();
    if ((err = cudaLaunchKernelEx(&cfg, k1, d)) != cudaSuccess) return err;
  }
  return launch_pdl(k2, dim3(d.tiles_before[a.nproj]), dim3(DN_THREADS), sm2, s, d);
}

}  // namespace apr
