// Base projection and adapters in one tcgen05 contraction:
//
//   y[t, :] = x[t, :] W^T + sum_j g_{t,j} B_{e_{t,j}} (A_{e_{t,j}} x[t, :])
//
// with one fp32 accumulator and one rounding to bf16 per output element.
// AdaFuse summary (gist.science), Resumen tecnico §2.B: the selected experts
// are fused into the backbone in a single pass.  Where the adapter add runs
// after a separate base GEMM, every output element is written by the GEMM,
// read back and written again; here the adapter term enters the GEMM's own
// accumulator, so y is written once and never read.
//
// The adapter term is the bank form of the contraction (the bank SGMM kernel
// uses the same identity):
//
//   sum_j g_j B_{e_j} v_j = Bcat V_t,  V[t, e*R16 + r] = g_{t,j} (A_e x_t)[r] if idx[t, j] == e
//                                      Bcat[n, e*R16 + r] = B_e[n, r]
//
// so the whole projection is one GEMM over K = d_in + E*R16:
//
//   y = [x | V] [W | Bcat]^T
//
// Steps of one call (all on the caller's stream, chained by programmatic
// dependent launch):
//  1. the shrink, also on the tensor cores: each projection's adapters are
//     packed into one bank [E * R16, d_in] and x is contracted with the whole
//     bank by the same tile kernel (x by TMA, no gather); its epilogue keeps
//     each token's selected adapters' columns, times their gates, as g * A_e x
//     per (token, slot) in bf16;
//  2. a pack kernel spreads those rows over the bank's rank slots (V, zeros
//     where a token did not select an adapter) and lays the projection's B_e
//     side by side (Bcat), both row-major in the workspace;
//  3. the GEMM: 64-wide K blocks by 2-D TMA boxes (128-byte swizzle) into a
//     ring, x/W blocks first and V/Bcat blocks after them; one thread issues
//     the MMAs into a double-buffered TMEM accumulator; four epilogue warps
//     round and store while the next tile accumulates.  Above 128 tokens the
//     tiles are 256 x 256 and computed by CTA pairs (cta_group::2, below);
//     a single 128-token tile runs on one CTA (128 x 256, M = 128 MMAs).  The
//     grid is persistent, tiles ordered row tile fastest so that the CTAs in
//     flight share W's column block in L2.
//
// Every mbarrier wait is bounded (1 s); on expiry the CTA records
// APR_ERR_TIMEOUT, stops issuing, drains its copies and frees its TMEM.
#include "apr_internal.cuh"
#include "tc_ptx.cuh"

#include <algorithm>

namespace apr {

constexpr int LL_BM = 128;                        // tokens per tile (TMEM lanes)
constexpr int LL_BN = 256;                        // output columns per tile (MMA N)
constexpr int LL_BK = 64;                         // K per block (one 128-byte swizzle atom)
constexpr int LL_ST = 4;                          // ring depth
constexpr int LL_THREADS = 192;                   // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr uint32_t LL_ABYTES = LL_BM * 128;       // 16 KB
constexpr uint32_t LL_BBYTES = LL_BN * 128;       // 32 KB
constexpr uint32_t LL_STAGE = LL_ABYTES + LL_BBYTES;
constexpr uint32_t LL_TMEM_COLS = 512;            // two 256-column accumulators
constexpr size_t LL_SMEM = (size_t)LL_ST * LL_STAGE + 256 + 1024;

// One-CTA tile kernel, instantiated as the fused GEMM's (BN = 256, y stored) and as the bank
// shrink's (BN = 128, gated columns scattered to the pair rows): ring depth and TMEM from BN.
constexpr int EPI_STORE_Y = 0, EPI_SHRINK = 1, EPI_ROUTE = 2;
template <int BN> struct TileCfg {
  static constexpr uint32_t stage = LL_ABYTES + (uint32_t)BN * 128;
  static constexpr int st = BN >= 256 ? 4 : 6;
  static constexpr uint32_t tmem_cols = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr size_t smem = (size_t)st * stage + 256 + 1024;
};

// Tile order: groups of LL_GN column tiles (of all projections in a row); inside a group the
// row tile advances every LL_GN tiles.  The CTAs in flight at any time then cover a band of about
// (CTAs / LL_GN) row tiles x LL_GN column tiles, whose x rows and W columns both stay in L2,
// instead of every row tile of x against one column block.
constexpr int LL_GN = 8;
__device__ __forceinline__ void grouped_tile(int tile, int mt, int ncols, int& nt, int& m) {
  const int per_group = LL_GN * mt;
  const int g = tile / per_group, r = tile - g * per_group;
  const int width = min(LL_GN, ncols - g * LL_GN);       // the last group may be narrower
  m = r / width;
  nt = g * LL_GN + (r - m * width);
}

struct LinPlan {
  CUtensorMap xmap;                      // x [T, d_in]: boxes of 64 columns x 128 rows
  CUtensorMap wmap[APR_MAX_PROJ];        // W_p [d_out, d_in]: 64 x 256
  CUtensorMap vmap[APR_MAX_PROJ];        // V_p [T, NB]: 64 x 128
  CUtensorMap bmap[APR_MAX_PROJ];        // Bcat_p [d_out, NB]: 64 x 256
  void* y[APR_MAX_PROJ];
  int d_out[APR_MAX_PROJ];
  int nt_before[APR_MAX_PROJ + 1];       // prefix of column tiles per projection
  int nproj, T, nbase, nlora, mt;
  void* ws;
  // bank shrink: the gated v rows [proj][t * k + j][R16] bf16, the routing
  __nv_bfloat16* vc;
  const int32_t* idx;
  const float* gate;
  int k, E, R16;
  // router: top-k adapters and gates of every token
  int32_t* ridx;
  float* rgate;
};

template <int BN, int EPI>
__global__ void __launch_bounds__(LL_THREADS, 1) linear_tile_kernel(const __grid_constant__ LinPlan P) {
  using C = TileCfg<BN>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)C::st * C::stage);
  const uint32_t bar_full = smem_u32(bars);                 // [ST] a K block landed (TMA bytes)
  const uint32_t bar_empty = smem_u32(bars + C::st);        // [ST] its MMAs are done
  const uint32_t bar_dfull = smem_u32(bars + 2 * C::st);    // [2]  accumulator complete
  const uint32_t bar_dempty = smem_u32(bars + 2 * C::st + 2); // [2] accumulator read out
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * C::st + 4);
  int* s_consumed = reinterpret_cast<int*>(s_tmem + 1);

  if (tid == 0) {
    for (int i = 0; i < C::st; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_dfull + 8 * i, 1);
      mbar_init(bar_dempty + 8 * i, 4 * 32);
    }
    *s_consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(s_tmem), C::tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  pdl_trigger();
  pdl_wait();                                      // x, V and Bcat come from the preceding kernels

  const int mt = P.mt, nkb = P.nbase + P.nlora;
  const int total = P.nt_before[P.nproj] * mt;
  auto tile_at = [&](int tile, int& p, int& n0, int& m0) {
    int nt, m;
    grouped_tile(tile, mt, P.nt_before[P.nproj], nt, m);
    m0 = m * LL_BM;
    p = 0;
    while (p + 1 < P.nproj && nt >= P.nt_before[p + 1]) ++p;
    n0 = (nt - P.nt_before[p]) * BN;
  };
  bool abort = false;
  int issued = 0;                                  // K blocks issued by the producer

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int tile = blockIdx.x; tile < total && !abort; tile += gridDim.x) {
        int p, n0, m0;
        tile_at(tile, p, n0, m0);
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = issued % C::st;
          if (!mbar_wait(bar_empty + 8 * s, ((issued / C::st) & 1) ^ 1)) { abort = true; break; }
          const uint32_t sa = sbase + (uint32_t)s * C::stage, sb = sa + LL_ABYTES;
          mbar_arrive_expect_tx(bar_full + 8 * s, C::stage);
          if (kb < P.nbase) {
            tma_load_2d(sa, &P.xmap, kb * LL_BK, m0, bar_full + 8 * s);
            tma_load_2d(sb, &P.wmap[p], kb * LL_BK, n0, bar_full + 8 * s);
          } else {
            const int lb = kb - P.nbase;
            tma_load_2d(sa, &P.vmap[p], lb * LL_BK, m0, bar_full + 8 * s);
            tma_load_2d(sb, &P.bmap[p], lb * LL_BK, n0, bar_full + 8 * s);
          }
          ++issued;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t id = idesc_bf16(LL_BM, BN);
      int g = 0, it = 0;
      for (int tile = blockIdx.x; tile < total && !abort; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        if (!mbar_wait(bar_dempty + 8 * ab, ((it >> 1) & 1) ^ 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)ab * BN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % C::st;
          if (!mbar_wait(bar_full + 8 * s, (g / C::st) & 1)) { abort = true; break; }
          tc_fence_after();
          const uint32_t sa = sbase + (uint32_t)s * C::stage, sb = sa + LL_ABYTES;
#pragma unroll
          for (int kk = 0; kk < LL_BK / 16; ++kk)
            mma_bf16(d, desc_k_sw128(sa + kk * 32), desc_k_sw128(sb + kk * 32), id, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(bar_empty + 8 * s);           // the slot is free once these MMAs have read it
        }
        if (abort) break;
        mma_commit(bar_dfull + 8 * ab);
      }
      *s_consumed = g;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;                  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total && !abort; tile += gridDim.x, ++it) {
      int p, n0, m0;
      tile_at(tile, p, n0, m0);
      const int ab = it & 1;
      if (!mbar_wait(bar_dfull + 8 * ab, (it >> 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const int t = m0 + row, d_out = P.d_out[p];
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)ab * BN;
      if (EPI == EPI_ROUTE) {
        // the row's E logits (exact: products of bf16 values summed in fp32) -> the k largest,
        // the lower adapter index first among equal logits, then the softmax over them
        float tv[APR_MAX_K];
        int te[APR_MAX_K];
        float kth = -INFINITY;                                  // the k-th largest so far
#pragma unroll
        for (int j = 0; j < APR_MAX_K; ++j) {
          tv[j] = -INFINITY;
          te[j] = 0x7FFFFFFF;
        }
#pragma unroll 1
        for (int c32 = 0; c32 < BN / 32; ++c32) {
          float v[32];
          tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int e = n0 + c32 * 32 + u;
            float x = v[u];
            if (e >= P.E || !(x > kth)) continue;              // ascending e: an equal logit never displaces
            int xe = e;
#pragma unroll
            for (int j = 0; j < APR_MAX_K; ++j) {              // insertion, largest first; a displaced
              if (j < P.k && (x > tv[j] || (x == tv[j] && xe < te[j]))) {   // entry keeps index order
                const float sv = tv[j];
                const int se = te[j];
                tv[j] = x;
                te[j] = xe;
                x = sv;
                xe = se;
              }
            }
#pragma unroll
            for (int j = 0; j < APR_MAX_K; ++j)
              if (j == P.k - 1) kth = tv[j];
          }
        }
        bool short_k = false;
#pragma unroll
        for (int j = 0; j < APR_MAX_K; ++j)
          if (j == P.k - 1) short_k = te[j] == 0x7FFFFFFF;
        if (t < P.T) {
          if (short_k) {                                        // fewer than k non-NaN logits
            report(P.ws, APR_ERR_DEVICE_INDEX, K_TOPK, t);
#pragma unroll
            for (int j = 0; j < APR_MAX_K; ++j)
              if (te[j] == 0x7FFFFFFF) {
                te[j] = 0;
                tv[j] = 0.f;
              }
          }
          float w[APR_MAX_K], sum = 0.f;
#pragma unroll
          for (int j = 0; j < APR_MAX_K; ++j) {
            if (j >= P.k) break;
            w[j] = expf(tv[j] - tv[0]);
            sum += w[j];
          }
#pragma unroll
          for (int j = 0; j < APR_MAX_K; ++j) {
            if (j >= P.k) break;
            P.ridx[(size_t)t * P.k + j] = te[j];
            P.rgate[(size_t)t * P.k + j] = w[j] / sum;
          }
        }
      } else if (EPI == EPI_SHRINK) {
        // row t's bank columns n0 .. n0 + BN: the columns of each adapter the token selected,
        // times its gate, go to the token's pair row (t * k + j) of v
        int ej[APR_MAX_K];
        float gj[APR_MAX_K];
#pragma unroll
        for (int j = 0; j < APR_MAX_K; ++j) {
          ej[j] = -1;
          gj[j] = 0.f;
          if (j < P.k && t < P.T) {
            ej[j] = P.idx[(size_t)t * P.k + j];
            gj[j] = P.gate[(size_t)t * P.k + j];
            if (ej[j] < 0 || ej[j] >= P.E) {
              if (n0 == 0) report(P.ws, APR_ERR_DEVICE_INDEX, K_LINEAR, ej[j]);
              ej[j] = -1;
            }
          }
        }
        __nv_bfloat16* vrow = P.vc + ((size_t)p * P.T * P.k + (size_t)t * P.k) * P.R16;
#pragma unroll 1
        for (int c32 = 0; c32 < BN / 32; ++c32) {
          float v[32];
          tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = n0 + c32 * 32 + 16 * h;                 // first bank column of this half
#pragma unroll
            for (int j = 0; j < APR_MAX_K; ++j) {
              const int lo = ej[j] * P.R16;
              if (ej[j] >= 0 && c >= lo && c < lo + P.R16) {
                uint4 u[2];
                uint32_t* w = reinterpret_cast<uint32_t*>(u);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  const __nv_bfloat162 b2 =
                      __floats2bfloat162_rn(gj[j] * v[16 * h + 2 * q], gj[j] * v[16 * h + 2 * q + 1]);
                  w[q] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                uint4* dst = reinterpret_cast<uint4*>(vrow + (size_t)j * P.R16 + (c - lo));
                dst[0] = u[0];
                dst[1] = u[1];
              }
            }
          }
        }
      } else {
      __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(P.y[p]) + (size_t)t * d_out;
#pragma unroll 1
      for (int c32 = 0; c32 < BN / 32; ++c32) {
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
        const int col = n0 + c32 * 32;
        if (t < P.T) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (col + h * 8 < d_out) {
              uint4 u;
              uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[h * 8 + 2 * q], v[h * 8 + 2 * q + 1]);
                w[q] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(yrow + col + h * 8) = u;
            }
          }
        }
      }
      }
      tc_fence_before();
      mbar_arrive(bar_dempty + 8 * ab);
    }
  }
  abort = __syncthreads_or(abort);
  if (abort) {
    if (tid == 0) report(P.ws, APR_ERR_TIMEOUT, K_LINEAR, (int)blockIdx.x);
    // copies issued but never consumed land before the shared memory is released
    if (warp == 0 && lane == 0)
      for (int g = *s_consumed; g < issued; ++g) (void)mbar_wait(bar_full + 8 * (g % C::st), (g / C::st) & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C::tmem_cols);
}

// ---------------------------------------------------------------- CTA pairs
// The same contraction on 256 x 256 tiles computed by a pair of CTAs (a cluster of two) with
// one MMA stream (tcgen05 cta_group::2): each CTA loads its 128 token rows of the A operand and
// its 128 of the 256 output columns of the B operand, the leader issues M = 256, N = 256 MMAs
// that read both CTAs' shared memory, and each CTA's TMEM receives its 128 rows of D.  Per SM
// that is half the operand bytes of the one-CTA tile for the same MMA work.  All the loads of a
// K block complete on the leader's barrier; the leader's commits free the slot in both CTAs and
// hand each CTA's epilogue its accumulator; each epilogue warp returns the accumulator to the
// leader with a remote arrive.

constexpr int L2_ST = 6;                          // ring depth (32 KB per stage per CTA)
constexpr uint32_t L2_STAGE = 2 * 128 * 128;      // A 128 x 64 and B 128 x 64, bf16
constexpr size_t L2_SMEM = (size_t)L2_ST * L2_STAGE + 256 + 1024;

__global__ void __launch_bounds__(LL_THREADS, 1) linear_lora_pair_kernel(const __grid_constant__ LinPlan P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();            // 0: leader (issues the MMAs), 1: peer
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)L2_ST * L2_STAGE);
  const uint32_t bar_full = smem_u32(bars);                  // [ST] leader: both CTAs' K block landed
  const uint32_t bar_empty = smem_u32(bars + L2_ST);         // [ST] the slot's MMAs are done
  const uint32_t bar_dfull = smem_u32(bars + 2 * L2_ST);     // [2]  accumulator complete
  const uint32_t bar_dempty = smem_u32(bars + 2 * L2_ST + 2);// [2]  leader: read out by 8 epilogue warps
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * L2_ST + 4);
  int* s_consumed = reinterpret_cast<int*>(s_tmem + 1);      // leader: K blocks the MMAs took
  int* s_issued = s_consumed + 1;                            // leader: [2] K blocks each producer issued

  if (tid == 0) {
    for (int i = 0; i < L2_ST; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_dfull + 8 * i, 1);
      mbar_init(bar_dempty + 8 * i, 8);
    }
    *s_consumed = 0;
    s_issued[0] = s_issued[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc_pair(smem_u32(s_tmem), LL_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                              // both CTAs' barriers and TMEM exist
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  pdl_trigger();
  pdl_wait();

  const int mt = P.mt, nkb = P.nbase + P.nlora;   // mt: 256-row tiles
  const int total = P.nt_before[P.nproj] * mt;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  auto tile_at = [&](int tile, int& p, int& n0, int& m0) {
    int nt, m;
    grouped_tile(tile, mt, P.nt_before[P.nproj], nt, m);
    m0 = m * 2 * LL_BM;
    p = 0;
    while (p + 1 < P.nproj && nt >= P.nt_before[p + 1]) ++p;
    n0 = (nt - P.nt_before[p]) * LL_BN;
  };
  bool abort = false;
  int issued = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = cluster_map(bar_full, 0);
      for (int tile = pair; tile < total && !abort; tile += npairs) {
        int p, n0, m0;
        tile_at(tile, p, n0, m0);
        const int ma = m0 + (int)rank * LL_BM, nb = n0 + (int)rank * (LL_BN / 2);
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = issued % L2_ST;
          if (!mbar_wait(bar_empty + 8 * s, ((issued / L2_ST) & 1) ^ 1)) { abort = true; break; }
          const uint32_t sa = sbase + (uint32_t)s * L2_STAGE, sb = sa + L2_STAGE / 2;
          if (rank == 0) mbar_arrive_expect_tx(bar_full + 8 * s, 2 * L2_STAGE);
          if (kb < P.nbase) {
            tma_load_2d_pair(sa, &P.xmap, kb * LL_BK, ma, full_leader + 8 * s);
            tma_load_2d_pair(sb, &P.wmap[p], kb * LL_BK, nb, full_leader + 8 * s);
          } else {
            const int lb = kb - P.nbase;
            tma_load_2d_pair(sa, &P.vmap[p], lb * LL_BK, ma, full_leader + 8 * s);
            tma_load_2d_pair(sb, &P.bmap[p], lb * LL_BK, nb, full_leader + 8 * s);
          }
          ++issued;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue (leader)
    if (lane == 0 && rank == 0) {
      const uint32_t id = idesc_bf16(2 * LL_BM, LL_BN);
      int g = 0, it = 0;
      for (int tile = pair; tile < total && !abort; tile += npairs, ++it) {
        const int ab = it & 1;
        if (!mbar_wait(bar_dempty + 8 * ab, ((it >> 1) & 1) ^ 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)ab * LL_BN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % L2_ST;
          if (!mbar_wait(bar_full + 8 * s, (g / L2_ST) & 1)) { abort = true; break; }
          tc_fence_after();
          const uint32_t sa = sbase + (uint32_t)s * L2_STAGE, sb = sa + L2_STAGE / 2;
#pragma unroll
          for (int kk = 0; kk < LL_BK / 16; ++kk)
            mma_bf16_pair(d, desc_k_sw128(sa + kk * 32), desc_k_sw128(sb + kk * 32), id, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_pair(bar_empty + 8 * s, 3);   // the slot is free in both CTAs
        }
        if (abort) break;
        mma_commit_pair(bar_dfull + 8 * ab, 3);    // both halves of D are complete
      }
      *s_consumed = g;
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t dempty_leader = cluster_map(bar_dempty, 0);
    int it = 0;
    for (int tile = pair; tile < total && !abort; tile += npairs, ++it) {
      int p, n0, m0;
      tile_at(tile, p, n0, m0);
      const int ab = it & 1;
      if (!mbar_wait(bar_dfull + 8 * ab, (it >> 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const int t = m0 + (int)rank * LL_BM + row, d_out = P.d_out[p];
      __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(P.y[p]) + (size_t)t * d_out;
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)ab * LL_BN;
#pragma unroll 1
      for (int c32 = 0; c32 < LL_BN / 32; ++c32) {
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
        const int col = n0 + c32 * 32;
        if (t < P.T) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (col + h * 8 < d_out) {
              uint4 u;
              uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[h * 8 + 2 * q], v[h * 8 + 2 * q + 1]);
                w[q] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(yrow + col + h * 8) = u;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(dempty_leader + 8 * ab);
    }
  }
  abort = __syncthreads_or(abort);
  // the producers' counts go to the leader, so that after a timeout it can wait for every copy
  // still in flight (their bytes complete on its barriers) before either CTA releases its memory
  if (warp == 0 && lane == 0)
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_map(smem_u32(s_issued + rank), 0)), "r"(issued)
                 : "memory");
  cluster_sync_all();
  const bool any_abort = abort || s_issued[0] != *s_consumed || s_issued[1] != *s_consumed;
  if (rank == 0 && any_abort) {
    if (tid == 0) report(P.ws, APR_ERR_TIMEOUT, K_LINEAR, (int)blockIdx.x);
    if (warp == 0 && lane == 0) {
      const int most = max(s_issued[0], s_issued[1]);
      for (int g = *s_consumed; g < most; ++g) (void)mbar_wait(bar_full + 8 * (g % L2_ST), (g / L2_ST) & 1);
    }
  } else if (rank == 1 && abort && tid == 0) {
    report(P.ws, APR_ERR_TIMEOUT, K_LINEAR, (int)blockIdx.x);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                              // no copy or remote arrive still targets either CTA
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem, LL_TMEM_COLS);
}

// ---------------------------------------------------------------- V and Bcat

struct PackArgs {
  const __nv_bfloat16* vc;               // gated v rows [proj][t * k + j][R16]
  __nv_bfloat16* V;                      // [proj][T][NB]
  __nv_bfloat16* Bcat[APR_MAX_PROJ];     // [d_out_p][NB]
  const void* const* B[APR_MAX_PROJ];
  int d_out[APR_MAX_PROJ];
  const int32_t* idx;
  const int32_t* ranks;
  int T, k, E, R16, NB, nproj;
  void* ws;
};

// One 16-byte chunk (8 rank slots) per thread step.  blockIdx.y = 0: the V rows of every
// projection (row = proj * T + t, whose gated v rows start at vc + row * k * R16);
// blockIdx.y = 1 + p: projection p's Bcat.
__global__ void __launch_bounds__(256) linear_pack_kernel(const __grid_constant__ PackArgs a) {
  pdl_wait();                                      // the shrink's rows, and the buffers' last readers
  pdl_trigger();
  const int cpr = a.NB / 8;                        // chunks per bank row
  const int stride = gridDim.x * blockDim.x;
  if (blockIdx.y == 0) {
    const int total = a.nproj * a.T * cpr;
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += stride) {
      const int row = w / cpr, c = w - row * cpr;
      const int t = row % a.T;
      const int e = c * 8 / a.R16, r0 = c * 8 - e * a.R16;
      uint4 val = make_uint4(0, 0, 0, 0);
      for (int j = 0; j < a.k; ++j) {
        const int ej = __ldg(a.idx + (size_t)t * a.k + j);
        if (ej == e) val = *reinterpret_cast<const uint4*>(a.vc + ((size_t)row * a.k + j) * a.R16 + r0);
        else if ((ej < 0 || ej >= a.E) && c == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_LINEAR, ej);
      }
      *reinterpret_cast<uint4*>(a.V + (size_t)row * a.NB + c * 8) = val;
    }
  } else {
    const int p = blockIdx.y - 1;
    const __nv_bfloat16* const* Bp = reinterpret_cast<const __nv_bfloat16* const*>(a.B[p]);
    __nv_bfloat16* dst = a.Bcat[p];
    const int total = a.d_out[p] * cpr;
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += stride) {
      const int n = w / cpr, c = w - n * cpr;
      const int e = c * 8 / a.R16, r0 = c * 8 - e * a.R16;
      const int re = __ldg(a.ranks + e);
      const bool rank_ok = re >= 8 && re <= a.R16 && (re & 7) == 0;
      if (!rank_ok && n == 0 && r0 == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_LINEAR, e);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (rank_ok && r0 < re) val = *reinterpret_cast<const uint4*>(Bp[e] + (size_t)n * re + r0);
      *reinterpret_cast<uint4*>(dst + (size_t)n * a.NB + c * 8) = val;
    }
  }
}

// ---------------------------------------------------------------- bank shrink
// The shrink of the bank form: for each projection, S = x . Abank^T with Abank[e * R16 + i] =
// A_e[i] (zero rows past an adapter's rank), one GEMM over the whole bank (E/k times the
// products of the gathered shrink, on the tensor cores), x read by contiguous TMA boxes instead
// of gathered rows.  Its epilogue keeps, for every token, the columns of the adapters it
// selected, scaled by their gates, and writes them to the token's pair rows of v.

struct APackArgs {
  const void* const* A[APR_MAX_PROJ];
  __nv_bfloat16* Ab[APR_MAX_PROJ];       // [E * R16][d_in]
  const int32_t* ranks;
  int E, R16, d_in;
  void* ws;
};

// one 16-byte chunk per thread step; blockIdx.y: the projection
__global__ void __launch_bounds__(256) bank_pack_a_kernel(const __grid_constant__ APackArgs a) {
  pdl_wait();                                      // the bank buffer's last readers
  pdl_trigger();
  const int p = blockIdx.y;
  const __nv_bfloat16* const* Ap = reinterpret_cast<const __nv_bfloat16* const*>(a.A[p]);
  __nv_bfloat16* dst = a.Ab[p];
  const int cpr = a.d_in / 8;
  const int total = a.E * a.R16 * cpr;
  for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += gridDim.x * blockDim.x) {
    const int row = w / cpr, c = w - row * cpr;
    const int e = row / a.R16, i = row - e * a.R16;
    const int re = __ldg(a.ranks + e);
    const bool ok = re >= 8 && re <= a.R16 && (re & 7) == 0;
    if (!ok && i == 0 && c == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_LINEAR, e);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (ok && i < re) val = *reinterpret_cast<const uint4*>(Ap[e] + (size_t)i * a.d_in + c * 8);
    *reinterpret_cast<uint4*>(dst + (size_t)row * a.d_in + c * 8) = val;
  }
}

cudaError_t launch_bank_shrink(const SgmmArgs& a, size_t vc_off, size_t abank_off, cudaStream_t s) {
  constexpr int BN = 128;
  const int R16 = round16i(a.max_rank), NB = a.E * R16;
  APackArgs pk;
  memset(&pk, 0, sizeof(pk));
  pk.ranks = a.ranks;
  pk.E = a.E;
  pk.R16 = R16;
  pk.d_in = a.d_in;
  pk.ws = a.ws;
  LinPlan P;
  memset(&P, 0, sizeof(P));
  cudaError_t err;
  if ((err = encode_tile_map(&P.xmap, a.x, a.T, a.d_in, LL_BM)) != cudaSuccess) return err;
  P.nt_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) {
    pk.A[p] = a.proj[p].A;
    pk.Ab[p] = ws_at<__nv_bfloat16>(a.ws, abank_off + (size_t)p * NB * a.d_in * 2);
    if ((err = encode_tile_map(&P.wmap[p], pk.Ab[p], NB, a.d_in, BN)) != cudaSuccess) return err;
    P.d_out[p] = NB;
    P.nt_before[p + 1] = P.nt_before[p] + (NB + BN - 1) / BN;
  }
  P.nproj = a.nproj;
  P.T = a.T;
  P.nbase = a.d_in / LL_BK;
  P.nlora = 0;
  P.mt = (a.T + LL_BM - 1) / LL_BM;
  P.ws = a.ws;
  P.vc = ws_at<__nv_bfloat16>(a.ws, vc_off);
  P.idx = a.idx;
  P.gate = a.gate;
  P.k = a.k;
  P.E = a.E;
  P.R16 = R16;
  static SmemLimit lim;
  using Cfg = TileCfg<BN>;
  if ((err = lim.ensure((const void*)linear_tile_kernel<BN, EPI_SHRINK>, Cfg::smem)) != cudaSuccess) return err;
  const int nsm = device_sm_count();
  const int chunks = NB * (a.d_in / 8);
  const int pgrid = std::min((chunks + 255) / 256, 2 * nsm);
  if ((err = launch_pdl(bank_pack_a_kernel, dim3(pgrid, a.nproj), dim3(256), 0, s, pk)) != cudaSuccess) return err;
  const long tiles = (long)P.nt_before[a.nproj] * P.mt;
  const int grid = (int)std::min<long>(tiles, nsm);
  return launch_pdl(linear_tile_kernel<BN, EPI_SHRINK>, dim3(grid), dim3(LL_THREADS), Cfg::smem, s, P);
}

// ---------------------------------------------------------------- router on the tensor cores
// Logits L = h Wr^T for a bank of at most 256 adapters as one tile GEMM (h and Wr by TMA, M = 128
// tokens, N = the bank padded to 64/128/256), top-k and gates in the epilogue from TMEM: one
// launch, no partials in memory.

bool route_tc_supported(int dtype, int d, int E, const void* h, const void* Wr) {
  return dtype == APR_BF16 && d % LL_BK == 0 && E >= 1 && E <= 256 &&
         reinterpret_cast<uintptr_t>(h) % 16 == 0 && reinterpret_cast<uintptr_t>(Wr) % 16 == 0;
}

template <int BN>
static cudaError_t launch_route_tc_bn(LinPlan& P, cudaStream_t s) {
  static SmemLimit lim;
  using Cfg = TileCfg<BN>;
  cudaError_t err;
  if ((err = lim.ensure((const void*)linear_tile_kernel<BN, EPI_ROUTE>, Cfg::smem)) != cudaSuccess) return err;
  const int grid = std::min(P.mt, device_sm_count());
  return launch_pdl(linear_tile_kernel<BN, EPI_ROUTE>, dim3(grid), dim3(LL_THREADS), Cfg::smem, s, P);
}

cudaError_t launch_route_tc(const void* h, const void* Wr, int T, int d, int E, int k, int32_t* idx, float* gate,
                            void* ws, cudaStream_t s) {
  const int BN = E <= 64 ? 64 : (E <= 128 ? 128 : 256);
  LinPlan P;
  memset(&P, 0, sizeof(P));
  cudaError_t err;
  if ((err = encode_tile_map(&P.xmap, h, T, d, LL_BM)) != cudaSuccess) return err;
  if ((err = encode_tile_map(&P.wmap[0], Wr, E, d, BN)) != cudaSuccess) return err;
  P.nt_before[0] = 0;
  P.nt_before[1] = 1;
  P.d_out[0] = E;
  P.nproj = 1;
  P.T = T;
  P.nbase = d / LL_BK;
  P.nlora = 0;
  P.mt = (T + LL_BM - 1) / LL_BM;
  P.ws = ws;
  P.k = k;
  P.E = E;
  P.ridx = idx;
  P.rgate = gate;
  if (BN == 64) return launch_route_tc_bn<64>(P, s);
  if (BN == 128) return launch_route_tc_bn<128>(P, s);
  return launch_route_tc_bn<256>(P, s);
}

// ---------------------------------------------------------------- host side

bool linear_lora_supported(const SgmmArgs& a) { return sgmm_bank_supported(a, APR_BF16); }

cudaError_t launch_linear_lora(const SgmmArgs& a, const void* const* W, size_t scratch_off, cudaStream_t s) {
  const int R16 = round16i(a.max_rank), NB = a.E * R16;
  const LinearScratch L = linear_scratch(a.T, a.k, a.E, a.max_rank, a.nproj, a.d_in);
  PackArgs pk;
  memset(&pk, 0, sizeof(pk));
  pk.vc = ws_at<__nv_bfloat16>(a.ws, scratch_off + L.vc);
  pk.V = ws_at<__nv_bfloat16>(a.ws, scratch_off + L.v);
  pk.idx = a.idx;
  pk.ranks = a.ranks;
  pk.T = a.T;
  pk.k = a.k;
  pk.E = a.E;
  pk.R16 = R16;
  pk.NB = NB;
  pk.nproj = a.nproj;
  pk.ws = a.ws;
  size_t boff = scratch_off + L.bcat;
  long most = (long)a.nproj * a.T * (NB / 8);     // chunks of the largest role
  for (int p = 0; p < a.nproj; ++p) {
    pk.Bcat[p] = ws_at<__nv_bfloat16>(a.ws, boff);
    pk.B[p] = a.proj[p].B;
    pk.d_out[p] = a.proj[p].d_out;
    most = std::max(most, (long)a.proj[p].d_out * (NB / 8));
    boff += align_up((size_t)a.proj[p].d_out * NB * 2);
  }

  // CTA pairs (256-token tiles) unless the call has a single 128-token tile
  const bool pairs = a.T > LL_BM;
  const int brows = pairs ? LL_BN / 2 : LL_BN;     // rows of a B box: the CTA's share of the N columns
  LinPlan P;
  memset(&P, 0, sizeof(P));
  cudaError_t err;
  if ((err = encode_tile_map(&P.xmap, a.x, a.T, a.d_in, LL_BM)) != cudaSuccess) return err;
  P.nt_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) {
    const int d_out = a.proj[p].d_out;
    if ((err = encode_tile_map(&P.wmap[p], W[p], d_out, a.d_in, brows)) != cudaSuccess) return err;
    if ((err = encode_tile_map(&P.vmap[p], pk.V + (size_t)p * a.T * NB, a.T, NB, LL_BM)) != cudaSuccess) return err;
    if ((err = encode_tile_map(&P.bmap[p], pk.Bcat[p], d_out, NB, brows)) != cudaSuccess) return err;
    P.y[p] = a.proj[p].y;
    P.d_out[p] = d_out;
    P.nt_before[p + 1] = P.nt_before[p] + (d_out + LL_BN - 1) / LL_BN;
  }
  P.nproj = a.nproj;
  P.T = a.T;
  P.nbase = (a.d_in + LL_BK - 1) / LL_BK;
  P.nlora = (NB + LL_BK - 1) / LL_BK;
  const int tile_rows = pairs ? 2 * LL_BM : LL_BM;
  P.mt = (a.T + tile_rows - 1) / tile_rows;
  P.ws = a.ws;

  static SmemLimit lim, lim2;
  if ((err = lim.ensure((const void*)linear_tile_kernel<LL_BN, EPI_STORE_Y>, TileCfg<LL_BN>::smem)) != cudaSuccess)
    return err;
  if ((err = lim2.ensure((const void*)linear_lora_pair_kernel, L2_SMEM)) != cudaSuccess) return err;
  if ((err = launch_bank_shrink(a, scratch_off + L.vc, scratch_off + L.abank, s)) != cudaSuccess) return err;
  const int nsm = device_sm_count();
  const int pgrid = (int)std::min<long>((most + 255) / 256, 4L * nsm);
  if ((err = launch_pdl(linear_pack_kernel, dim3(pgrid, 1 + a.nproj), dim3(256), 0, s, pk)) != cudaSuccess) return err;
  const long tiles = (long)P.nt_before[a.nproj] * P.mt;
  if (!pairs) {
    const int grid = (int)std::min<long>(tiles, nsm);
    return launch_pdl(linear_tile_kernel<LL_BN, EPI_STORE_Y>, dim3(grid), dim3(LL_THREADS), TileCfg<LL_BN>::smem, s, P);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(2 * (unsigned)std::min<long>(tiles, nsm / 2));
  cfg.blockDim = dim3(LL_THREADS);
  cfg.dynamicSmemBytes = L2_SMEM;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, linear_lora_pair_kernel, P);
}

}  // namespace apr
