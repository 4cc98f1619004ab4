// Batch-1 merge on the 5th-generation tensor cores (tcgen05).
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int TC_THREADS = 128;
constexpr int TC_BM = 128;                      // rows of W per strip
constexpr int TC_MAXN1 = 64;                    // k * rank (rounded up to 16)
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr uint32_t TC_D2_COL = 128;             // D buffers at columns 128 and 256

static int round16(int r) { return (r + 15) / 16 * 16; }

// Batch-1 merge (AdaFuse summary §2.B decoding steps 3 and 5), every weight in
// one launch, out of place:  W' = W + sum_j g_j B_{e_j} A_{e_j}.
// A work item is a strip of 128 rows of one weight.  The strip's gated B rows
// Bg[n][j*R16 + i] = g_j B_{e_j}[n][i] are formed once (fp32 -> bf16 hi + lo,
// K-major), then for every 128-column tile: D[128 x 128] = Bg_hi.A^T +
// Bg_lo.A^T on tcgen05 with A^T as an MN-major operand (rows of A_e are
// contiguous along the output columns), TMEM double buffered; the W tile and
// the A tile arrive two tiles ahead by cp.async into 3-deep rings, and the
// epilogue adds D to W in fp32, rounds once and the warp writes its 32 rows
// of W' back with coalesced 128-bit stores (merge_tc_kernel).
// merge_tma_kernel does the same with the W tiles loaded and the W' tiles
// stored by 2-D TMA boxes (64 columns x 128 rows, 128-byte swizzle) from
// tensor maps built once per weight set (apr_merge_plan_init); the W tile
// lands on a transaction-count mbarrier and the epilogue adds D in shared
// memory before one thread stores the tile.

constexpr int MT_BN = 128;                      // columns per tile
constexpr int MT_NY = 3;                        // ring depth
constexpr int MT_WSTRIDE = MT_BN * 2 + 16;      // bytes per staged W row
constexpr int MT_WBUF = TC_BM * MT_WSTRIDE;
constexpr int MT_ABUF = MT_BN * TC_MAXN1 * 2;   // MN-major A^T tile
constexpr int MT_MAXPROJ = 4096;

struct MtSmem {
  static constexpr size_t GH = 0;                                        // 16 KB
  static constexpr size_t GL = GH + (size_t)TC_BM * TC_MAXN1 * 2;        // 16 KB
  static constexpr size_t WR = GL + (size_t)TC_BM * TC_MAXN1 * 2;        // W ring
  static constexpr size_t AR = WR + (size_t)MT_NY * MT_WBUF;             // A ring
  static constexpr size_t BAR = AR + (size_t)MT_NY * MT_ABUF;
  static constexpr size_t META = BAR + 2 * 8;
  static constexpr size_t PREF = META + 128;                             // [nproj + 1] strip prefix
  static constexpr size_t fixed_bytes() { return PREF + 1024; }
};

// K-major A operand / MN-major B operand instruction descriptor (bf16 -> fp32).
__host__ __device__ constexpr uint32_t idesc_bf16_bmn(int M, int N) { return idesc_bf16(M, N) | (1u << 16); }

__global__ void __launch_bounds__(TC_THREADS, 1) merge_tc_kernel(const apr_merge_proj* __restrict__ projs,
                                                                 int nproj, int E, int r, int R16,
                                                                 const int32_t* __restrict__ idx,
                                                                 const float* __restrict__ gate, int k,
                                                                 void* ws) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = k * R16;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + MtSmem::BAR);
  const uint32_t bar_mma = smem_u32(bars);                     // [2]
  volatile int* s_flags = reinterpret_cast<volatile int*>(smem + MtSmem::META);   // [0] tmem, [1] bad
  int* s_e = const_cast<int*>(s_flags) + 4;                    // [<= 8]
  float* s_g = reinterpret_cast<float*>(s_e + 8);              // [<= 8]
  int* s_pref = reinterpret_cast<int*>(smem + MtSmem::PREF);
  const uint32_t sGH = smem_u32(smem + MtSmem::GH);
  const uint32_t sGL = smem_u32(smem + MtSmem::GL);
  unsigned char* sWp = smem + MtSmem::WR;
  const uint32_t sW = smem_u32(sWp);
  const uint32_t sA = smem_u32(smem + MtSmem::AR);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(bar_mma + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_flags[1] = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<int*>(s_flags))),
                 "r"(TC_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)s_flags[0];
  pdl_wait();
  pdl_trigger();

  if (tid < k) {
    const int e = idx[tid];
    if (e < 0 || e >= E) s_flags[1] = 1;
    s_e[tid] = e;
    s_g[tid] = gate[tid];
  }
  // strips (128 rows) per weight, prefix over the weights
  if (tid == 0) {
    int acc = 0;
    s_pref[0] = 0;
    for (int p = 0; p < nproj; ++p) {
      acc += (projs[p].d_out + TC_BM - 1) / TC_BM;
      s_pref[p + 1] = acc;
    }
  }
  __syncthreads();
  bool abort = false;
  if (s_flags[1]) {
    if (tid == 0 && blockIdx.x == 0) report(ws, APR_ERR_DEVICE_INDEX, K_MERGE, 0);
  } else {
    const int total = s_pref[nproj];
    const uint32_t sbo_g = (uint32_t)(K / 8) * 128;         // Bg: next 8-row group
    const uint32_t id = idesc_bf16_bmn(TC_BM, MT_BN);
    uint32_t ph_mma = 0;
    for (int strip = blockIdx.x; strip < total && !abort; strip += gridDim.x) {
      int lo = 0, hi = nproj;                                 // weight of this strip
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pref[mid] <= strip) lo = mid; else hi = mid;
      }
      const apr_merge_proj pj = projs[lo];
      const int row0 = (strip - s_pref[lo]) * TC_BM;
      const int nrows = min(TC_BM, pj.d_out - row0);
      const __nv_bfloat16* __restrict__ Wt = reinterpret_cast<const __nv_bfloat16*>(pj.W);
      __nv_bfloat16* __restrict__ Wp = reinterpret_cast<__nv_bfloat16*>(pj.Wp);
      // gated B rows of the strip, bf16 hi + lo, K-major
      {
        const int n = row0 + tid;
        for (int j = 0; j < k; ++j) {
          const __nv_bfloat16* B = reinterpret_cast<const __nv_bfloat16*>(pj.B[s_e[j]]);
          for (int c8 = 0; c8 < R16; c8 += 8) {
            float f[8];
            if (tid < nrows && c8 < r) {
              load8(B + (size_t)n * r + c8, f);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] = 0.f;
            }
            uint32_t h4[4], l4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float a0 = f[2 * i] * s_g[j], a1 = f[2 * i + 1] * s_g[j];
              const __nv_bfloat162 hh = __floats2bfloat162_rn(a0, a1);
              const float2 hf = __bfloat1622float2(hh);
              h4[i] = *reinterpret_cast<const uint32_t*>(&hh);
              l4[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
            }
            const int kc8 = (j * R16 + c8) >> 3;
            const uint32_t off = (uint32_t)(tid >> 3) * sbo_g + (uint32_t)kc8 * 128 + (uint32_t)(tid & 7) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sGH + off), "r"(h4[0]), "r"(h4[1]),
                         "r"(h4[2]), "r"(h4[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sGL + off), "r"(l4[0]), "r"(l4[1]),
                         "r"(l4[2]), "r"(l4[3])
                         : "memory");
          }
        }
      }
      fence_proxy_async();                       // Bg was written by ordinary stores
      const int nct = (pj.d_in + MT_BN - 1) / MT_BN;
      auto issue_tile = [&](int ct) {
        const int slot = ct % MT_NY;
        const int c0 = ct * MT_BN;
        const int ncols = min(MT_BN, pj.d_in - c0);
        // A^T tile, MN-major: core matrix (8 columns x 8 rank rows) at (col/8)*128 + (kk/8)*2048
        const uint32_t abase = sA + (uint32_t)slot * MT_ABUF;
        for (int w = tid; w < K * (MT_BN / 8); w += TC_THREADS) {
          const int kk = w / (MT_BN / 8), c = w % (MT_BN / 8);
          const int j = kk / R16, i = kk % R16;
          const uint32_t dst = abase + (uint32_t)c * 128 + (uint32_t)(kk >> 3) * 2048 + (uint32_t)(kk & 7) * 16;
          const bool valid = i < r && c * 8 < ncols;
          const __nv_bfloat16* A = reinterpret_cast<const __nv_bfloat16*>(pj.A[s_e[j]]);
          cp_async16_zfill(dst, valid ? A + (size_t)i * pj.d_in + c0 + c * 8 : A, valid);
        }
        // W rows of the tile: 16 lanes per 256-byte row segment, 2 rows per instruction
        const uint32_t wbase = sW + (uint32_t)slot * MT_WBUF;
        const int ch = lane & 15;
        if (ch * 8 < ncols) {
#pragma unroll 4
          for (int k2 = 0; k2 < 16; ++k2) {
            const int row = warp * 32 + 2 * k2 + (lane >> 4);
            if (row < nrows)
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(wbase + (uint32_t)row * MT_WSTRIDE + ch * 16),
                           "l"(Wt + (size_t)(row0 + row) * pj.d_in + c0 + ch * 8)
                           : "memory");
          }
        }
      };
      for (int ct = 0; ct < MT_NY - 1; ++ct) {
        if (ct < nct) issue_tile(ct);
        cp_async_commit();
      }
      for (int ct = 0; ct < nct; ++ct) {
        const int b = ct & 1;
        const int slot = ct % MT_NY;
        const int c0 = ct * MT_BN;
        const int ncols = min(MT_BN, pj.d_in - c0);
        if (ct + MT_NY - 1 < nct) issue_tile(ct + MT_NY - 1);
        cp_async_commit();
        cp_async_wait<MT_NY - 1>();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const uint32_t ab = sA + (uint32_t)slot * MT_ABUF;
          const uint32_t dcol = tmem + TC_D2_COL + (uint32_t)b * MT_BN;
          for (int kk = 0; kk < K / 16; ++kk)
            mma_bf16(dcol, desc_k_plain(sGH + kk * 256, 128, sbo_g), desc_k_plain(ab + kk * 4096, 2048, 128), id,
                     kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < K / 16; ++kk)
            mma_bf16(dcol, desc_k_plain(sGL + kk * 256, 128, sbo_g), desc_k_plain(ab + kk * 4096, 2048, 128), id, 1u);
          mma_commit(bar_mma + 8 * b);
        }
        if (!mbar_wait(bar_mma + 8 * b, (ph_mma >> b) & 1)) abort = true;
        ph_mma ^= 1u << b;
        tc_fence_after();
        abort = __syncthreads_or(abort);
        if (abort) break;
        {
          const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + TC_D2_COL + (uint32_t)b * MT_BN;
          unsigned char* wrow = sWp + (size_t)slot * MT_WBUF + (size_t)tid * MT_WSTRIDE;
          for (int cc = 0; cc < ncols; cc += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)cc, v);
            if (tid < nrows) {
              uint4* pr = reinterpret_cast<uint4*>(wrow + cc * 2);
              uint4 u0 = pr[0], u1 = pr[1];
              __nv_bfloat162* h0 = reinterpret_cast<__nv_bfloat162*>(&u0);
              __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&u1);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f0 = __bfloat1622float2(h0[i]);
                const float2 f1 = __bfloat1622float2(h1[i]);
                h0[i] = __floats2bfloat162_rn(f0.x + v[2 * i], f0.y + v[2 * i + 1]);
                h1[i] = __floats2bfloat162_rn(f1.x + v[8 + 2 * i], f1.y + v[8 + 2 * i + 1]);
              }
              pr[0] = u0;
              pr[1] = u1;
            }
          }
          __syncwarp();
          const int ch = lane & 15;
          if (ch * 8 < ncols) {
#pragma unroll 4
            for (int k2 = 0; k2 < 16; ++k2) {
              const int row = warp * 32 + 2 * k2 + (lane >> 4);
              if (row < nrows) {
                const uint4 val = *reinterpret_cast<const uint4*>(sWp + (size_t)slot * MT_WBUF +
                                                                 (size_t)row * MT_WSTRIDE + ch * 16);
                __stcs(reinterpret_cast<uint4*>(Wp + (size_t)(row0 + row) * pj.d_in + c0 + ch * 8), val);
              }
            }
          }
        }
        tc_fence_before();
        __syncthreads();
      }
      cp_async_wait_all();
      __syncthreads();
    }
  }
  if (abort && tid == 0) report(ws, APR_ERR_TIMEOUT, K_MERGE, (int)blockIdx.x);
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                 : "memory");
  }
}


// ---------------------------------------------------------------- TMA variant
//
// The same merge with W and W' described by TMA tensor maps (a plan built once
// per set of weights): each 128 x 128 W tile arrives as two 64-column boxes
// with the 128-byte swizzle on a transaction-count mbarrier, three tiles in
// flight; the epilogue adds D in place in shared memory and one thread writes
// the W' tile back with two TMA stores, clipped at the weight's edges.  The
// A^T tiles (small, L2-resident) still come by cp.async.

constexpr int MM_NY = 3;
constexpr int MM_WBUF = TC_BM * MT_BN * 2;      // 32 KB: two 64-column swizzled boxes

struct MmSmem {
  static constexpr size_t GH = 0;
  static constexpr size_t GL = GH + (size_t)TC_BM * TC_MAXN1 * 2;
  static constexpr size_t WR = GL + (size_t)TC_BM * TC_MAXN1 * 2;        // 1024-aligned W ring
  static constexpr size_t AR = WR + (size_t)MM_NY * MM_WBUF;
  static constexpr size_t BAR = AR + (size_t)MM_NY * MT_ABUF;
  static constexpr size_t META = BAR + (2 + MM_NY) * 8;
  static constexpr size_t PREF = META + 128;
  static constexpr size_t fixed_bytes() { return PREF + 1024; }
};
static_assert(MmSmem::WR % 1024 == 0 && MM_WBUF % 1024 == 0, "swizzled boxes need 1024-byte alignment");


__global__ void __launch_bounds__(TC_THREADS, 1) merge_tma_kernel(const apr_merge_proj* __restrict__ projs,
                                                                  const CUtensorMap* __restrict__ plan,
                                                                  int nproj, int E, int r, int R16,
                                                                 const int32_t* __restrict__ idx,
                                                                 const float* __restrict__ gate, int k,
                                                                 void* ws) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int K = k * R16;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + MmSmem::BAR);
  const uint32_t bar_mma = smem_u32(bars);                     // [2]
  const uint32_t bar_w = smem_u32(bars + 2);                   // [MM_NY] W tile landed (TMA transaction count)
  volatile int* s_flags = reinterpret_cast<volatile int*>(smem + MmSmem::META);   // [0] tmem, [1] bad
  int* s_e = const_cast<int*>(s_flags) + 4;                    // [<= 8]
  float* s_g = reinterpret_cast<float*>(s_e + 8);              // [<= 8]
  int* s_pref = reinterpret_cast<int*>(smem + MmSmem::PREF);
  const uint32_t sGH = smem_u32(smem + MmSmem::GH);
  const uint32_t sGL = smem_u32(smem + MmSmem::GL);
  unsigned char* sWp = smem + MmSmem::WR;
  const uint32_t sW = smem_u32(sWp);
  const uint32_t sA = smem_u32(smem + MmSmem::AR);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(bar_mma + 8 * i, 1);
    for (int i = 0; i < MM_NY; ++i) mbar_init(bar_w + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_flags[1] = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<int*>(s_flags))),
                 "r"(TC_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)s_flags[0];
  pdl_wait();
  pdl_trigger();

  if (tid < k) {
    const int e = idx[tid];
    if (e < 0 || e >= E) s_flags[1] = 1;
    s_e[tid] = e;
    s_g[tid] = gate[tid];
  }
  // strips (128 rows) per weight, prefix over the weights
  if (tid == 0) {
    int acc = 0;
    s_pref[0] = 0;
    for (int p = 0; p < nproj; ++p) {
      acc += (projs[p].d_out + TC_BM - 1) / TC_BM;
      s_pref[p + 1] = acc;
    }
  }
  __syncthreads();
  bool abort = false;
  if (s_flags[1]) {
    if (tid == 0 && blockIdx.x == 0) report(ws, APR_ERR_DEVICE_INDEX, K_MERGE, 0);
  } else {
    const int total = s_pref[nproj];
    const uint32_t sbo_g = (uint32_t)(K / 8) * 128;         // Bg: next 8-row group
    const uint32_t id = idesc_bf16_bmn(TC_BM, MT_BN);
    uint32_t ph_mma = 0;
    uint32_t gt = 0;                                          // W tiles so far (ring slot and phase)
    for (int strip = blockIdx.x; strip < total && !abort; strip += gridDim.x) {
      int lo = 0, hi = nproj;                                 // weight of this strip
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pref[mid] <= strip) lo = mid; else hi = mid;
      }
      const apr_merge_proj pj = projs[lo];
      const int row0 = (strip - s_pref[lo]) * TC_BM;
      const int nrows = min(TC_BM, pj.d_out - row0);
      // gated B rows of the strip, bf16 hi + lo, K-major
      {
        const int n = row0 + tid;
        for (int j = 0; j < k; ++j) {
          const __nv_bfloat16* B = reinterpret_cast<const __nv_bfloat16*>(pj.B[s_e[j]]);
          for (int c8 = 0; c8 < R16; c8 += 8) {
            float f[8];
            if (tid < nrows && c8 < r) {
              load8(B + (size_t)n * r + c8, f);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] = 0.f;
            }
            uint32_t h4[4], l4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float a0 = f[2 * i] * s_g[j], a1 = f[2 * i + 1] * s_g[j];
              const __nv_bfloat162 hh = __floats2bfloat162_rn(a0, a1);
              const float2 hf = __bfloat1622float2(hh);
              h4[i] = *reinterpret_cast<const uint32_t*>(&hh);
              l4[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
            }
            const int kc8 = (j * R16 + c8) >> 3;
            const uint32_t off = (uint32_t)(tid >> 3) * sbo_g + (uint32_t)kc8 * 128 + (uint32_t)(tid & 7) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sGH + off), "r"(h4[0]), "r"(h4[1]),
                         "r"(h4[2]), "r"(h4[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sGL + off), "r"(l4[0]), "r"(l4[1]),
                         "r"(l4[2]), "r"(l4[3])
                         : "memory");
          }
        }
      }
      fence_proxy_async();                       // Bg was written by ordinary stores
      const int nct = (pj.d_in + MT_BN - 1) / MT_BN;
      const uint32_t gt0 = gt;
      auto issue_tile = [&](int ct) {
        const int slot = (gt0 + ct) % MM_NY;
        const int c0 = ct * MT_BN;
        const int ncols = min(MT_BN, pj.d_in - c0);
        // A^T tile, MN-major: core matrix (8 columns x 8 rank rows) at (col/8)*128 + (kk/8)*2048
        const uint32_t abase = sA + (uint32_t)slot * MT_ABUF;
        for (int w = tid; w < K * (MT_BN / 8); w += TC_THREADS) {
          const int kk = w / (MT_BN / 8), c = w % (MT_BN / 8);
          const int j = kk / R16, i = kk % R16;
          const uint32_t dst = abase + (uint32_t)c * 128 + (uint32_t)(kk >> 3) * 2048 + (uint32_t)(kk & 7) * 16;
          const bool valid = i < r && c * 8 < ncols;
          const __nv_bfloat16* A = reinterpret_cast<const __nv_bfloat16*>(pj.A[s_e[j]]);
          cp_async16_zfill(dst, valid ? A + (size_t)i * pj.d_in + c0 + c * 8 : A, valid);
        }
        // W tile: two 64-column x 128-row TMA boxes (128B-swizzled) on the slot's barrier
        if (tid == 0) {
          bulk_wait_read_all();                  // the slot's previous W' store has read it out
          const uint32_t wslot = sW + (uint32_t)((gt0 + ct) % MM_NY) * MM_WBUF;
          const uint32_t wb = bar_w + 8 * ((gt0 + ct) % MM_NY);
          mbar_arrive_expect_tx(wb, MM_WBUF);
          tma_load_2d(wslot, &plan[2 * lo], c0, row0, wb);
          tma_load_2d(wslot + MM_WBUF / 2, &plan[2 * lo], c0 + 64, row0, wb);
        }
      };
      for (int ct = 0; ct < MM_NY - 1; ++ct) {
        if (ct < nct) issue_tile(ct);
        cp_async_commit();
      }
      for (int ct = 0; ct < nct; ++ct) {
        const int b = ct & 1;
        const int slot = (gt0 + ct) % MM_NY;
        const int c0 = ct * MT_BN;
        const int ncols = min(MT_BN, pj.d_in - c0);
        if (ct + MM_NY - 1 < nct) issue_tile(ct + MM_NY - 1);
        cp_async_commit();
        cp_async_wait<MM_NY - 1>();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const uint32_t ab = sA + (uint32_t)slot * MT_ABUF;       // A ring follows the W ring
          const uint32_t dcol = tmem + TC_D2_COL + (uint32_t)b * MT_BN;
          for (int kk = 0; kk < K / 16; ++kk)
            mma_bf16(dcol, desc_k_plain(sGH + kk * 256, 128, sbo_g), desc_k_plain(ab + kk * 4096, 2048, 128), id,
                     kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < K / 16; ++kk)
            mma_bf16(dcol, desc_k_plain(sGL + kk * 256, 128, sbo_g), desc_k_plain(ab + kk * 4096, 2048, 128), id, 1u);
          mma_commit(bar_mma + 8 * b);
        }
        if (!mbar_wait(bar_mma + 8 * b, (ph_mma >> b) & 1)) abort = true;
        ph_mma ^= 1u << b;
        if (!mbar_wait(bar_w + 8 * slot, ((gt0 + ct) / MM_NY) & 1)) abort = true;
        tc_fence_after();
        abort = __syncthreads_or(abort);
        if (abort) break;
        {
          const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + TC_D2_COL + (uint32_t)b * MT_BN;
          unsigned char* wslot = sWp + (size_t)slot * MM_WBUF;
          const int sw = tid & 7;
          for (int cc = 0; cc < ncols; cc += 16) {
            float v[16];
            tmem_ld16(lane_addr + (uint32_t)cc, v);
            if (tid < nrows) {
              unsigned char* rb = wslot + (size_t)(cc >> 6) * (MM_WBUF / 2) + (size_t)tid * 128;
              const int q0 = (cc & 63) >> 3;
              uint4* p0 = reinterpret_cast<uint4*>(rb + ((q0 ^ sw) << 4));
              uint4* p1 = reinterpret_cast<uint4*>(rb + (((q0 + 1) ^ sw) << 4));
              uint4 u0 = *p0, u1 = *p1;
              __nv_bfloat162* h0 = reinterpret_cast<__nv_bfloat162*>(&u0);
              __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&u1);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f0 = __bfloat1622float2(h0[i]);
                const float2 f1 = __bfloat1622float2(h1[i]);
                h0[i] = __floats2bfloat162_rn(f0.x + v[2 * i], f0.y + v[2 * i + 1]);
                h1[i] = __floats2bfloat162_rn(f1.x + v[8 + 2 * i], f1.y + v[8 + 2 * i + 1]);
              }
              *p0 = u0;
              *p1 = u1;
            }
          }
          fence_proxy_async();                   // the TMA store reads what these threads wrote
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {                          // W' tile out: two boxes, clipped at the weight's edges
          const uint32_t wslot = sW + (uint32_t)slot * MM_WBUF;
          tma_store_2d(&plan[2 * lo + 1], wslot, c0, row0);
          if (c0 + 64 < pj.d_in) tma_store_2d(&plan[2 * lo + 1], wslot + MM_WBUF / 2, c0 + 64, row0);
          bulk_commit();
        }
        tc_fence_before();
        __syncthreads();
      }
      cp_async_wait_all();
      gt = gt0 + nct;
      __syncthreads();
    }
  }
  if (abort && tid == 0) report(ws, APR_ERR_TIMEOUT, K_MERGE, (int)blockIdx.x);
  cp_async_wait_all();
  if (tid == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled, fetched through the runtime (no link against libcuda).
static PFN_cuTensorMapEncodeTiled tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  });
  return fn;
}

// Row-scatter map of a [rows, cols] bf16 matrix: boxes of 64 columns x 1 row,
// 128-byte swizzle (the tile::scatter4 / gather4 form: four rows per copy).
cudaError_t encode_row_map(CUtensorMap* m, void* base, int rows, int cols) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
                 CUDA_SUCCESS
             ? cudaSuccess
             : cudaErrorInvalidValue;
}

cudaError_t encode_tile_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? cudaSuccess
             : cudaErrorInvalidValue;
}

size_t merge_plan_bytes(int nproj) { return (size_t)nproj * 2 * sizeof(CUtensorMap); }

// One tensor map per W and per W': [d_out rows, d_in columns] bf16, boxes of
// 64 columns x 128 rows, 128-byte swizzle, zeros outside on loads.
cudaError_t merge_plan_build(const apr_merge_proj* projs, int nproj, void* plan) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  std::vector<CUtensorMap> maps((size_t)2 * nproj);
  for (int p = 0; p < nproj; ++p) {
    const cuuint64_t dims[2] = {(cuuint64_t)projs[p].d_in, (cuuint64_t)projs[p].d_out};
    const cuuint64_t strides[1] = {(cuuint64_t)projs[p].d_in * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)TC_BM};
    const cuuint32_t estr[2] = {1, 1};
    for (int w = 0; w < 2; ++w) {
      void* base = const_cast<void*>(w == 0 ? projs[p].W : projs[p].Wp);
      if (enc(&maps[2 * p + w], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  return cudaMemcpy(plan, maps.data(), merge_plan_bytes(nproj), cudaMemcpyHostToDevice);
}

cudaError_t launch_merge_tma(const apr_merge_proj* projs, const void* plan, int nproj, int E, int r,
                             const int32_t* idx, const float* gate, int k, void* ws, cudaStream_t s) {
  const size_t smem = MmSmem::fixed_bytes() + sizeof(int) * ((size_t)nproj + 1);
  static SmemLimit limit;
  cudaError_t err = limit.ensure((const void*)merge_tma_kernel, smem);
  if (err != cudaSuccess) return err;
  const int nsm = device_sm_count();
  return launch_pdl(merge_tma_kernel, dim3(nsm), dim3(TC_THREADS), smem, s, projs,
                    reinterpret_cast<const CUtensorMap*>(plan), nproj, E, r, round16(r), idx, gate, k, ws);
}

bool merge_tensor_supported(int k, int r, int nproj) {
  return k * round16(r) <= TC_MAXN1 && nproj <= MT_MAXPROJ;
}

cudaError_t launch_merge_tensor(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                const float* gate, int k, void* ws, cudaStream_t s) {
  const size_t smem = MtSmem::fixed_bytes() + sizeof(int) * ((size_t)nproj + 1);
  static SmemLimit limit;
  cudaError_t err = limit.ensure((const void*)merge_tc_kernel, smem);
  if (err != cudaSuccess) return err;
  const int nsm = device_sm_count();
  return launch_pdl(merge_tc_kernel, dim3(nsm), dim3(TC_THREADS), smem, s, projs, nproj, E, r, round16(r), idx,
                    gate, k, ws);
}

}  // namespace apr
