// SGMM on the 5th-generation tensor cores (tcgen05) for long segments
// (prefill).  AdaFuse summary (gist.science), Resumen tecnico §2.B: the
// segmented gather product applies the selected low-rank adapters to the
// tokens gathered per adapter in one batched product, fused into the add onto
// the base projection output, with prefetching and tiling.
//
// The routing plan orders tokens by their adapter set; a work item is one
// set tile (<= 128 tokens that share the same k <= 2 adapters {e0, e1}) and
// one projection.  Per item, in one CTA of 128 threads (1 CTA per SM, TMEM
// fully owned, persistent over the items):
//
//  shrink  D1[128 x N1] = X_tile[128 x d_in] . [A_e0 ; A_e1]^T on tcgen05
//          (kind::f16, bf16 in, fp32 accumulate in TMEM), N1 = k * R16 where
//          R16 is the rank rounded up to 16 (zero rows pad the smaller ranks).
//          The gathered x rows arrive by TMA (tile::gather4: four token rows x
//          128 bytes per instruction, 128B-swizzled, one issuing lane per warp
//          for its 32 tokens, rows of absent tokens zero-filled) and the small
//          A rows by 16-byte cp.async; both complete on the stage's "full"
//          mbarrier (6 stages in flight).  One thread of the MMA warp issues
//          the MMAs of a stage once it is full and commits them to the stage's
//          "empty" mbarrier, which frees the stage for the next fill.
//  gate    D1 is read back with tcgen05.ld (one TMEM lane per token), scaled
//          by the token's gates and split into bf16 hi + lo parts (so the
//          expand keeps ~16 mantissa bits of v), written to shared memory as
//          the K-major A operand of the expand.
//  expand  for every 128-column tile of d_out: D2[128 x 128] = V_hi.Bcat^T +
//          V_lo.Bcat^T with Bcat[n] = [B_e0[n] | B_e1[n]] (K2 = N1), TMEM
//          double buffered.  Bcat (cp.async) and the y_base rows (TMA gather4)
//          of a tile are fetched two tiles ahead into 3-deep rings that reuse
//          the shrink stages' shared memory; the epilogue adds D2 in its
//          token's row, rounds to bf16 once, and the rows leave by TMA
//          scatter4 (plain stores for the one 4-row group a tile's end cuts).
//
// Warps 0-3 stage operands and run epilogues, warp 4 issues the MMAs; each
// worker warp owns 32 token rows of every buffer, so reuse of a ring slot only
// waits for that warp's own bulk stores.
//
// Every mbarrier wait is bounded by the global timer (1 s); on expiry the CTA
// records APR_ERR_TIMEOUT, drains its own copies and frees its TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int TC_THREADS = 128;
constexpr int TC_BM = 128;       // tokens per tile (= kSetTile)
constexpr int TC_BK = 64;        // input columns per stage (one 128-byte swizzle row)
constexpr int TC_STAGES = 6;
constexpr int TC_MAXN1 = 64;     // k * R16
constexpr int TC_NT = 128;       // output columns per expand tile
constexpr int TC_NY = 3;         // depth of the Bcat / y_base rings (prefetch distance 2)
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr uint32_t TC_D2_COL = 128;           // D2 buffers at columns 128 and 256
constexpr int TC_STAGE_BYTES = TC_BM * 128 + TC_MAXN1 * 128;   // x tile + A rows
constexpr int TC_YBUF_BYTES = 2 * TC_BM * 128;                  // two 64-column halves, 128B-swizzled rows
constexpr int TC_BBUF_BYTES = TC_NT * TC_MAXN1 * 2;

struct TcSmem {
  // the shrink stages and the expand's rings are never live at the same time
  static constexpr size_t STAGE_AREA = (size_t)TC_STAGES * TC_STAGE_BYTES;
  static constexpr size_t RING_AREA = (size_t)TC_NY * (TC_YBUF_BYTES + TC_BBUF_BYTES);
  static constexpr size_t U = 0;
  static constexpr size_t U_BYTES = STAGE_AREA > RING_AREA ? STAGE_AREA : RING_AREA;
  static constexpr size_t YR = U;                                             // y ring (1024-aligned slots)
  static constexpr size_t BR = U + (size_t)TC_NY * TC_YBUF_BYTES;             // Bcat ring
  static constexpr size_t VH = U + (U_BYTES + 1023) / 1024 * 1024;            // 16 KB
  static constexpr size_t VL = VH + (size_t)TC_BM * TC_MAXN1 * 2;             // 16 KB
  static constexpr size_t BAR = VL + (size_t)TC_BM * TC_MAXN1 * 2;            // mbarriers
  static constexpr int NBARS = 2 * TC_STAGES + 2 + TC_NY + 4;
  static constexpr size_t META = BAR + (size_t)NBARS * 8;
  static constexpr size_t TOTAL = META + 3 * TC_BM * 4 + 64;
  static constexpr size_t ALLOC = TOTAL + 1024;                               // for 1024-byte alignment
};
static_assert(TcSmem::ALLOC <= 227 * 1024, "shared memory budget");
static_assert(TC_STAGE_BYTES % 1024 == 0, "stages keep 1024-byte alignment");
static_assert(TcSmem::BR % 16 == 0 && TC_YBUF_BYTES % 1024 == 0, "aligned rings");

// ---------------------------------------------------------------- the kernel

struct TcArgs {
  CUtensorMap tm_x;                    // x [T, d_in], box 64 x 1, 128B swizzle
  CUtensorMap tm_yb[APR_MAX_PROJ];     // y_base [T, d_out]
  CUtensorMap tm_y[APR_MAX_PROJ];      // y [T, d_out]
  SgmmArgs a;
  int R16;     // rank slot per adapter (multiple of 16)
  int N1;      // k * R16
};

constexpr int TC_WORKERS = 128;                  // warps 0-3: loads and epilogues
constexpr int TC_BLOCK = TC_WORKERS + 32;        // warp 4: MMA issue

__device__ __forceinline__ void workers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(TC_WORKERS) : "memory"); }

// Warp-specialised: warps 0-3 stage operands with TMA and cp.async (completion
// arrives on mbarriers) and run the epilogues; lane 0 of warp 4 issues every
// tcgen05.mma and commits it to the barrier that releases the consumer.  No
// block-wide barrier inside an item, so loads, MMAs and epilogues of different
// chunks and tiles overlap.
__global__ void __launch_bounds__(TC_BLOCK, 1) sgmm_tc_kernel(const __grid_constant__ TcArgs args) {
  const SgmmArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool worker = tid < TC_WORKERS;
  const int K = a.k, R16 = args.R16, N1 = args.N1, K2 = N1;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TcSmem::BAR);
  const uint32_t bar_full = smem_u32(bars);                              // [S]  stage loaded
  const uint32_t bar_empty = smem_u32(bars + TC_STAGES);                 // [S]  stage consumed
  const uint32_t bar_d1 = smem_u32(bars + 2 * TC_STAGES);                // shrink accumulator ready
  const uint32_t bar_v = smem_u32(bars + 2 * TC_STAGES + 1);             // V written
  const uint32_t bar_tfull = smem_u32(bars + 2 * TC_STAGES + 2);         // [NY] tile operands loaded
  const uint32_t bar_d2full = smem_u32(bars + 2 * TC_STAGES + 2 + TC_NY);      // [2] expand accumulator ready
  const uint32_t bar_d2empty = smem_u32(bars + 2 * TC_STAGES + 4 + TC_NY);     // [2] expand accumulator read
  int* s_tok = reinterpret_cast<int*>(smem + TcSmem::META);
  float* s_g0 = reinterpret_cast<float*>(s_tok + TC_BM);
  float* s_g1 = s_g0 + TC_BM;
  volatile int* s_flags = reinterpret_cast<volatile int*>(s_g1 + TC_BM);   // [0] tmem, [2..3] set, [4] bad
  const uint32_t sU = smem_u32(smem + TcSmem::U);
  const uint32_t sVH = smem_u32(smem + TcSmem::VH);
  const uint32_t sVL = smem_u32(smem + TcSmem::VL);
  unsigned char* sYp = smem + TcSmem::YR;     // rings overlay the stages
  const uint32_t sY = smem_u32(sYp);
  const uint32_t sB = smem_u32(smem + TcSmem::BR);

  if (tid == 0) {
    for (int i = 0; i < TC_STAGES; ++i) {
      mbar_init(bar_full + 8 * i, TC_WORKERS + 4);       // A copies of every worker + x rows of every warp
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_d1, 1);
    mbar_init(bar_v, TC_WORKERS);
    for (int i = 0; i < TC_NY; ++i) mbar_init(bar_tfull + 8 * i, TC_WORKERS + 4);   // Bcat + y_base rows
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_d2full + 8 * i, 1);
      mbar_init(bar_d2empty + 8 * i, TC_WORKERS);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

  const WsLayout L = ws_layout(a.T, a.k, a.E);
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const int* tok_order = ws_at<int>(a.ws, L.tok_order);
  const SetTile* stiles = ws_at<SetTile>(a.ws, L.stiles);
  const int nst = hdr->n_stiles;
  const long nitems = (long)nst * a.nproj;
  const int d_in = a.d_in;
  const int nk = d_in / TC_BK;
  const uint32_t id1 = idesc_bf16(TC_BM, N1);
  const uint32_t id2 = idesc_bf16(TC_BM, TC_NT);
  const uint32_t sbo_v = (uint32_t)(K2 / 8) * 128;   // V and Bcat: next 8-row group
  uint32_t gchunk = 0;      // shrink chunks so far (stage = gchunk % S, use = gchunk / S)
  uint32_t gtile = 0;       // expand tiles so far (ring slot = gtile % NY, D2 buffer = gtile & 1)
  uint32_t nitem = 0;       // items so far (parity of d1 / V barriers)
  bool abort = false;

  for (long item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int st = (int)(item / a.nproj);
    const int p = (int)(item % a.nproj);
    const int d_out = a.proj[p].d_out;
    const int nnt = (d_out + TC_NT - 1) / TC_NT;
    if (worker) {
      // tokens, their adapter set (sorted) and gates in that order
      const SetTile tile = stiles[st];
      int tok = -1, e0 = 0, e1 = 0;
      float g0 = 0.f, g1 = 0.f;
      if (tid < tile.len) {
        tok = tok_order[tile.start + tid];
        e0 = a.idx[(size_t)tok * K];
        g0 = a.gate[(size_t)tok * K];
        if (K == 2) {
          e1 = a.idx[(size_t)tok * K + 1];
          g1 = a.gate[(size_t)tok * K + 1];
          if (e1 < e0) {
            const int te = e0; e0 = e1; e1 = te;
            const float tg = g0; g0 = g1; g1 = tg;
          }
        }
      }
      s_tok[tid] = tok;
      s_g0[tid] = g0;
      s_g1[tid] = g1;
      if (tid == 0) {
        s_flags[2] = e0;
        s_flags[3] = e1;
        bool bad = (e0 < 0 || e0 >= a.E || (K == 2 && (e1 < 0 || e1 >= a.E)));
        if (!bad) {
          const int r0 = a.ranks[e0], r1 = K == 2 ? a.ranks[e1] : 8;
          bad = r0 <= 0 || r0 > R16 || (r0 & 7) || r1 <= 0 || r1 > R16 || (r1 & 7);
        }
        s_flags[4] = bad ? 1 : 0;
        if (bad) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e0);
      }
    }
    __syncthreads();
    if (s_flags[4] || abort) {
      __syncthreads();
      continue;
    }
    const int e0 = s_flags[2], e1 = s_flags[3];
    const int rk[2] = {a.ranks[e0], K == 2 ? a.ranks[e1] : 0};
    const uint32_t g0 = gchunk, t0 = gtile;
    // this warp's 32 token rows as TMA row coordinates (T = past the end: zero fill)
    int trow[32];
    if (worker && lane == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int tk = s_tok[warp * 32 + i];
        trow[i] = tk >= 0 ? tk : a.T;
      }
    }

    if (worker) {
      // -------------------------------------------------------- shrink operands
      const __nv_bfloat16* Aj[2];
      Aj[0] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].A[e0]);
      Aj[1] = K == 2 ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].A[e1]) : Aj[0];
      for (int c = 0; c < nk && !abort; ++c) {
        const uint32_t g = g0 + c;
        const uint32_t s = g % TC_STAGES;
        if (g >= TC_STAGES && !mbar_wait(bar_empty + 8 * s, ((g / TC_STAGES) - 1) & 1)) { abort = true; break; }
        // x rows of this warp's 32 tokens: 8 TMA gathers of 4 rows x 128 bytes
        if (lane == 0) {
          const uint32_t fb = bar_full + 8 * s;
          mbar_arrive_expect_tx(fb, 8 * 4 * 128);
          const uint32_t xdst = sU + s * TC_STAGE_BYTES + (uint32_t)(warp * 32) * 128;
#pragma unroll
          for (int g4 = 0; g4 < 8; ++g4)
            tma_gather4(xdst + g4 * 512, &args.tm_x, c * TC_BK, trow[4 * g4], trow[4 * g4 + 1], trow[4 * g4 + 2],
                        trow[4 * g4 + 3], fb);
        }
        const uint32_t abase = sU + s * TC_STAGE_BYTES + TC_BM * 128;
        for (int w = tid; w < N1 * 8; w += TC_WORKERS) {
          const int j = w >> 3, q = w & 7;
          const int slot = j / R16, r = j % R16;
          const uint32_t dst = abase + (uint32_t)j * 128 + ((q ^ (j & 7)) << 4);
          const bool valid = r < rk[slot];
          cp_async16_zfill(dst, valid ? Aj[slot] + (size_t)r * d_in + (size_t)c * TC_BK + q * 8 : Aj[0], valid);
        }
        cp_async_arrive(bar_full + 8 * s);
      }
      // -------------------------------------------------------- gates -> V (bf16 hi + lo)
      if (!abort && !mbar_wait(bar_d1, nitem & 1)) abort = true;
      tc_fence_after();
      if (!abort) {
        const int row = tid;                       // TMEM lane = token row
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const float ga = s_g0[row], gb = s_g1[row];
        for (int c0 = 0; c0 < N1; c0 += 16) {
          float v[16];
          tmem_ld16(lane_addr + (uint32_t)c0, v);
          const float gg = (c0 / R16) == 0 ? ga : gb;
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a0 = v[2 * i] * gg, a1 = v[2 * i + 1] * gg;
            const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            const float2 hf = __bfloat1622float2(h);
            hi[i] = *reinterpret_cast<const uint32_t*>(&h);
            lo[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
          }
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            const int kc8 = (c0 >> 3) + h8;
            const uint32_t off = (uint32_t)(row >> 3) * sbo_v + (uint32_t)kc8 * 128 + (uint32_t)(row & 7) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sVH + off), "r"(hi[4 * h8]),
                         "r"(hi[4 * h8 + 1]), "r"(hi[4 * h8 + 2]), "r"(hi[4 * h8 + 3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sVL + off), "r"(lo[4 * h8]),
                         "r"(lo[4 * h8 + 1]), "r"(lo[4 * h8 + 2]), "r"(lo[4 * h8 + 3])
                         : "memory");
          }
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar_v);
      }
      // -------------------------------------------------------- expand operands and epilogues
      const __nv_bfloat16* Bj[2];
      Bj[0] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e0]);
      Bj[1] = K == 2 ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e1]) : Bj[0];
      __nv_bfloat16* __restrict__ y = reinterpret_cast<__nv_bfloat16*>(a.proj[p].y);
      auto issue_tile = [&](int nt) {
        const uint32_t slot = (t0 + nt) % TC_NY;
        const int n0 = nt * TC_NT;
        const int ncols = min(TC_NT, d_out - n0);
        const uint32_t bbase = sB + slot * TC_BBUF_BYTES;
        const int cpr = K2 / 8;
        for (int w = tid; w < TC_NT * cpr; w += TC_WORKERS) {
          const int n = w / cpr, q = w % cpr;
          const int kslot = q / (R16 / 8), cq = q % (R16 / 8);
          const uint32_t dst = bbase + (uint32_t)(n >> 3) * sbo_v + (uint32_t)q * 128 + (uint32_t)(n & 7) * 16;
          const bool valid = n < ncols && cq * 8 < rk[kslot];
          cp_async16_zfill(dst, valid ? Bj[kslot] + (size_t)(n0 + n) * rk[kslot] + cq * 8 : Bj[0], valid);
        }
        cp_async_arrive(bar_tfull + 8 * slot);
        // y_base rows of this warp's tokens: TMA gathers into the two swizzled 64-column halves
        if (lane == 0) {
          bulk_wait_read_all();                    // this warp's stores from the slot are read out
          const uint32_t tb = bar_tfull + 8 * slot;
          const int nh = (ncols + 63) / 64;
          mbar_arrive_expect_tx(tb, nh * 8 * 4 * 128);
          for (int h = 0; h < nh; ++h) {
            const uint32_t ydst = sY + slot * TC_YBUF_BYTES + h * (TC_BM * 128) + (uint32_t)(warp * 32) * 128;
#pragma unroll
            for (int g4 = 0; g4 < 8; ++g4)
              tma_gather4(ydst + g4 * 512, &args.tm_yb[p], n0 + 64 * h, trow[4 * g4], trow[4 * g4 + 1],
                          trow[4 * g4 + 2], trow[4 * g4 + 3], tb);
          }
        }
      };
      for (int nt = 0; nt < TC_NY - 1 && nt < nnt && !abort; ++nt) issue_tile(nt);
      for (int nt = 0; nt < nnt && !abort; ++nt) {
        const uint32_t g = t0 + nt;
        const uint32_t slot = g % TC_NY, b = g & 1;
        const int n0 = nt * TC_NT;
        const int ncols = min(TC_NT, d_out - n0);
        if (nt + TC_NY - 1 < nnt) issue_tile(nt + TC_NY - 1);   // slot of tile nt-1: consumed
        if (!mbar_wait(bar_tfull + 8 * slot, (g / TC_NY) & 1)) { abort = true; break; }
        if (!mbar_wait(bar_d2full + 8 * b, (g >> 1) & 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + TC_D2_COL + b * TC_NT;
        unsigned char* yslot = sYp + (size_t)slot * TC_YBUF_BYTES;
        const int sw = tid & 7;
        const bool mine = s_tok[tid] >= 0;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[16];
          tmem_ld16(lane_addr + (uint32_t)c0, v);
          if (mine) {
            const int h = c0 >> 6, q = (c0 & 63) >> 3;
            unsigned char* rbase = yslot + (size_t)h * (TC_BM * 128) + (size_t)tid * 128;
            uint4* p0 = reinterpret_cast<uint4*>(rbase + ((q ^ sw) << 4));
            uint4* p1 = reinterpret_cast<uint4*>(rbase + (((q + 1) ^ sw) << 4));
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
        tc_fence_before();
        mbar_arrive(bar_d2empty + 8 * b);          // D2[b] may be overwritten
        // rows of a 4-row group with a missing token are written by their owners ...
        const int g4 = (tid & 31) >> 2;
        const bool full_group = s_tok[warp * 32 + 4 * g4] >= 0 && s_tok[warp * 32 + 4 * g4 + 1] >= 0 &&
                                s_tok[warp * 32 + 4 * g4 + 2] >= 0 && s_tok[warp * 32 + 4 * g4 + 3] >= 0;
        if (mine && !full_group) {
          for (int qq = 0; qq < ncols / 8; ++qq) {
            const int h = qq >> 3, q = qq & 7;
            const uint4 val = *reinterpret_cast<const uint4*>(yslot + (size_t)h * (TC_BM * 128) + (size_t)tid * 128 +
                                                              ((q ^ sw) << 4));
            *reinterpret_cast<uint4*>(y + (size_t)s_tok[tid] * d_out + n0 + qq * 8) = val;
          }
        }
        // ... and full groups leave by TMA scatter, 4 rows x 64 columns per instruction
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          const int nh = (ncols + 63) / 64;
          for (int gg = 0; gg < 8; ++gg) {
            const int r = warp * 32 + 4 * gg;
            if (s_tok[r] < 0 || s_tok[r + 1] < 0 || s_tok[r + 2] < 0 || s_tok[r + 3] < 0) continue;
            for (int h = 0; h < nh; ++h)
              tma_scatter4(&args.tm_y[p], n0 + 64 * h, s_tok[r], s_tok[r + 1], s_tok[r + 2], s_tok[r + 3],
                           smem_u32(yslot + (size_t)h * (TC_BM * 128) + (size_t)r * 128));
          }
          bulk_commit();
        }
        __syncwarp();
      }
      // the next item's stages overlay the y ring: this warp's stores must have read it out
      if (lane == 0) bulk_wait_read_all();
      cp_async_wait_all();
    } else if (lane == 0) {
      // -------------------------------------------------------- MMA issue (one thread)
      for (int c = 0; c < nk && !abort; ++c) {
        const uint32_t g = g0 + c;
        const uint32_t s = g % TC_STAGES;
        if (!mbar_wait(bar_full + 8 * s, (g / TC_STAGES) & 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t xs = sU + s * TC_STAGE_BYTES;
        const uint32_t as = xs + TC_BM * 128;
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk)
          mma_bf16(tmem, desc_k_sw128(xs + kk * 32), desc_k_sw128(as + kk * 32), id1, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_empty + 8 * s);
      }
      if (!abort) mma_commit(bar_d1);
      if (!abort && !mbar_wait(bar_v, nitem & 1)) abort = true;
      tc_fence_after();
      for (int nt = 0; nt < nnt && !abort; ++nt) {
        const uint32_t g = t0 + nt;
        const uint32_t slot = g % TC_NY, b = g & 1;
        if (!mbar_wait(bar_tfull + 8 * slot, (g / TC_NY) & 1)) { abort = true; break; }
        if (g >= 2 && !mbar_wait(bar_d2empty + 8 * b, ((g >> 1) - 1) & 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t bb = sB + slot * TC_BBUF_BYTES;
        const uint32_t dcol = tmem + TC_D2_COL + b * TC_NT;
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(sVH + kk * 256, 128, sbo_v), desc_k_plain(bb + kk * 256, 128, sbo_v), id2,
                   kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(sVL + kk * 256, 128, sbo_v), desc_k_plain(bb + kk * 256, 128, sbo_v), id2, 1u);
        mma_commit(bar_d2full + 8 * b);
      }
    }
    gchunk = g0 + nk;
    gtile = t0 + nnt;
    ++nitem;
    abort = __syncthreads_or(abort);
  }
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  cp_async_wait_all();
  if (lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side

static int round16(int r) { return (r + 15) / 16 * 16; }

bool sgmm_tensor_supported(const SgmmArgs& a, int dtype) {
  if (dtype != APR_BF16) return false;
  if (a.k < 1 || a.k > 2) return false;
  if (a.k * round16(a.max_rank) > TC_MAXN1) return false;
  if (a.d_in % TC_BK != 0) return false;
  for (int p = 0; p < a.nproj; ++p)
    if (a.proj[p].d_out % 16 != 0) return false;
  return true;
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

// Row-major bf16 [rows, cols] matrix seen by TMA as boxes of one row x 64
// columns (128 bytes) with the 128-byte swizzle; reads past the last row or
// column return zeros, writes there are dropped.
static bool encode_rows(PFN_cuTensorMapEncodeTiled enc, CUtensorMap* m, const void* base, int rows, int cols) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_sgmm_tensor(const SgmmArgs& a, cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    cudaError_t err = cudaFuncSetAttribute(sgmm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)TcSmem::ALLOC);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  TcArgs t;
  memset(&t, 0, sizeof(t));
  t.a = a;
  t.R16 = round16(a.max_rank);
  t.N1 = a.k * t.R16;
  if (!encode_rows(enc, &t.tm_x, a.x, a.T, a.d_in)) return cudaErrorInvalidValue;
  for (int p = 0; p < a.nproj; ++p) {
    if (!encode_rows(enc, &t.tm_yb[p], a.proj[p].y_base, a.T, a.proj[p].d_out) ||
        !encode_rows(enc, &t.tm_y[p], a.proj[p].y, a.T, a.proj[p].d_out))
      return cudaErrorInvalidValue;
  }
  // upper bound on items: set tiles <= T (one per token at worst); the kernel loops over the real count
  long max_items = (long)((a.T + TC_BM - 1) / TC_BM + a.T) * a.nproj;
  int grid = nsm;
  if (max_items < grid) grid = (int)max_items;
  return launch_pdl(sgmm_tc_kernel, dim3(grid), dim3(TC_BLOCK), TcSmem::ALLOC, s, t);
}


// ---------------------------------------------------------------- merge on the tensor cores
//
// Batch-1 merge (AdaFuse summary §2.B decoding steps 3 and 5), every weight in
// one launch, out of place:  W' = W + sum_j g_j B_{e_j} A_{e_j}.
// A work item is a strip of 128 rows of one weight.  The strip's gated B rows
// Bg[n][j*R16 + i] = g_j B_{e_j}[n][i] are formed once (fp32 -> bf16 hi + lo,
// K-major), then for every 128-column tile: D[128 x 128] = Bg_hi.A^T +
// Bg_lo.A^T on tcgen05 with A^T as an MN-major operand (rows of A_e are
// contiguous along the output columns), TMEM double buffered; the W tile and
// the A tile arrive two tiles ahead by cp.async into 3-deep rings, and the
// epilogue adds D to W in fp32, rounds once and the warp writes its 32 rows
// of W' back with coalesced 128-bit stores.

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

bool merge_tensor_supported(int k, int r, int nproj) {
  return k * round16(r) <= TC_MAXN1 && nproj <= MT_MAXPROJ;
}

cudaError_t launch_merge_tensor(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                const float* gate, int k, void* ws, cudaStream_t s) {
  const size_t smem = MtSmem::fixed_bytes() + sizeof(int) * ((size_t)nproj + 1);
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t err = cudaFuncSetAttribute(merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    configured = smem;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  return launch_pdl(merge_tc_kernel, dim3(nsm), dim3(TC_THREADS), smem, s, projs, nproj, E, r, round16(r), idx,
                    gate, k, ws);
}

}  // namespace apr
