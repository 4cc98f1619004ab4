// SGMM expand in token order over the whole adapter bank (tcgen05), for a few
// adapters and many tokens (prefill).  AdaFuse summary (gist.science), Resumen
// tecnico §2.B: the segmented product applies the selected low-rank adapters
// to the batch and is fused into the add onto the base projection output.
//
// The gathered expand moves every y row through per-row copies, and a CTA
// issues those at a fixed rate far below its share of HBM bandwidth.  Here the
// y rows are never gathered: a unit of work is a tile of 128 CONSECUTIVE
// tokens x 128 output columns of one projection, so y_base comes in and y goes
// out as 2-D TMA boxes of contiguous rows.  The adapters of those tokens are
// whatever the router chose, so the contraction runs over the whole bank:
//
//   D[t, n] = sum_{e < E} sum_{r < R16} V[t, e*R16 + r] * B_e[n, r]
//   V[t, e*R16 + r] = g_{t,j} (A_e x_t)[r]   if idx[t, j] == e, else 0
//
// K = E * R16 <= 256.  The product is E/k times the sparse one; the tensor
// pipe still idles most of the time on this HBM-bound step.
//
//  - V rows: the shrink (tc_shrink_kernel, pair order) leaves g * A_e x per
//    (token, slot) pair in bf16.  The gated rows of a tile's 128 tokens are
//    contiguous, so one bulk copy brings them into shared memory; a warpgroup
//    of "V" warps then spreads each token's k slots over the bank's rank
//    slots (a zero line where the token did not select the adapter) and
//    writes the 128 x K tile into tensor memory (one row per TMEM lane), where
//    it is the MMA's A operand.  Two V warpgroups take alternate units, each
//    with its own TMEM V buffer and staging buffer.
//  - Bcat[n][e*R16 + r] = B_e[c0 + n][r] for the unit's 128 columns stays in
//    shared memory while the CTA walks the row tiles of that column block
//    (K-major, 8x16-byte core matrices); it is reloaded only when the CTA
//    moves to the next column block.
//  - One thread issues the K/16 MMAs (M = N = 128) into a double-buffered
//    TMEM accumulator.  Eight epilogue warps add D to the y_base tile in
//    shared memory (128-byte swizzle), round once to bf16 and store their
//    32 x 64 piece with one TMA store; the y ring is 3 tiles deep.
//
// Units are ordered (projection, column block, row tile) and every CTA takes a
// contiguous range of them, so the work is balanced to one unit and a CTA
// loads at most a few Bcat blocks.  Every mbarrier wait is bounded (1 s): on
// expiry the CTA records APR_ERR_TIMEOUT, drains its copies and frees TMEM.
#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int BK_M = 128;           // tokens per row tile (TMEM lanes)
constexpr int BK_NT = 128;          // output columns per unit
constexpr int BK_MAXNB = 256;       // bank rank rows E * R16
constexpr int BK_MAXKR = 64;        // k * R16: a token's gated v row (registers of a V thread)
constexpr int BK_NY = 3;            // y ring depth
constexpr int BK_EPI = 256;         // warps 0-7: epilogue (column half x lane quarter)
constexpr int BK_VW = 128;          // one V warpgroup: V rows into TMEM, Bcat loads
constexpr int BK_NVG = 2;           // V warpgroups (warps 8-11 even units, 12-15 odd units)
constexpr int BK_BLOCK = BK_EPI + BK_NVG * BK_VW + 64;   // warp 16: TMA producer, warp 17: MMA issue
constexpr uint32_t BK_TMEM_COLS = 512;           // [V0 | V1 | D0 | D1], 128 columns each
constexpr int BK_YTILE = BK_M * BK_NT * 2;       // 32 KB: two 64-column halves of 128 x 128 B
constexpr int BK_BCAT = BK_MAXNB * BK_NT * 2;    // 64 KB
constexpr int BK_VC = BK_M * BK_MAXKR * 2;       // 16 KB: a tile's gated v rows (k slots of R16 bf16)

struct BankPlan {
  CUtensorMap ybase_map[APR_MAX_PROJ];   // y_base: boxes of 64 columns x 128 rows (loads)
  CUtensorMap y_map[APR_MAX_PROJ];       // y: boxes of 64 columns x 32 rows (one epilogue warp's stores)
  SgmmArgs a;
  int R16, NB;                           // rank slot per adapter, bank rows E * R16
  int nrt;                               // row tiles
  size_t vc_off;                         // scratch: gated v [proj][pair q][R16] bf16
  int cb_before[APR_MAX_PROJ + 1];       // prefix of 128-column blocks per projection
};

struct BkSmem {
  static constexpr size_t BCAT = 0;
  static constexpr size_t Y = BCAT + BK_BCAT;                        // 1024-aligned y ring
  static constexpr size_t VC = Y + (size_t)BK_NY * BK_YTILE;         // [2] gated v rows of a tile
  static constexpr size_t ZERO = VC + 2 * (size_t)BK_VC;             // 128 zero bytes
  static constexpr size_t BAR = ZERO + 128;
  static constexpr int NBAR = 2 * BK_NY + 12;
  static constexpr size_t META = BAR + NBAR * 8;
  static constexpr size_t total() { return META + 16 + 1024; }
};
static_assert(BkSmem::Y % 1024 == 0 && BK_YTILE % 1024 == 0, "swizzled boxes need 1024-byte alignment");

template <int R16>
__global__ void __launch_bounds__(BK_BLOCK, 1) bank_expand_kernel(const __grid_constant__ BankPlan P) {
  static_assert(R16 == 16 || R16 == 32 || R16 == 64, "rank slot");
  constexpr int RW = R16 / 2;                    // 32-bit words of one adapter's slot
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BkSmem::BAR);
  const uint32_t bar_yfull = smem_u32(bars);                  // [NY] y_base tile landed (TMA bytes)
  const uint32_t bar_yempty = smem_u32(bars + BK_NY);         // [NY] y tile read by the stores
  const uint32_t bar_vfull = smem_u32(bars + 2 * BK_NY);      // [2]  V rows in TMEM
  const uint32_t bar_vempty = smem_u32(bars + 2 * BK_NY + 2); // [2]  V read by the MMAs
  const uint32_t bar_dfull = smem_u32(bars + 2 * BK_NY + 4);  // [2]  accumulator ready
  const uint32_t bar_dempty = smem_u32(bars + 2 * BK_NY + 6); // [2]  accumulator read
  const uint32_t bar_bfull = smem_u32(bars + 2 * BK_NY + 8);  // Bcat loaded
  const uint32_t bar_bempty = smem_u32(bars + 2 * BK_NY + 9); // Bcat no longer read
  const uint32_t bar_vcfull = smem_u32(bars + 2 * BK_NY + 10);// [2]  a tile's gated v rows landed
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + BkSmem::META);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sB = sbase + (uint32_t)BkSmem::BCAT;
  const uint32_t sY = sbase + (uint32_t)BkSmem::Y;

  if (tid == 0) {
    for (int i = 0; i < BK_NY; ++i) {
      mbar_init(bar_yfull + 8 * i, 1);
      mbar_init(bar_yempty + 8 * i, BK_EPI / 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_vfull + 8 * i, BK_VW);
      mbar_init(bar_vempty + 8 * i, 1);
      mbar_init(bar_dfull + 8 * i, 1);
      mbar_init(bar_dempty + 8 * i, BK_EPI);
    }
    mbar_init(bar_bfull, BK_VW);
    mbar_init(bar_bempty, 1);
    mbar_init(bar_vcfull, 1);
    mbar_init(bar_vcfull + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(const_cast<uint32_t*>(s_tmem)), BK_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // the first V warpgroup stages the first column block's Bcat (weights) before waiting for
  // the preceding kernel; every other role waits first
  const bool early_bcat = tid >= BK_EPI && tid < BK_EPI + BK_VW;
  if (!early_bcat) {
    pdl_wait();
    pdl_trigger();
  }
  if (blockIdx.x == 0 && tid == 0) reinterpret_cast<WsHeader*>(a.ws)->sched = 0;   // this call's shrink is done

  const int K = a.k, T = a.T, NB = P.NB, nrt = P.nrt;
  const long nunits = (long)P.cb_before[a.nproj] * nrt;
  const long ibeg = (long)blockIdx.x * nunits / gridDim.x, iend = (long)(blockIdx.x + 1) * nunits / gridDim.x;
  const int n = (int)(iend - ibeg);
  // unit -> (projection, first column, first token, column block)
  auto unit_at = [&](int i, int& p, int& c0, int& t0, int& blk) {
    const long u = ibeg + i;
    blk = (int)(u / nrt);
    t0 = (int)(u - (long)blk * nrt) * BK_M;
    p = 0;
    while (p + 1 < a.nproj && blk >= P.cb_before[p + 1]) ++p;
    c0 = (blk - P.cb_before[p]) * BK_NT;
  };
  bool abort = false;

  if (tid < BK_EPI) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    for (int i = 0; i < n && !abort; ++i) {
      int p, c0, t0, blk;
      unit_at(i, p, c0, t0, blk);
      const int slot = i % BK_NY, db = i & 1;
      if (!mbar_wait(bar_dfull + 8 * db, (i >> 1) & 1)) { abort = true; break; }
      if (!mbar_wait(bar_yfull + 8 * slot, (i / BK_NY) & 1)) { abort = true; break; }
      tc_fence_after();
      unsigned char* yrow = smem + BkSmem::Y + (size_t)slot * BK_YTILE + (size_t)half * (BK_M * 128) + (size_t)row * 128;
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + 256u + (uint32_t)db * 128 + (uint32_t)half * 64;
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {            // 16-byte pieces (8 columns) of the row, swizzled
          uint4* pp = reinterpret_cast<uint4*>(yrow + (((4 * c32 + c8) ^ (row & 7)) << 4));
          uint4 u = *pp;
          __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const float2 f = __bfloat1622float2(hh[k2]);
            hh[k2] = __floats2bfloat162_rn(f.x + v[8 * c8 + 2 * k2], f.y + v[8 * c8 + 2 * k2 + 1]);
          }
          *pp = u;
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dempty + 8 * db);
      fence_proxy_async();                        // the tile's new bytes are visible to the TMA engine
      __syncwarp();
      if (lane == 0) {
        const int x = c0 + half * 64, y = t0 + quarter * 32;
        if (x < a.proj[p].d_out && y < T)          // rows and columns past the end are clipped by the map
          tma_store_2d(&P.y_map[p], sY + (uint32_t)slot * BK_YTILE + (uint32_t)half * (BK_M * 128) +
                                        (uint32_t)(quarter * 32) * 128, x, y);
        bulk_commit();
        bulk_wait_read_all();                      // the slot may be refilled once the store has read it
        mbar_arrive(bar_yempty + 8 * slot);
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_all();                // every y row written before the CTA ends
  } else if (tid < BK_EPI + BK_NVG * BK_VW) {
    // ---------------------------------------------------------------- V rows and Bcat
    const int vg = (tid - BK_EPI) / BK_VW;         // this warpgroup builds units i with i % 2 == vg
    const int vt = (tid - BK_EPI) % BK_VW;         // 0..127
    const int quarter = warp & 3;                  // warps 8-11 and 12-15 own TMEM lane quarters 0-3
    const int row = quarter * 32 + lane;
    const long npairs = (long)T * K;
    const uint32_t row_bytes = (uint32_t)(K * R16 * 2);          // a token's gated v row
    const __nv_bfloat16* vc = ws_at<__nv_bfloat16>(a.ws, P.vc_off);
    const uint32_t sVC = sbase + (uint32_t)BkSmem::VC + (uint32_t)vg * BK_VC, sZero = sbase + (uint32_t)BkSmem::ZERO;
    const uint32_t bar_vc = bar_vcfull + 8 * vg;
    int blk0 = 0;
    {
      int p, c0, t0;
      unit_at(0, p, c0, t0, blk0);
    }
    // Bcat[n][e*R16 + r] = B_e[c0 + n][r] of projection p's column block at c0 (zeros past a rank
    // or past d_out), K-major 8x16-byte core matrices; ends with the bfull arrival
    auto load_bcat = [&](int p, int c0) {
      const int d_out = a.proj[p].d_out;
      const int cpa = R16 / 8;                     // 16-byte chunks of one adapter's row slot
      for (int w = vt; w < a.E * BK_NT * cpa; w += BK_VW) {
        const int e = w / (BK_NT * cpa);
        const int rem = w - e * (BK_NT * cpa);
        const int nn = rem / cpa, c8 = rem - nn * cpa;
        const int re = a.ranks[e];
        const bool rank_ok = re >= 8 && re <= R16 && (re & 7) == 0;
        if (!rank_ok && nn == 0 && c8 == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e);
        const int kc = e * cpa + c8;
        const uint32_t dst = sB + (uint32_t)kc * (BK_NT / 8 * 128) + (uint32_t)(nn >> 3) * 128 + (uint32_t)(nn & 7) * 16;
        if (rank_ok && c8 * 8 < re && c0 + nn < d_out) {
          const __nv_bfloat16* B = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e]);
          cp_async16(smem + (dst - sbase), B + (size_t)(c0 + nn) * re + c8 * 8);
        } else {
          st_shared_zero16(dst);
        }
      }
      cp_async_wait_all();
      fence_proxy_async();                         // Bcat is read by the tensor core (async proxy)
      mbar_arrive(bar_bfull);
    };
    if (vg == 0) {
      if (n > 0) {                                 // unit 0 always starts a block
        int p, c0, t0, blk;
        unit_at(0, p, c0, t0, blk);
        load_bcat(p, c0);
      }
      pdl_wait();
      pdl_trigger();
    }
    // the gated v rows of unit i's tile (contiguous: tokens t0.. in pair order) -> this group's buffer
    auto issue_rows = [&](int i) {
      int p, c0, t0, blk;
      unit_at(i, p, c0, t0, blk);
      const uint32_t bytes = (uint32_t)min(BK_M, T - t0) * row_bytes;
      fence_proxy_async();                         // the buffer's last reads come before the copy's writes
      mbar_arrive_expect_tx(bar_vc, bytes);
      bulk_load_1d(sVC, vc + ((size_t)p * npairs + (size_t)t0 * K) * R16, bytes, bar_vc);
    };
    auto fetch_idx = [&](int i, int (&e)[4]) {
      int p, c0, t0, blk;
      unit_at(i, p, c0, t0, blk);
      const int t = t0 + row;
#pragma unroll
      for (int j = 0; j < 4; ++j) e[j] = (t < T && j < K) ? a.idx[(size_t)t * K + j] : -1;
    };
    // this group's V buffer starts as zeros; the zero line serves unselected rank slots
    if (vt < 8) st_shared_zero16(sZero + (uint32_t)vt * 16);
    {
      uint32_t z[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) z[c] = 0;
      for (int c = 0; c < 128; c += 32) tmem_st32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(vg * 128 + c), z);
      tmem_wait_st();
    }
    asm volatile("bar.sync 1, %0;" ::"n"(BK_NVG * BK_VW) : "memory");   // both groups: the zero line is written
    int ci[4] = {-1, -1, -1, -1};
    int issued = 0, consumed = 0;                  // row copies issued / waited for
    if (vg < n) {
      if (vt == 0) issue_rows(vg);
      issued = 1;
      fetch_idx(vg, ci);
    }
    for (int i = vg, uses = 0; i < n && !abort; i += BK_NVG, ++uses) {
      int p, c0, t0, blk;
      unit_at(i, p, c0, t0, blk);
      bool first = i == 0;
      if (!first) {
        int p2, c02, t02, blk2;
        unit_at(i - 1, p2, c02, t02, blk2);
        first = blk2 != blk;
      }
      if (first && i > 0) {
        // Bcat of a new column block (this group takes its first unit), after the MMAs are done
        // with the previous block (unit 0's block was staged before the wait above)
        const int nb = blk - blk0;                 // blocks before this one in the CTA's range
        if (!mbar_wait(bar_bempty, (nb - 1) & 1)) { abort = true; break; }
        load_bcat(p, c0);
      }
      const int vb = vg;
      if (!mbar_wait(bar_vc, uses & 1)) { abort = true; break; }
      consumed = uses + 1;
      if (i >= 2 && !mbar_wait(bar_vempty + 8 * vb, (uses - 1) & 1)) { abort = true; break; }
      tc_fence_after();
      // spread the token's k slots over the bank's E rank slots (the zero line where not selected),
      // 32 TMEM columns (32 / RW adapters) per store
      const uint32_t vaddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)vb * 128;
      const uint32_t myrow = sVC + (uint32_t)row * row_bytes;
      bool bad = false;
#pragma unroll
      for (int j = 0; j < 4; ++j) bad |= j < K && (ci[j] < 0 || ci[j] >= a.E) && t0 + row < T;
      if (bad) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, t0 + row);
      auto slot_src = [&](int e) -> uint32_t {
        uint32_t src = sZero;
#pragma unroll
        for (int j = 3; j >= 0; --j)
          if (ci[j] == e) src = myrow + (uint32_t)(j * R16 * 2);
        return src;
      };
      const int words = a.E * RW;                  // 32-bit columns of the V row
      int w0 = 0;
      for (; w0 + 32 <= words; w0 += 32) {
        uint32_t r[32];
#pragma unroll
        for (int s = 0; s < 32 / RW; ++s) {
          const uint32_t src = slot_src(w0 / RW + s);
#pragma unroll
          for (int c = 0; c < RW / 4; ++c) {
            const uint32_t a16 = src == sZero ? sZero : src + (uint32_t)c * 16;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(r[s * RW + 4 * c]), "=r"(r[s * RW + 4 * c + 1]), "=r"(r[s * RW + 4 * c + 2]),
                           "=r"(r[s * RW + 4 * c + 3])
                         : "r"(a16));
          }
        }
        tmem_st32(vaddr + (uint32_t)w0, r);
      }
      for (; w0 < words; w0 += 8) {                // a tail of 8-column pieces (E * RW not a multiple of 32)
        const int e = w0 / RW, c8 = (w0 % RW) / 8;
        const uint32_t src = slot_src(e);
        const uint32_t a16 = src == sZero ? sZero : src + (uint32_t)c8 * 32;
        uint32_t r8[8];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r8[0]), "=r"(r8[1]), "=r"(r8[2]), "=r"(r8[3]) : "r"(a16));
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r8[4]), "=r"(r8[5]), "=r"(r8[6]), "=r"(r8[7]) : "r"(src == sZero ? sZero : a16 + 16));
        tmem_st8(vaddr + (uint32_t)w0, r8);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_vfull + 8 * vb);
      // every thread of the group is done with its staging buffer before the next copy refills it
      if (vg == 0) asm volatile("bar.sync 2, %0;" ::"n"(BK_VW) : "memory");
      else asm volatile("bar.sync 3, %0;" ::"n"(BK_VW) : "memory");
      if (i + BK_NVG < n) {
        if (vt == 0) issue_rows(i + BK_NVG);
        ++issued;
        fetch_idx(i + BK_NVG, ci);
      }
    }
    cp_async_wait_all();
    // a row copy still in flight after an abort lands before the CTA exits (bounded wait)
    for (int u = consumed; u < issued; ++u) (void)mbar_wait(bar_vc, u & 1);
  } else if (warp == (BK_EPI + BK_NVG * BK_VW) / 32) {
    // ---------------------------------------------------------------- TMA producer: y_base tiles
    if (lane == 0) {
      for (int i = 0; i < n && !abort; ++i) {
        int p, c0, t0, blk;
        unit_at(i, p, c0, t0, blk);
        const int slot = i % BK_NY;
        if (i >= BK_NY && !mbar_wait(bar_yempty + 8 * slot, ((i / BK_NY) - 1) & 1)) { abort = true; break; }
        const uint32_t dst = sY + (uint32_t)slot * BK_YTILE;
        mbar_arrive_expect_tx(bar_yfull + 8 * slot, (uint32_t)BK_YTILE);
        tma_load_2d(dst, &P.ybase_map[p], c0, t0, bar_yfull + 8 * slot);
        tma_load_2d(dst + BK_M * 128, &P.ybase_map[p], c0 + 64, t0, bar_yfull + 8 * slot);
      }
    }
  } else if (lane == 0) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t id = idesc_bf16(BK_M, BK_NT);
    int prev_blk = -1, nblk = 0;
    for (int i = 0; i < n && !abort; ++i) {
      int p, c0, t0, blk;
      unit_at(i, p, c0, t0, blk);
      if (blk != prev_blk) {
        if (!mbar_wait(bar_bfull, nblk & 1)) { abort = true; break; }
        prev_blk = blk;
        ++nblk;
      }
      const int vb = i & 1;
      if (!mbar_wait(bar_vfull + 8 * vb, (i >> 1) & 1)) { abort = true; break; }
      if (i >= 2 && !mbar_wait(bar_dempty + 8 * vb, ((i >> 1) - 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const uint32_t dcol = tmem + 256u + (uint32_t)vb * 128, vcol = tmem + (uint32_t)vb * 128;
      // K step kk: B core matrices at sB + kk * 4096 (two 2048-byte K chunks); +256 in the
      // descriptor's address field (bytes / 16) per step
      const uint64_t bdesc0 = desc_k_plain(sB, BK_NT / 8 * 128, 128);
      for (int kk = 0; kk < NB / 16; ++kk)
        mma_bf16_ts(dcol, vcol + (uint32_t)kk * 8, bdesc0 + (uint64_t)kk * (2 * BK_NT / 8 * 128 / 16), id,
                    kk > 0 ? 1u : 0u);
      mma_commit(bar_dfull + 8 * vb);
      mma_commit(bar_vempty + 8 * vb);
      bool last = i + 1 >= n;
      if (!last) {
        int p2, c02, t02, blk2;
        unit_at(i + 1, p2, c02, t02, blk2);
        last = blk2 != blk;
      }
      if (last) mma_commit(bar_bempty);            // this Bcat is no longer read
    }
  }
  abort = __syncthreads_or(abort);
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, BK_TMEM_COLS);
}

// ---------------------------------------------------------------- host side

cudaError_t launch_tc_shrink_pairs(const SgmmArgs& a, size_t v_off, cudaStream_t s);

bool sgmm_bank_supported(const SgmmArgs& a, int dtype) {
  if (dtype != APR_BF16) return false;
  static_assert(BK_MAXKR == kBankMaxKR && BK_MAXNB == kBankMaxRows, "bank scratch sizing");
  if (bank_scratch_bytes(a.T, a.k, a.E, a.max_rank) == 0) return false;
  if (a.d_in % 64 != 0) return false;
  return true;
}

cudaError_t launch_sgmm_bank(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  BankPlan P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.R16 = round16i(a.max_rank);
  P.NB = a.E * P.R16;
  P.nrt = (a.T + BK_M - 1) / BK_M;
  P.vc_off = scratch_off;
  P.cb_before[0] = 0;
  cudaError_t err;
  for (int p = 0; p < a.nproj; ++p) {
    P.cb_before[p + 1] = P.cb_before[p] + (a.proj[p].d_out + BK_NT - 1) / BK_NT;
    if ((err = encode_tile_map(&P.ybase_map[p], a.proj[p].y_base, a.T, a.proj[p].d_out, BK_M)) != cudaSuccess)
      return err;
    if ((err = encode_tile_map(&P.y_map[p], a.proj[p].y, a.T, a.proj[p].d_out, 32)) != cudaSuccess) return err;
  }
  using Kern = void (*)(BankPlan);
  static SmemLimit lim[3];
  const int vi = P.R16 == 16 ? 0 : (P.R16 == 32 ? 1 : 2);
  static const Kern kerns[3] = {bank_expand_kernel<16>, bank_expand_kernel<32>, bank_expand_kernel<64>};
  const size_t smem = BkSmem::total();
  if ((err = lim[vi].ensure((const void*)kerns[vi], smem)) != cudaSuccess) return err;
  if ((err = launch_tc_shrink_pairs(a, scratch_off, s)) != cudaSuccess) return err;
  const long units = (long)P.cb_before[a.nproj] * P.nrt;
  const int nsm = device_sm_count();
  const int grid = (int)(units < nsm ? units : nsm);
  return launch_pdl(kerns[vi], dim3(grid), dim3(BK_BLOCK), smem, s, P);
}

}  // namespace apr
