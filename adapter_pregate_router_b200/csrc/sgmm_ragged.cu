// SGMM expand for many tenants: top-1 routing over many adapters of mixed
// ranks (tcgen05).  AdaFuse summary (gist.science), Resumen tecnico §2.B: the
// segmented gather product applies each token's selected low-rank adapter to
// the tokens gathered per adapter and is fused into the add onto the base
// projection output; the Chameleon page (7minutos.es), adapter cache: tenants'
// adapters range over ranks 8-128.
//
// With many adapters each one holds only a few tokens, so a tile of one
// adapter leaves most of the 128 MMA rows empty.  Here a tile is a ragged run
// of consecutive plan tokens (sorted by adapter): up to 128 tokens of up to 16
// adapters whose rank slots (each rank rounded up to 16) add up to <= 256.  The
// shrink (tc_shrink_kernel) leaves g * A_e x of every token in plan order and
// builds the tiles.  A unit is (tile, projection, 128 output columns):
//
//   D[t, n] = sum_{s < nu} sum_{r < w_s} V[t, koff_s + r] * B_{u_s}[c0 + n, r]
//   V[t, koff_s + r] = g_t (A_{u_s} x_t)[r]  if token t selected u_s, else 0
//
//  - V: the gated v rows of a tile's tokens are contiguous (plan order); one
//    bulk copy stages them, and a warpgroup writes each token's row of V (its
//    slot, zeros elsewhere) into tensor memory, the MMA's A operand; two TMEM
//    V buffers, rebuilt when the tile or the projection changes.
//  - Bcat[n][koff_s + r] = B_{u_s}[c0 + n][r]: 16-byte cp.async from four
//    producer warps into K-major 8x16-byte core matrices (zeros past a rank).
//  - y_base rows of the tile's tokens come in by TMA tile::gather4 (four token
//    rows of 64 columns per copy, 128-byte swizzle); y rows go out by
//    tile::scatter4 (groups of four tokens) and 16-byte stores (the rest).
//  - One thread issues the kt/16 MMAs (M = N = 128) into a double-buffered
//    TMEM accumulator; eight epilogue warps add D to y_base in shared memory
//    and round once to bf16.  Two stages of (y tile, Bcat) overlap loads, MMAs
//    and stores of consecutive units.
//
// Units are ordered (tile, projection, column block) and every CTA takes a
// contiguous range of them: the work is balanced to one unit and V is rebuilt
// only when a CTA's range moves to the next (tile, projection).  Every mbarrier
// wait is bounded (1 s): on expiry the CTA records APR_ERR_TIMEOUT, drains its
// copies and frees its tensor memory.
#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int RG_M = 128;                     // tokens per tile (TMEM lanes)
constexpr int RG_NT = 128;                    // output columns per unit
constexpr int RG_NS = 2;                      // stages of (y tile, Bcat)
constexpr int RG_EPI = 256;                   // warps 0-7: epilogue (lane quarter x column half)
constexpr int RG_VW = 128;                    // warps 8-11: V rows into TMEM
constexpr int RG_PW = 128;                    // warps 12-15: Bcat; warp 12 also gathers y_base rows
constexpr int RG_BLOCK = RG_EPI + RG_VW + RG_PW + 32;   // warp 16: MMA issue
constexpr uint32_t RG_TMEM_COLS = 512;        // [V0 | V1 | D0 | D1], 128 columns each
constexpr int RG_YTILE = RG_M * RG_NT * 2;    // 32 KB: two 64-column halves of 128 rows x 128 B
constexpr int RG_BCAT = kRgKmax * RG_NT * 2;  // 64 KB
constexpr int RG_VROW = 256;                  // a token's staged gated v row (R16 <= 128 bf16)

struct RgPlan {
  CUtensorMap yb_map[APR_MAX_PROJ];   // y_base rows: 64-column boxes, gather4 loads
  CUtensorMap y_map[APR_MAX_PROJ];    // y rows: 64-column boxes, scatter4 stores
  SgmmArgs a;
  int R16;                            // rank slot of the staged v rows
  int max_tiles;
  size_t vc_off, tiles_off;           // scratch: gated v [proj][position][R16] bf16; tile count, tiles
  int cb_before[APR_MAX_PROJ + 1];    // prefix of 128-column blocks per projection
};

struct RgSmem {
  static constexpr size_t Y = 0;                                  // [NS] y tiles
  static constexpr size_t BCAT = Y + (size_t)RG_NS * RG_YTILE;    // [NS] Bcat
  static constexpr size_t VC = BCAT + (size_t)RG_NS * RG_BCAT;    // the tile's gated v rows
  static constexpr size_t ZERO = VC + (size_t)RG_M * RG_VROW;     // 128 zero bytes
  static constexpr size_t BAR = ZERO + 128;
  static constexpr int NBAR = 2 * RG_NS + 9;
  static constexpr size_t META = BAR + NBAR * 8;
  static constexpr size_t total() { return META + 16 + 1024; }
};
static_assert(RgSmem::BCAT % 1024 == 0 && RG_YTILE % 1024 == 0, "swizzled rows need 1024-byte alignment");
static_assert(RgSmem::total() <= 232448, "shared memory per block");

__global__ void __launch_bounds__(RG_BLOCK, 1) ragged_expand_kernel(const __grid_constant__ RgPlan P) {
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RgSmem::BAR);
  const uint32_t bar_full = smem_u32(bars);                    // [NS] y_base rows (bytes) and Bcat landed
  const uint32_t bar_empty = smem_u32(bars + RG_NS);           // [NS] stage read by the MMAs and the stores
  const uint32_t bar_vfull = smem_u32(bars + 2 * RG_NS);       // [2]  V rows in TMEM
  const uint32_t bar_vempty = smem_u32(bars + 2 * RG_NS + 2);  // [2]  V read by the MMAs
  const uint32_t bar_dfull = smem_u32(bars + 2 * RG_NS + 4);   // [2]  accumulator ready
  const uint32_t bar_dempty = smem_u32(bars + 2 * RG_NS + 6);  // [2]  accumulator read
  const uint32_t bar_vc = smem_u32(bars + 2 * RG_NS + 8);      // staged v rows landed
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + RgSmem::META);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sY = sbase + (uint32_t)RgSmem::Y, sB = sbase + (uint32_t)RgSmem::BCAT;

  if (tid == 0) {
    for (int i = 0; i < RG_NS; ++i) {
      mbar_init(bar_full + 8 * i, RG_PW + 1);
      mbar_init(bar_empty + 8 * i, RG_EPI / 32 + 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_vfull + 8 * i, RG_VW);
      mbar_init(bar_vempty + 8 * i, 1);
      mbar_init(bar_dfull + 8 * i, 1);
      mbar_init(bar_dempty + 8 * i, RG_EPI);
    }
    mbar_init(bar_vc, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(const_cast<uint32_t*>(s_tmem)), RG_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && tid == 0) reinterpret_cast<WsHeader*>(a.ws)->sched = 0;   // this call's shrink is done

  const int* tcount = ws_at<int>(a.ws, P.tiles_off);
  const RgTile* tiles = reinterpret_cast<const RgTile*>(tcount + 4);
  int ntiles = *tcount;
  if (ntiles > P.max_tiles) {
    if (tid == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, ntiles);
    ntiles = P.max_tiles;
  }
  const int T = a.T, R16 = P.R16, CB = P.cb_before[a.nproj];
  const long nunits = (long)ntiles * CB;
  const long ibeg = (long)blockIdx.x * nunits / gridDim.x, iend = (long)(blockIdx.x + 1) * nunits / gridDim.x;
  const int n = (int)(iend - ibeg);
  // unit -> (tile, projection, first column)
  auto unit_at = [&](int i, int& ti, int& p, int& c0) {
    const long u = ibeg + i;
    ti = (int)(u / CB);
    const int rem = (int)(u - (long)ti * CB);
    p = 0;
    while (p + 1 < a.nproj && rem >= P.cb_before[p + 1]) ++p;
    c0 = (rem - P.cb_before[p]) * RG_NT;
  };
  // does unit i start a new (tile, projection), i.e. a new V?
  auto new_v = [&](int i) -> bool {
    if (i == 0) return true;
    int ti, p, c0, ti2, p2, c02;
    unit_at(i, ti, p, c0);
    unit_at(i - 1, ti2, p2, c02);
    return ti != ti2 || p != p2;
  };
  bool abort = false;

  if (tid < RG_EPI) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    int cur_ti = -1, len = 0, tok = -1;
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      if (ti != cur_ti) {
        cur_ti = ti;
        len = tiles[ti].len;
        tok = row < len ? a.perm[tiles[ti].start + row] : -1;
      }
      const int s = i % RG_NS, db = i & 1;
      if (!mbar_wait(bar_dfull + 8 * db, (i >> 1) & 1)) { abort = true; break; }
      if (!mbar_wait(bar_full + 8 * s, (i / RG_NS) & 1)) { abort = true; break; }
      tc_fence_after();
      const int d_out = a.proj[p].d_out;
      const int nvalid = min(max(len - quarter * 32, 0), 32);        // the warp's rows that hold tokens
      unsigned char* yhalf = smem + RgSmem::Y + (size_t)s * RG_YTILE + (size_t)half * (RG_M * 128);
      if (nvalid > 0) {
        unsigned char* yrow = yhalf + (size_t)row * 128;
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + 256u + (uint32_t)db * 128 + (uint32_t)half * 64;
#pragma unroll
        for (int c32 = 0; c32 < 2; ++c32) {
          float v[32];
          tmem_ld32(taddr + (uint32_t)(c32 * 32), v);
          if (tok >= 0) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {          // 16-byte pieces (8 columns) of the row, swizzled
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
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dempty + 8 * db);
      fence_proxy_async();                            // the new bytes are visible to the TMA engine
      __syncwarp();
      const int x = c0 + half * 64;
      if (nvalid > 0 && x < d_out) {
        // groups of four token rows by tile::scatter4 (the map clips columns past d_out)
        const int ng = nvalid >> 2;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int t0 = __shfl_sync(0xffffffffu, tok, 4 * g), t1 = __shfl_sync(0xffffffffu, tok, 4 * g + 1);
          const int t2 = __shfl_sync(0xffffffffu, tok, 4 * g + 2), t3 = __shfl_sync(0xffffffffu, tok, 4 * g + 3);
          if (lane == 0 && g < ng)
            tma_scatter4(&P.y_map[p], x, t0, t1, t2, t3,
                         smem_u32(yhalf + (size_t)(quarter * 32 + 4 * g) * 128));
        }
        // the last one to three rows by 16-byte stores, 8 lanes per row
        const int rr = 4 * ng + (lane >> 3);
        const int tk = __shfl_sync(0xffffffffu, tok, rr);
        const int col = half * 64 + (lane & 7) * 8;
        if (rr < nvalid && c0 + col < d_out) {
          const int r = quarter * 32 + rr;
          const uint4 val = *reinterpret_cast<const uint4*>(yhalf + (size_t)r * 128 + (((lane & 7) ^ (r & 7)) << 4));
          __stcs(reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.proj[p].y) + (size_t)tk * d_out + c0 + col),
                 val);
        }
      }
      if (lane == 0) {
        bulk_commit();
        bulk_wait_read_all();                          // the stage may be refilled once the copies read it
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }
    if (lane == 0) bulk_wait_all();                    // every y row written before the CTA ends
  } else if (tid < RG_EPI + RG_VW) {
    // ---------------------------------------------------------------- V rows into TMEM
    const int vt = tid - RG_EPI;
    const int quarter = warp & 3;                      // warps 8-11: TMEM lane quarters 0-3
    const int row = quarter * 32 + lane;
    const uint32_t sVC = sbase + (uint32_t)RgSmem::VC, sZero = sbase + (uint32_t)RgSmem::ZERO;
    const __nv_bfloat16* vc = ws_at<__nv_bfloat16>(a.ws, P.vc_off);
    const uint32_t row_bytes = (uint32_t)R16 * 2;
    if (vt < 8) st_shared_zero16(sZero + (uint32_t)vt * 16);
    asm volatile("bar.sync 1, %0;" ::"n"(RG_VW) : "memory");
    // the gated v rows of unit i's tile and projection (contiguous in plan order)
    auto issue_rows = [&](int i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const RgTile& tl = tiles[ti];
      const uint32_t bytes = (uint32_t)tl.len * row_bytes;
      fence_proxy_async();                             // earlier reads of the buffer come before the copy
      mbar_arrive_expect_tx(bar_vc, bytes);
      bulk_load_1d(sVC, vc + ((size_t)p * T + tl.start) * R16, bytes, bar_vc);
    };
    // the adapter of this thread's token in unit i's tile (-1: no token)
    auto fetch_adapter = [&](int i) -> int {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const RgTile& tl = tiles[ti];
      return row < tl.len ? a.idx[a.perm[tl.start + row]] : -1;
    };
    int issued = 0, consumed = 0, item = 0, e_next = -1;
    int i = 0;
    if (n > 0) {
      if (vt == 0) issue_rows(0);
      issued = 1;
      e_next = fetch_adapter(0);
    }
    for (; i < n && !abort; ++i) {
      if (!new_v(i)) continue;
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const int vb = item & 1;
      if (!mbar_wait(bar_vc, item & 1)) { abort = true; break; }
      consumed = item + 1;
      if (item >= 2 && !mbar_wait(bar_vempty + 8 * vb, ((item >> 1) - 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const RgTile& tl = tiles[ti];
      const int kt = tl.kt, nu = tl.nu;
      const int e = e_next;
      // this token's slot (words of 32 bits: two bf16 rank rows)
      int ko = 0, wd = 0;
      if (e >= 0) {
        int s = 0;
        while (s < nu && tl.u[s] != e) ++s;
        if (s < nu) {
          ko = tl.koff[s] / 2;
          wd = ((s + 1 < nu ? tl.koff[s + 1] : kt) - tl.koff[s]) / 2;
        } else {
          report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e);
        }
      }
      const uint32_t myrow = sVC + (uint32_t)row * row_bytes;
      const uint32_t vaddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)vb * 128;
      auto piece = [&](int pw) -> uint32_t {         // 16-byte piece at word pw of the row: v or zeros
        return (pw >= ko && pw < ko + wd) ? myrow + (uint32_t)(pw - ko) * 4 : sZero;
      };
      const int words = kt / 2;
      int w0 = 0;
      for (; w0 + 32 <= words; w0 += 32) {
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(r[4 * j]), "=r"(r[4 * j + 1]), "=r"(r[4 * j + 2]), "=r"(r[4 * j + 3])
                       : "r"(piece(w0 + 4 * j)));
        tmem_st32(vaddr + (uint32_t)w0, r);
      }
      for (; w0 < words; w0 += 8) {
        uint32_t r8[8];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r8[0]), "=r"(r8[1]), "=r"(r8[2]), "=r"(r8[3]) : "r"(piece(w0)));
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r8[4]), "=r"(r8[5]), "=r"(r8[6]), "=r"(r8[7]) : "r"(piece(w0 + 4)));
        tmem_st8(vaddr + (uint32_t)w0, r8);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_vfull + 8 * vb);
      ++item;
      asm volatile("bar.sync 1, %0;" ::"n"(RG_VW) : "memory");   // the staged rows are no longer read
      int nx = i + 1;
      while (nx < n && !new_v(nx)) ++nx;
      if (nx < n) {
        if (vt == 0) issue_rows(nx);
        ++issued;
        e_next = fetch_adapter(nx);
      }
    }
    // a row copy still in flight after an abort lands before the CTA exits (bounded wait)
    for (int u = consumed; u < issued; ++u) (void)mbar_wait(bar_vc, u & 1);
  } else if (tid < RG_EPI + RG_VW + RG_PW) {
    // ---------------------------------------------------------------- producers: y_base rows, Bcat
    const int pt = tid - RG_EPI - RG_VW;
    const bool gatherer = pt < 32;                     // warp 12 issues the y_base gathers
    int cur_ti = -1, len = 0, start = 0, tk[4] = {0, 0, 0, 0};
    int last = -1;                                     // last unit whose stage this thread filled
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const int s = i % RG_NS;
      if (i >= RG_NS && !mbar_wait(bar_empty + 8 * s, ((i / RG_NS) - 1) & 1)) { abort = true; break; }
      const RgTile& tl = tiles[ti];
      if (ti != cur_ti) {
        cur_ti = ti;
        len = tl.len;
        start = tl.start;
        if (gatherer) {
          // rows 4 * lane .. + 3; rows past the tile repeat its first token (loaded, never stored)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int r = 4 * lane + q;
            tk[q] = a.perm[start + (r < len ? r : 0)];
          }
        }
      }
      const int d_out = a.proj[p].d_out;
      const uint32_t ys = sY + (uint32_t)s * RG_YTILE, bs = sB + (uint32_t)s * RG_BCAT;
      if (gatherer) {
        const int nh = c0 + 64 < d_out ? 2 : 1, ngr = (len + 3) >> 2;
        if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)(ngr * nh * 512));
        __syncwarp();
        if (lane < ngr)
          for (int h = 0; h < nh; ++h)
            tma_gather4(ys + (uint32_t)h * (RG_M * 128) + (uint32_t)(4 * lane) * 128, &P.yb_map[p], c0 + 64 * h, tk[0],
                        tk[1], tk[2], tk[3], bar_full + 8 * s);
      }
      // Bcat: every slot's 128 rows x w_s/8 16-byte chunks (zeros past the rank or past d_out)
      const int nu = tl.nu, kt = tl.kt;
      bool zeros = false;
      for (int q = 0; q < nu; ++q) {
        const int e = tl.u[q], ko = tl.koff[q];
        const int w = (q + 1 < nu ? tl.koff[q + 1] : kt) - ko;
        const int r = (e >= 0 && e < a.E) ? a.ranks[e] : 0;
        const bool rank_ok = r >= 8 && r <= w && (r & 7) == 0;
        const __nv_bfloat16* B = rank_ok ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e]) : nullptr;
        const int cps = w / 8;
        for (int w8 = pt; w8 < RG_NT * cps; w8 += RG_PW) {
          const int nn = w8 / cps, c = w8 - nn * cps;
          const uint32_t dst = bs + (uint32_t)(ko / 8 + c) * (RG_NT / 8 * 128) + (uint32_t)(nn >> 3) * 128 +
                               (uint32_t)(nn & 7) * 16;
          if (B && c * 8 < r && c0 + nn < d_out) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(B + (size_t)(c0 + nn) * r + c * 8)
                         : "memory");
          } else {
            st_shared_zero16(dst);
            zeros = true;
          }
        }
      }
      if (zeros) fence_proxy_async();
      cp_async_arrive(bar_full + 8 * s);
      last = i;
    }
    cp_async_wait_all();
    // after an abort, the gathers of the stages filled last land before the CTA exits (bounded)
    if (abort && gatherer && lane == 0)
      for (int i = max(last - RG_NS + 1, 0); i <= last; ++i) (void)mbar_wait(bar_full + 8 * (i % RG_NS), (i / RG_NS) & 1);
  } else if (lane == 0) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t id = idesc_bf16(RG_M, RG_NT);
    int item = -1;
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      if (new_v(i)) {
        ++item;
        if (!mbar_wait(bar_vfull + 8 * (item & 1), (item >> 1) & 1)) { abort = true; break; }
      }
      const int vb = item & 1, s = i % RG_NS, db = i & 1;
      if (!mbar_wait(bar_full + 8 * s, (i / RG_NS) & 1)) { abort = true; break; }
      if (i >= 2 && !mbar_wait(bar_dempty + 8 * db, ((i >> 1) - 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const int kt = tiles[ti].kt;
      const uint32_t dcol = tmem + 256u + (uint32_t)db * 128, vcol = tmem + (uint32_t)vb * 128;
      // K step kk: B core matrices at bs + kk * 4096 (two 2048-byte K chunks): +256 in the
      // descriptor's address field (bytes / 16) per step
      const uint64_t bdesc0 = desc_k_plain(sB + (uint32_t)s * RG_BCAT, RG_NT / 8 * 128, 128);
      for (int kk = 0; kk < kt / 16; ++kk)
        mma_bf16_ts(dcol, vcol + (uint32_t)kk * 8, bdesc0 + (uint64_t)kk * (2 * RG_NT / 8 * 128 / 16), id,
                    kk > 0 ? 1u : 0u);
      mma_commit(bar_dfull + 8 * db);
      mma_commit(bar_empty + 8 * s);
      if (i + 1 >= n || new_v(i + 1)) mma_commit(bar_vempty + 8 * vb);   // this V is no longer read
    }
  }
  abort = __syncthreads_or(abort);
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, RG_TMEM_COLS);
}

// ---------------------------------------------------------------- host side

bool sgmm_ragged_supported(const SgmmArgs& a, int dtype) {
  return dtype == APR_BF16 && rg_dims_ok(a.k, a.max_rank) && a.d_in % 64 == 0;
}

cudaError_t launch_sgmm_ragged(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  RgPlan P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.R16 = round16i(a.max_rank);
  P.max_tiles = rg_max_tiles(a.T, a.E);
  P.vc_off = scratch_off;
  P.tiles_off = scratch_off + rg_vc_bytes(a.T, a.max_rank);
  P.cb_before[0] = 0;
  cudaError_t err;
  for (int p = 0; p < a.nproj; ++p) {
    P.cb_before[p + 1] = P.cb_before[p] + (a.proj[p].d_out + RG_NT - 1) / RG_NT;
    if ((err = encode_row_map(&P.yb_map[p], const_cast<void*>(a.proj[p].y_base), a.T, a.proj[p].d_out)) != cudaSuccess)
      return err;
    if ((err = encode_row_map(&P.y_map[p], a.proj[p].y, a.T, a.proj[p].d_out)) != cudaSuccess) return err;
  }
  static SmemLimit lim;
  const size_t smem = RgSmem::total();
  if ((err = lim.ensure((const void*)ragged_expand_kernel, smem)) != cudaSuccess) return err;
  if ((err = launch_tc_shrink_ragged(a, P.vc_off, P.tiles_off, P.max_tiles, s)) != cudaSuccess) return err;
  const long units = (long)P.max_tiles * P.cb_before[a.nproj];
  const int nsm = device_sm_count();
  const int grid = (int)(units < nsm ? units : nsm);
  return launch_pdl(ragged_expand_kernel, dim3(grid), dim3(RG_BLOCK), smem, s, P);
}

}  // namespace apr
