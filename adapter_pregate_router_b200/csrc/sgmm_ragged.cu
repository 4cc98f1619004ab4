// SGMM for many tenants: top-1 routing over many adapters of mixed ranks
// (tcgen05).  AdaFuse summary (gist.science), Resumen tecnico §2.B: the
// segmented gather product applies each token's selected low-rank adapter to
// the tokens gathered per adapter and is fused into the add onto the base
// projection output; the Chameleon page (7minutos.es), adapter cache: tenants'
// adapters range over ranks 8-128.
//
// Two launches per call.
//
// Shrink (rg_shrink_kernel): v = g * A_e x for every token, by plan position.
// An item is one pair tile of an adapter (<= 128 tokens) and a group of
// projections; the adapter's rank rows are the MMA's M side and the tokens its
// N side, so a short segment costs only its own tokens.  A arrives by 2-D TMA
// boxes from tensor maps the kernel writes per item (a template per rank with
// the adapter's address), x rows by 16-byte cp.async; each stage packs as many
// 64-column sub-blocks of the item's own rows as fit.  The same kernel builds
// the ragged tiles and each used adapter's B tensor map for the expand.
//
// Expand (ragged_expand_kernel): with many adapters each one holds only a few
// tokens, so a tile of one adapter would leave most of the 128 MMA rows empty.
// A ragged tile is a run of consecutive plan tokens (sorted by adapter): up to
// 128 tokens of up to 16 adapters whose rank slots (each rank rounded up to
// 16) add up to <= 256.  A unit is (tile, projection, 128 output columns):
//
//   D[t, n] = sum_{s < nu} sum_{r < w_s} V[t, koff_s + r] * B_{u_s}[c0 + n, r]
//   V[t, koff_s + r] = g_t (A_{u_s} x_t)[r]  if token t selected u_s, else 0
//
//  - V: the gated v rows of a tile's tokens are contiguous (plan order); one
//    bulk copy stages them, and a warpgroup writes each token's row of V (its
//    slot, zeros elsewhere) into tensor memory, the MMA's A operand; two TMEM
//    V buffers, rebuilt when the tile or the projection changes.
//  - Bcat[n][koff_s + r] = B_{u_s}[c0 + n][r]: TMA boxes of 8 rank columns x
//    128 rows of B_{u_s}, each landing as one K chunk of 8x16-byte core
//    matrices (zeros past the rank and past d_out).
//  - y_base rows of the tile's tokens come in by 16-byte cp.async (a row's 256
//    bytes on 16 consecutive threads, 128-byte swizzle); y rows go out by
//    16-byte stores.  (Per-row TMA gather copies measured slower for both x
//    and y here.)
//  - One thread issues the kt/16 MMAs (M = N = 128) into a double-buffered
//    TMEM accumulator; eight epilogue warps add D to y_base in shared memory
//    and round once to bf16.  Two stages of (y tile, Bcat) overlap loads, MMAs
//    and stores of consecutive units.
//
// Units are ordered (tile, projection, column block) and every CTA takes a
// contiguous range of them: the work is balanced to one unit and V is rebuilt
// only when a CTA's range moves to the next (tile, projection).  Every mbarrier
// wait is bounded (1 s) and its outcome is made the same for all lanes of a warp
// (no warp can be left at a barrier its other lanes abandoned); on expiry the CTA
// records APR_ERR_TIMEOUT, drains its copies and frees its tensor memory.
#include <memory>

#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int RG_M = 128;                     // tokens per tile (TMEM lanes)
constexpr int RG_NT = 128;                    // output columns per unit
constexpr int RG_NS = 2;                      // stages of (y tile, Bcat)
constexpr int RG_EPI = 256;                   // warps 0-7: epilogue (lane quarter x column half)
constexpr int RG_VW = 128;                    // warps 8-11: V rows into TMEM
constexpr int RG_YW = 128;                    // warps 13-16: y_base rows by 16-byte cp.async
constexpr int RG_BLOCK = RG_EPI + RG_VW + 32 + RG_YW + 32;   // warp 12: Bcat by TMA, warp 17: MMA issue
constexpr uint32_t RG_TMEM_COLS = 512;        // [V0 | V1 | D0 | D1], 128 columns each
constexpr int RG_YTILE = RG_M * RG_NT * 2;    // 32 KB: two 64-column halves of 128 rows x 128 B
constexpr int RG_BCAT = kRgKmax * RG_NT * 2;  // 64 KB
constexpr int RG_VROW = 256;                  // a token's staged gated v row (R16 <= 128 bf16)

struct RgPlan {
  SgmmArgs a;
  int R16;                            // rank slot of the staged v rows
  int max_tiles;
  size_t vc_off, tiles_off, bmaps_off;   // scratch: gated v [proj][position][R16] bf16; tile count and
                                         // tiles; B tensor maps [proj][adapter]
  int cb_before[APR_MAX_PROJ + 1];    // prefix of 128-column blocks per projection
};

struct RgSmem {
  static constexpr size_t Y = 0;                                  // [NS] y tiles
  static constexpr size_t BCAT = Y + (size_t)RG_NS * RG_YTILE;    // [NS] Bcat
  static constexpr size_t VC = BCAT + (size_t)RG_NS * RG_BCAT;    // the tile's gated v rows
  static constexpr size_t ZERO = VC + (size_t)RG_M * RG_VROW;     // 128 zero bytes
  static constexpr size_t BAR = ZERO + 128;
  static constexpr int NBAR = 2 * RG_NS + 10;
  static constexpr size_t META = BAR + NBAR * 8;
  static constexpr size_t total() { return META + 16 + 1024; }
};
static_assert(RgSmem::BCAT % 1024 == 0 && RG_YTILE % 1024 == 0, "swizzled rows need 1024-byte alignment");
static_assert(RgSmem::total() <= 232448, "shared memory per block");

// ---------------------------------------------------------------- checks shared by both kernels

__device__ __forceinline__ bool rg_rank_ok(int r, int R16) { return r >= 8 && r <= R16 && (r & 7) == 0; }
__device__ __forceinline__ bool rg_ptr_ok(const void* q) { return q && (reinterpret_cast<uintptr_t>(q) & 15) == 0; }
// Adapter e of projection p has a B tensor map (built by the shrink, used by the expand).
__device__ __forceinline__ bool rg_b_ok(const SgmmArgs& a, int p, int e, int R16) {
  return e >= 0 && e < a.E && rg_rank_ok(a.ranks[e], R16) && rg_ptr_ok(a.proj[p].B[e]);
}

// ---------------------------------------------------------------- ragged tiles

// The ragged tiles of a top-1 plan, built by one warp whose lanes all hold the same walk state
// (lane s < kRgSlots also holds slot s of the open tile).  Adapters are taken in order; a tile
// closes before an adapter (or the rest of one) that would make it hold more than kSetTile
// tokens, more than kRgSlots adapters or more than kRgKmax rank rows.  The count is written even
// past `max_tiles` (the expand checks it).
__device__ void rg_plan(const SgmmArgs& a, int R16, int* count, RgTile* tiles, int max_tiles) {
  const int lane = threadIdx.x & 31;
  int t_start = 0, t_len = 0, t_nu = 0, t_kt = 0, nt = 0;
  int my_u = 0, my_koff = 0;
  auto close = [&]() {
    if (t_len > 0) {
      if (nt < max_tiles) {
        RgTile* tl = tiles + nt;
        if (lane < kRgSlots) {
          tl->u[lane] = (short)(lane < t_nu ? my_u : -1);
          tl->koff[lane] = (short)(lane < t_nu ? my_koff : t_kt);
        }
        if (lane == 0) {
          tl->start = t_start;
          tl->len = t_len;
          tl->nu = t_nu;
          tl->kt = t_kt;
        }
      }
      ++nt;
    }
    t_len = t_nu = t_kt = 0;
  };
  for (int e0 = 0; e0 < a.E; e0 += 32) {
    const int e = e0 + lane;
    int beg = 0, cnt = 0, w = 16;
    if (e < a.E) {
      beg = a.seg_off[e];
      cnt = a.seg_off[e + 1] - beg;
      const int r = a.ranks[e];
      if (rg_rank_ok(r, R16)) w = (r + 15) / 16 * 16;   // an invalid rank (reported) keeps 16 zero rows
    }
    unsigned m = __ballot_sync(0xffffffffu, cnt > 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      int c = __shfl_sync(0xffffffffu, cnt, j), pos = __shfl_sync(0xffffffffu, beg, j);
      const int wj = __shfl_sync(0xffffffffu, w, j);
      while (c > 0) {
        if (t_nu == kRgSlots || t_kt + wj > kRgKmax || t_len == kSetTile) close();
        if (t_len == 0) t_start = pos;
        const int take = min(c, kSetTile - t_len);
        if (lane == t_nu) {
          my_u = e0 + j;
          my_koff = t_kt;
        }
        ++t_nu;
        t_kt += wj;
        t_len += take;
        c -= take;
        pos += take;
      }
    }
  }
  close();
  if (lane == 0) *count = nt;
}

// ---------------------------------------------------------------- shrink

// v = g * A_e x for every pair, by plan position: [proj][position][R16] bf16 (rank rows past
// r_e are zeros).  An item is one pair tile of adapter e (<= 128 consecutive plan positions) and
// a group of <= 4 projections whose rank slots add up to <= 256.  The contraction puts the
// adapter's rank rows on the MMA's M side and the tokens on N:
//   D[j, n] = sum_k A_{q(j), e}[j mod w, k] x_{t_n}[k]   (w = round16(r_e), M = 128 per accumulator,
//                                                        N = round16(len))
// so a short segment costs only its own tokens.  A stage (64 KB) packs as many 64-column
// sub-blocks as fit the item: each holds the item's N token rows and nq * w rank rows (128-byte
// swizzled rows); an accumulator's MMAs read 128 rank rows, the rows past nq * w being whatever
// follows (the products of those rows are never read), so a small item moves up to 8 sub-blocks
// (512 columns) per stage instead of paying a fixed 128-row tile.  A setup warp prepares the next
// item (its tokens and gates, and its A tensor maps: the projection's template for rank r_e with
// A_e's address, zeros past r_e) while one warp issues the current item's A boxes (64 columns x w
// rows); four loader warps copy the tokens' x rows with 16-byte cp.async; one thread issues the
// MMAs; eight epilogue warps read D back (a TMEM lane per rank row), scale by each token's gate and
// store bf16.  Items come from a work counter (after
// one static item per CTA), so CTAs drawing high-rank adapters take fewer of them.
constexpr int RS_EPI = 256;                   // warps 2-9
constexpr int RS_XW = 128;                    // warps 10-13: x rows by 16-byte cp.async
constexpr int RS_BLOCK = 64 + RS_EPI + RS_XW + 32;   // warp 0: item setup, warp 1: MMA issue, warp 14: A boxes
constexpr int RS_STAGE = 64 * 1024;           // one stage
constexpr int RS_PAD = 128 * 128;             // after the last stage: the rank rows an MMA may read past it
constexpr int RS_MAXSB = 8;                   // 64-column sub-blocks per stage at most
constexpr int RS_NQ = 4;                      // projections per item at most

struct RsPlan {
  CUtensorMap xmap;                               // x rows (encoded with the plan; the loads are cp.async)
  CUtensorMap atmpl[APR_MAX_PROJ][APR_MAX_RANK / 8];   // A_e of rank 8 (j + 1): [r, d_in], 64 x round16(r) boxes, swizzled
  CUtensorMap btmpl[APR_MAX_PROJ][APR_MAX_RANK / 8];   // B_e of rank 8 (j + 1): [d_out, r], 8 x 128 boxes, plain
  SgmmArgs a;
  int R16, pg, npg, stages, max_tiles;
  size_t vc_off, tiles_off, amaps_off, bmaps_off;
};

struct RsItem {
  int e, q0, nq, start, len;
  int w;                                      // rank slot round16(r_e)
  int nsb;                                    // 64-column sub-blocks per stage
  int nst;                                    // stages
};

struct RsSmem {
  int S;
  size_t bar, item, gate, tok, mapbuf, tmem, total;
};
__host__ __device__ inline RsSmem rs_smem(int S) {
  RsSmem L;
  L.S = S;
  L.bar = (size_t)S * RS_STAGE + RS_PAD;
  L.item = L.bar + (size_t)(2 * S + 6) * 8;
  L.gate = L.item + 2 * sizeof(RsItem);
  L.tok = L.gate + 2 * 128 * 4;
  L.mapbuf = (L.tok + 2 * 128 * 4 + 127) / 128 * 128;
  L.tmem = L.mapbuf + (RS_NQ + 1) * 128;
  L.total = L.tmem + 16 + 1024;
  return L;
}

__global__ void __launch_bounds__(RS_BLOCK, 1) rg_shrink_kernel(const __grid_constant__ RsPlan P) {
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = P.stages, R16 = P.R16, pg = P.pg, T = a.T;
  const RsSmem L = rs_smem(S);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  const uint32_t bar_full = smem_u32(bars), bar_empty = smem_u32(bars + S);
  const uint32_t bar_ifull = smem_u32(bars + 2 * S), bar_iempty = smem_u32(bars + 2 * S + 2);
  const uint32_t bar_dfull = smem_u32(bars + 2 * S + 4), bar_dempty = smem_u32(bars + 2 * S + 5);
  RsItem* s_item = reinterpret_cast<RsItem*>(smem + L.item);
  float* s_g = reinterpret_cast<float*>(smem + L.gate);
  int* s_tok = reinterpret_cast<int*>(smem + L.tok);
  const uint32_t sbase = smem_u32(smem), s_mapbuf = sbase + (uint32_t)L.mapbuf;
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + L.tmem);

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(bar_full + 8 * i, 1 + RS_XW);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_ifull + 8 * i, 1);
      mbar_init(bar_iempty + 8 * i, 2 + RS_EPI / 32 + RS_XW / 32);   // A warp, MMA thread, epilogue and loader warps
    }
    mbar_init(bar_dfull, 1);
    mbar_init(bar_dempty, RS_EPI);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(const_cast<uint32_t*>(s_tmem)), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  pdl_wait();
  pdl_trigger();

  const WsLayout W = ws_layout(a.T, a.k, a.E);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  const PairTile* qtiles = ws_at<PairTile>(a.ws, W.qtiles);
  const long nitems = (long)hdr->n_qtiles * P.npg;
  const int nblk = a.d_in / 64;                  // 64-column blocks of d_in
  bool abort = false;
  // stage layout of an item: x sub-blocks (N rows each), then rank sub-blocks (nq * w rows each)
  auto xsub = [&](const RsItem& it, uint32_t st, int b) -> uint32_t {
    return st + (uint32_t)(b * ((it.len + 15) / 16 * 16)) * 128;
  };
  auto asub = [&](const RsItem& it, uint32_t st, int b) -> uint32_t {
    return st + (uint32_t)(it.nsb * ((it.len + 15) / 16 * 16)) * 128 + (uint32_t)(b * it.nq * it.w) * 128;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- setup and A boxes
    // the expand's B tensor maps of this CTA's share of the (projection, adapter) pairs in use
    CUtensorMap* bmaps = ws_at<CUtensorMap>(a.ws, P.bmaps_off);
    for (int pe = blockIdx.x; pe < a.nproj * a.E; pe += gridDim.x) {
      const int p = pe / a.E, e = pe - p * a.E;
      if (a.seg_off[e + 1] > a.seg_off[e] && rg_b_ok(a, p, e, R16))
        tmap_build(bmaps + pe, s_mapbuf + RS_NQ * 128, &P.btmpl[p][a.ranks[e] / 8 - 1], a.proj[p].B[e]);
    }
    CUtensorMap* amaps = ws_at<CUtensorMap>(a.ws, P.amaps_off) + (size_t)blockIdx.x * kRgMaxStages * RS_NQ;
    uint32_t k = 0;
    long item = blockIdx.x;
    while (!abort) {
      const int slot = k & 1;
      if (k >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar_iempty + 8 * slot, ((k >> 1) - 1) & 1))) {
        abort = true;
        break;
      }
      if (item >= nitems) {                            // no more work: a sentinel item
        if (lane == 0) {
          s_item[slot].e = -1;
          mbar_arrive(bar_ifull + 8 * slot);
        }
        break;
      }
      const PairTile tile = qtiles[item / P.npg];
      const int q0 = (int)(item % P.npg) * pg, nq = min(pg, a.nproj - q0), e = tile.e;
      const int r = (e >= 0 && e < a.E) ? a.ranks[e] : 0;
      bool ok = rg_rank_ok(r, R16) && tile.len > 0 && tile.len <= kSetTile;
      for (int qi = 0; qi < nq && ok; ++qi) ok = rg_ptr_ok(a.proj[q0 + qi].A[e]);
      long next = 0;
      if (lane == 0) next = (long)gridDim.x + (long)atomicAdd(&hdr->sched, 1u);
      next = __shfl_sync(0xffffffffu, next, 0);
      if (!ok) {
        if (lane == 0 && tile.len > 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e);
        item = next;
        continue;
      }
      const int len = tile.len;
      // the item's tokens (for the x loaders) and gates
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = 4 * lane + j;
        const int q = a.perm[tile.start + (row < len ? row : 0)];
        s_tok[slot * 128 + row] = q;                   // top-1: the pair id is the token
        s_g[slot * 128 + row] = row < len ? a.gate[q] : 0.f;
      }
      // sub-blocks per stage: the item's rows, plus the rank rows its last MMA reads past them
      const int w = (r + 15) / 16 * 16, N = (len + 15) / 16 * 16, arows = nq * w;
      const int slack = ((arows + 127) / 128) * 128 - arows;
      int nsb = (RS_STAGE - slack * 128) / ((N + arows) * 128);
      nsb = max(1, min(nsb, min(RS_MAXSB, nblk)));
      RsItem it;
      it.e = e;
      it.q0 = q0;
      it.nq = nq;
      it.start = tile.start;
      it.len = len;
      it.w = w;
      it.nsb = nsb;
      it.nst = (nblk + nsb - 1) / nsb;
      // the item's A maps go to map slot `slot`: free, since every copy of item k - 2 has landed
      CUtensorMap* am = amaps + (size_t)slot * RS_NQ;
      for (int qi = 0; qi < nq; ++qi)
        tmap_build(am + qi, s_mapbuf + qi * 128, &P.atmpl[q0 + qi][r / 8 - 1], a.proj[q0 + qi].A[e]);
      if (lane == 0) s_item[slot] = it;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ifull + 8 * slot);
      ++k;
      item = next;
    }
  } else if (warp == 2 + RS_EPI / 32 + RS_XW / 32) {
    // ---------------------------------------------------------------- A boxes
    const CUtensorMap* amaps = ws_at<const CUtensorMap>(a.ws, P.amaps_off) + (size_t)blockIdx.x * kRgMaxStages * RS_NQ;
    uint32_t g = 0, k = 0;
    while (true) {
      const int slot = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_ifull + 8 * slot, (k >> 1) & 1))) { abort = true; break; }
      const RsItem it = s_item[slot];
      if (it.e < 0) break;
      const CUtensorMap* am = amaps + (size_t)slot * RS_NQ;
      if (lane == 0)
        for (int qi = 0; qi < it.nq; ++qi) tmap_acquire(am + qi);
      const int arows = it.nq * it.w;
      for (int c = 0; c < it.nst; ++c, ++g) {
        const uint32_t s = g % S;
        if (g >= (uint32_t)S && !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((g / S) - 1) & 1))) {
          abort = true;
          break;
        }
        const int nb = min(it.nsb, nblk - c * it.nsb);
        const uint32_t st = sbase + s * (uint32_t)RS_STAGE;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)(nb * arows * 128));
          for (int b = 0; b < nb; ++b)
            for (int qi = 0; qi < it.nq; ++qi)
              tma_load_2d(asub(it, st, b) + (uint32_t)(qi * it.w) * 128, am + qi, 64 * (c * it.nsb + b), 0,
                          bar_full + 8 * s);
        }
        __syncwarp();
      }
      if (abort) break;
      if (lane == 0) mbar_arrive(bar_iempty + 8 * slot);
      ++k;
    }
    // after an abort, the copies of the last stages land before the CTA exits (bounded)
    if (abort && lane == 0)
      for (uint32_t j = g > (uint32_t)S ? g - S : 0; j < g; ++j) (void)mbar_wait(bar_full + 8 * (j % S), (j / S) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      uint32_t g = 0, k = 0;
      while (true) {
        const int slot = k & 1;
        if (!mbar_wait(bar_ifull + 8 * slot, (k >> 1) & 1)) { abort = true; break; }
        const RsItem it = s_item[slot];
        if (it.e < 0) break;
        const int N = (it.len + 15) / 16 * 16, nacc = (it.nq * it.w + 127) / 128;
        const uint32_t id = idesc_bf16(128, N);
        if (k >= 1 && !mbar_wait(bar_dempty, (k - 1) & 1)) { abort = true; break; }
        tc_fence_after();
        for (int c = 0; c < it.nst; ++c, ++g) {
          const uint32_t s = g % S;
          if (!mbar_wait(bar_full + 8 * s, (g / S) & 1)) { abort = true; break; }
          tc_fence_after();
          const int nb = min(it.nsb, nblk - c * it.nsb);
          const uint32_t st = sbase + s * (uint32_t)RS_STAGE;
          for (int b = 0; b < nb; ++b)
            for (int m = 0; m < nacc; ++m)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + (uint32_t)m * 128, desc_k_sw128(asub(it, st, b) + (uint32_t)m * (128 * 128) + kk * 32),
                         desc_k_sw128(xsub(it, st, b) + kk * 32), id, (c > 0 || b > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_empty + 8 * s);
        }
        if (abort) break;
        mma_commit(bar_dfull);
        mbar_arrive(bar_iempty + 8 * slot);            // every copy of the item has landed: its maps are free
        ++k;
      }
    }
  } else if (warp >= 2 + RS_EPI / 32) {
    // ---------------------------------------------------------------- x loaders
    // per sub-block, thread xt copies 16-byte piece (xt & 7) of token rows (xt >> 3) + 16 m: 8
    // consecutive threads per 128-byte row piece, into the 128-byte swizzled rows
    const int xt = tid - (64 + RS_EPI);
    const int chunk = xt & 7, r0 = xt >> 3;
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    uint32_t g = 0, k = 0;
    while (true) {
      const int slot = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_ifull + 8 * slot, (k >> 1) & 1))) { abort = true; break; }
      const RsItem it = s_item[slot];
      if (it.e < 0) break;
      int tok[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int r = r0 + 16 * m;
        tok[m] = r < it.len ? s_tok[slot * 128 + r] : -1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_iempty + 8 * slot);   // the item's tokens are in registers
      for (int c = 0; c < it.nst; ++c, ++g) {
        const uint32_t s = g % S;
        if (g >= (uint32_t)S && !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((g / S) - 1) & 1))) {
          abort = true;
          break;
        }
        const int nb = min(it.nsb, nblk - c * it.nsb);
        const uint32_t st = sbase + s * (uint32_t)RS_STAGE;
        for (int b = 0; b < nb; ++b) {
          const uint32_t xs = xsub(it, st, b);
          const __nv_bfloat16* src = x + 64 * (c * it.nsb + b) + chunk * 8;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int r = r0 + 16 * m;
            if (tok[m] >= 0)
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(xs + (uint32_t)r * 128 + (uint32_t)((chunk ^ (r & 7)) << 4)),
                           "l"(src + (size_t)tok[m] * a.d_in)
                           : "memory");
          }
        }
        cp_async_arrive(bar_full + 8 * s);
      }
      if (abort) break;
      ++k;
    }
    cp_async_wait_all();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2, quarter = warp & 3;
    if (ew == 0 && blockIdx.x == gridDim.x - 1) {
      int* cnt = ws_at<int>(a.ws, P.tiles_off);
      rg_plan(a, R16, cnt, reinterpret_cast<RgTile*>(cnt + 4), P.max_tiles);
    }
    __nv_bfloat16* vc = ws_at<__nv_bfloat16>(a.ws, P.vc_off);
    uint32_t k = 0;
    while (true) {
      const int slot = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_ifull + 8 * slot, (k >> 1) & 1))) { abort = true; break; }
      const RsItem it = s_item[slot];
      if (it.e < 0) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dfull, k & 1))) { abort = true; break; }
      tc_fence_after();
      const int N = (it.len + 15) / 16 * 16, nacc = (it.nq * it.w + 127) / 128;
      // two accumulators: warps 2-5 read the first, 6-9 the second; one: they split the columns
      const int m = nacc == 2 ? (ew >> 2) : 0, csel = nacc == 2 ? -1 : (ew >> 2);
      const int j = 128 * m + 32 * quarter + lane;       // rank row of this TMEM lane
      const int qi = j / it.w, rr = j - qi * it.w;
      const bool valid = qi < it.nq;
      __nv_bfloat16* dst = vc + ((size_t)(it.q0 + qi) * T + it.start) * R16 + rr;
      const float* gg = s_g + slot * 128;
      for (int c16 = 0; c16 < N / 16; ++c16) {
        if (csel >= 0 && (c16 & 1) != csel) continue;
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)m * 128 + (uint32_t)c16 * 16, v);
        if (valid) {
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int n = c16 * 16 + t;
            if (n < it.len) dst[(size_t)n * R16] = __float2bfloat16_rn(v[t] * gg[n]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dempty);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_iempty + 8 * slot);
      ++k;
    }
  }
  abort = __syncthreads_or(abort);
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- expand

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
  const uint32_t bar_vcfree = smem_u32(bars + 2 * RG_NS + 9);  // staged v rows read by every V thread
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + RgSmem::META);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sY = sbase + (uint32_t)RgSmem::Y, sB = sbase + (uint32_t)RgSmem::BCAT;

  if (tid == 0) {
    for (int i = 0; i < RG_NS; ++i) {
      mbar_init(bar_full + 8 * i, 1 + RG_YW);
      mbar_init(bar_empty + 8 * i, RG_EPI / 32 + 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_vfull + 8 * i, RG_VW);
      mbar_init(bar_vempty + 8 * i, 1);
      mbar_init(bar_dfull + 8 * i, 1);
      mbar_init(bar_dempty + 8 * i, RG_EPI);
    }
    mbar_init(bar_vc, 1);
    mbar_init(bar_vcfree, RG_VW);
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
      bool ok = mbar_wait(bar_dfull + 8 * db, (i >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bar_full + 8 * s, (i / RG_NS) & 1));
      if (!ok) { abort = true; break; }
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
      __syncwarp();
      const int x = c0 + half * 64;
      if (nvalid > 0 && x < d_out) {
        // the warp's rows by 16-byte stores: 8 lanes per 128-byte row piece, 4 rows per pass
        __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.proj[p].y);
        const int col = half * 64 + (lane & 7) * 8;
#pragma unroll
        for (int it4 = 0; it4 < 8; ++it4) {
          const int rr = 4 * it4 + (lane >> 3);
          const int tk = __shfl_sync(0xffffffffu, tok, rr);
          if (rr < nvalid && c0 + col < d_out) {
            const int r = quarter * 32 + rr;
            const uint4 val = *reinterpret_cast<const uint4*>(yhalf + (size_t)r * 128 + (((lane & 7) ^ (r & 7)) << 4));
            __stcs(reinterpret_cast<uint4*>(y + (size_t)tk * d_out + c0 + col), val);
          }
        }
      }
      __syncwarp();                                    // the stores have read the stage
      if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }
  } else if (tid < RG_EPI + RG_VW) {
    // ---------------------------------------------------------------- V rows into TMEM
    const int vt = tid - RG_EPI;
    const int quarter = warp & 3;                      // warps 8-11: TMEM lane quarters 0-3
    const int row = quarter * 32 + lane;
    const uint32_t sVC = sbase + (uint32_t)RgSmem::VC, sZero = sbase + (uint32_t)RgSmem::ZERO;
    const __nv_bfloat16* vc = ws_at<__nv_bfloat16>(a.ws, P.vc_off);
    const uint32_t row_bytes = (uint32_t)R16 * 2;
    if (vt < 8) st_shared_zero16(sZero + (uint32_t)vt * 16);
    asm volatile("bar.sync 1, %0;" ::"n"(RG_VW) : "memory");   // the zero line is written (no wait before)
    // the gated v rows of unit i's tile and projection (contiguous in plan order); copy j reuses
    // the staging buffer once every V thread has read copy j - 1
    auto issue_rows = [&](int i, int j) -> bool {
      if (j > 0 && !mbar_wait(bar_vcfree, (j - 1) & 1)) return false;
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const RgTile& tl = tiles[ti];
      const uint32_t bytes = (uint32_t)tl.len * row_bytes;
      fence_proxy_async();                             // earlier reads of the buffer come before the copy
      mbar_arrive_expect_tx(bar_vc, bytes);
      bulk_load_1d(sVC, vc + ((size_t)p * T + tl.start) * R16, bytes, bar_vc);
      return true;
    };
    // the adapter of this thread's token in unit i's tile (-1: no token)
    auto fetch_adapter = [&](int i) -> int {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const RgTile& tl = tiles[ti];
      return row < tl.len ? a.idx[a.perm[tl.start + row]] : -1;
    };
    int issued = 0, consumed = 0, item = 0, e_next = -1;
    if (n > 0) {
      if (vt == 0) (void)issue_rows(0, 0);
      issued = 1;
      e_next = fetch_adapter(0);
    }
    for (int i = 0; i < n && !abort; ++i) {
      if (!new_v(i)) continue;
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const int vb = item & 1;
      bool ok = mbar_wait(bar_vc, item & 1);
      if (ok) consumed = item + 1;
      if (item >= 2) ok = ok && mbar_wait(bar_vempty + 8 * vb, ((item >> 1) - 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) { abort = true; break; }
      tc_fence_after();
      const RgTile& tl = tiles[ti];
      const int kt = tl.kt, nu = tl.nu;
      const int e = e_next;
      // this token's slot (words of 32 bits: two bf16 rank rows)
      int ko = 0, wd = 0;
      if (e >= 0) {
        int q = 0;
        while (q < nu && tl.u[q] != e) ++q;
        if (q < nu) {
          ko = tl.koff[q] / 2;
          wd = ((q + 1 < nu ? tl.koff[q + 1] : kt) - tl.koff[q]) / 2;
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
      mbar_arrive(bar_vcfree);                          // this thread no longer reads the staged rows
      ++item;
      int nx = i + 1;
      while (nx < n && !new_v(nx)) ++nx;
      if (nx < n) {
        bool sent = true;
        if (vt == 0) sent = issue_rows(nx, item);
        if (!__all_sync(0xffffffffu, sent)) { abort = true; break; }   // warp 8; the others time out on the copy
        ++issued;
        e_next = fetch_adapter(nx);
      }
    }
    // a row copy still in flight after an abort lands before the CTA exits (bounded wait)
    for (int u = consumed; u < issued; ++u) (void)mbar_wait(bar_vc, u & 1);
  } else if (tid < RG_EPI + RG_VW + 32) {
    // ---------------------------------------------------------------- producer warp: y_base rows, Bcat
    // lane q < nu owns slot q of the current (tile, projection): the tensor map of B_{u_q} (built by
    // the shrink), its first 16-byte K chunk and chunks per row; an invalid slot is zeros
    const CUtensorMap* bmaps = ws_at<const CUtensorMap>(a.ws, P.bmaps_off);
    const CUtensorMap* my_map = nullptr;
    int my_kc0 = 0, my_cps = 0, bbytes = 0;
    int cur_ti = -1, cur_p = -1, len = 0, tk[4] = {0, 0, 0, 0};
    int last = -1;                                     // last unit whose stage this warp filled
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const int s = i % RG_NS;
      if (i >= RG_NS && !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((i / RG_NS) - 1) & 1))) {
        abort = true;
        break;
      }
      const RgTile& tl = tiles[ti];
      const bool new_tile = ti != cur_ti, new_proj = new_tile || p != cur_p;
      cur_ti = ti;
      cur_p = p;
      (void)tk;
      (void)len;
      if (new_proj) {
        const int nu = tl.nu;
        my_map = nullptr;
        my_cps = 0;
        if (lane < nu) {
          const int e = tl.u[lane], ko = tl.koff[lane];
          const int w = (lane + 1 < nu ? tl.koff[lane + 1] : tl.kt) - ko;
          my_kc0 = ko / 8;
          my_cps = w / 8;
          if (rg_b_ok(a, p, e, R16)) {
            my_map = bmaps + (size_t)p * a.E + e;
            tmap_acquire(my_map);
          }
        }
        bbytes = __reduce_add_sync(0xffffffffu, my_map ? my_cps * (RG_NT * 16) : 0);
      }
      const int d_out = a.proj[p].d_out;
      const uint32_t ys = sY + (uint32_t)s * RG_YTILE, bs = sB + (uint32_t)s * RG_BCAT;
      // an invalid slot: zero chunks by plain stores, ordered before the arrival below
      if (!my_map && my_cps > 0) {
        for (int c = 0; c < my_cps; ++c)
          for (int r16 = 0; r16 < RG_NT; ++r16) st_shared_zero16(bs + (uint32_t)(my_kc0 + c) * (RG_NT * 16) + (uint32_t)r16 * 16);
        fence_proxy_async();
      }
      __syncwarp();
      (void)ys;
      (void)d_out;
      if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)bbytes);
      __syncwarp();
      // Bcat chunk kc = rank rows 8c..8c+7 of the slot for the unit's 128 columns: one box of 8
      // columns x 128 rows of B, which lands as the chunk's 16 core matrices (zeros past the rank
      // and past d_out)
      if (my_map)
        for (int c = 0; c < my_cps; ++c)
          tma_load_2d(bs + (uint32_t)(my_kc0 + c) * (RG_NT * 16), my_map, 8 * c, c0, bar_full + 8 * s);
      last = i;
    }
    // after an abort, the copies of the stages filled last land before the CTA exits (bounded)
    if (abort && lane == 0)
      for (int i = max(last - RG_NS + 1, 0); i <= last; ++i) (void)mbar_wait(bar_full + 8 * (i % RG_NS), (i / RG_NS) & 1);
  } else if (tid < RG_EPI + RG_VW + 32 + RG_YW) {
    // ---------------------------------------------------------------- y_base rows
    // thread yt copies 16-byte pieces yt, yt + 128, ... of the unit's 128 rows x 256 bytes (16
    // pieces per row, a row's pieces on consecutive threads) into the 128-byte swizzled halves
    const int yt = tid - (RG_EPI + RG_VW + 32);
    const int q = yt & 15, half = q >> 3, chunk = q & 7, r0 = yt >> 4;   // rows r0, r0 + 8, ...
    int cur_ti = -1, len = 0, tok[16];
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      const int s = i % RG_NS;
      if (i >= RG_NS && !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((i / RG_NS) - 1) & 1))) {
        abort = true;
        break;
      }
      if (ti != cur_ti) {
        cur_ti = ti;
        const RgTile& tl = tiles[ti];
        len = tl.len;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int r = r0 + 8 * m;
          tok[m] = r < len ? a.perm[tl.start + r] : -1;
        }
      }
      const int d_out = a.proj[p].d_out;
      const int col = c0 + half * 64 + chunk * 8;
      const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].y_base) + col;
      const uint32_t ys = sY + (uint32_t)s * RG_YTILE + (uint32_t)half * (RG_M * 128);
      if (col < d_out) {
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int r = r0 + 8 * m;
          if (tok[m] >= 0)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ys + (uint32_t)r * 128 + (uint32_t)((chunk ^ (r & 7)) << 4)),
                         "l"(yb + (size_t)tok[m] * d_out)
                         : "memory");
        }
      }
      cp_async_arrive(bar_full + 8 * s);
    }
    cp_async_wait_all();
  } else if (lane == 0) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t id = idesc_bf16(RG_M, RG_NT);
    int item = -1, kt = 0;
    for (int i = 0; i < n && !abort; ++i) {
      int ti, p, c0;
      unit_at(i, ti, p, c0);
      if (new_v(i)) {
        kt = tiles[ti].kt;
        ++item;
        if (!mbar_wait(bar_vfull + 8 * (item & 1), (item >> 1) & 1)) { abort = true; break; }
      }
      const int vb = item & 1, s = i % RG_NS, db = i & 1;
      if (!mbar_wait(bar_full + 8 * s, (i / RG_NS) & 1)) { abort = true; break; }
      if (i >= 2 && !mbar_wait(bar_dempty + 8 * db, ((i >> 1) - 1) & 1)) { abort = true; break; }
      tc_fence_after();
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
  const int R16 = round16i(a.max_rank);
  const int nsm = device_sm_count();
  cudaError_t err;
  // ---- shrink
  std::unique_ptr<RsPlan> S(new RsPlan);
  memset(S.get(), 0, sizeof(RsPlan));
  S->a = a;
  S->R16 = R16;
  S->pg = 256 / R16 < a.nproj ? 256 / R16 : a.nproj;
  if (S->pg > RS_NQ) S->pg = RS_NQ;
  S->npg = (a.nproj + S->pg - 1) / S->pg;
  S->stages = 3;
  if (S->stages > kRgMaxStages) S->stages = kRgMaxStages;
  S->max_tiles = rg_max_tiles(a.T, a.E);
  S->vc_off = scratch_off;
  S->tiles_off = scratch_off + rg_vc_bytes(a.T, a.max_rank);
  S->amaps_off = scratch_off + rg_amaps_off(a.T, a.E, a.max_rank);
  S->bmaps_off = scratch_off + rg_bmaps_off(a.T, a.E, a.max_rank);
  if ((err = encode_row_map(&S->xmap, const_cast<void*>(a.x), a.T, a.d_in)) != cudaSuccess) return err;
  for (int p = 0; p < a.nproj; ++p)
    for (int r = 8; r <= R16; r += 8) {
      if ((err = cached_box_map(&S->atmpl[p][r / 8 - 1], a.x, r, a.d_in, (long)a.d_in * 2, 64, round16i(r), true)) !=
          cudaSuccess)
        return err;
      if ((err = cached_box_map(&S->btmpl[p][r / 8 - 1], a.x, a.proj[p].d_out, r, (long)r * 2, 8, RG_NT, false)) !=
          cudaSuccess)
        return err;
    }
  // ---- expand
  RgPlan P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.R16 = R16;
  P.max_tiles = S->max_tiles;
  P.vc_off = S->vc_off;
  P.tiles_off = S->tiles_off;
  P.bmaps_off = S->bmaps_off;
  P.cb_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) {
    P.cb_before[p + 1] = P.cb_before[p] + (a.proj[p].d_out + RG_NT - 1) / RG_NT;
  }
  static SmemLimit lim1, lim2;
  const size_t smem1 = rs_smem(S->stages).total, smem2 = RgSmem::total();
  if ((err = lim1.ensure((const void*)rg_shrink_kernel, smem1)) != cudaSuccess) return err;
  if ((err = lim2.ensure((const void*)ragged_expand_kernel, smem2)) != cudaSuccess) return err;
  const long items = (long)max_qtiles(a.T, a.k, a.E) * S->npg;
  long g1 = items < nsm ? items : nsm;
  if (g1 > kRgMaxCtas) g1 = kRgMaxCtas;
  if ((err = launch_pdl(rg_shrink_kernel, dim3((unsigned)g1), dim3(RS_BLOCK), smem1, s, *S)) != cudaSuccess) return err;
  const long units = (long)P.max_tiles * P.cb_before[a.nproj];
  const int grid = (int)(units < nsm ? units : nsm);
  return launch_pdl(ragged_expand_kernel, dim3(grid), dim3(RG_BLOCK), smem2, s, P);
}

}  // namespace apr
