// SGMM on the 5th-generation tensor cores (tcgen05) for long segments
// (prefill, many tenants).  AdaFuse summary (gist.science), Resumen tecnico
// §2.B: the segmented gather product applies the selected low-rank adapters to
// the tokens gathered per adapter in one batched product, fused into the add
// onto the base projection output.
//
// Two persistent kernels, one CTA per SM:
//
//  shrink  item = one pair tile (<= 128 token/slot pairs routed to the same
//          adapter e, in plan order) and a group of projections (all of them
//          when nproj * R16 <= 256; R16 = max rank rounded up to 16).
//          D1[128 x N1] = X_tile . [A_{q,e}]_q^T on tcgen05 (kind::f16, bf16
//          in, fp32 in TMEM): the tile's x rows are gathered 64 columns per
//          stage with 16-byte cp.async into 128B-swizzled K-major stages, the
//          A rows likewise; the copies complete on the stage's mbarrier, one
//          thread of the MMA warp issues the MMAs and commits them to the
//          stage's "empty" barrier.  Full tiles of one adapter keep the work
//          balanced and read each A_e once per 128 pairs.  The epilogue reads
//          D1 back (one TMEM lane per pair), scales by the pair's gate and
//          stores v as bf16 hi + lo halves (~16 mantissa bits) in the pair's
//          row of the plan order: V[q][pos][hi: R16 | lo: R16].
//  expand  item = (tile, projection, 1024 output columns).  A tile is a
//          mixed tile (<= 128 consecutive plan tokens whose adapters number
//          <= 4; slots u0 < u1 < u2 < u3) when 4 * R16 <= 64, else a set tile
//          (<= 128 tokens sharing the same k <= 2 adapters).  Per 128-column
//          tile D2[128 x 128] = V_hi . Bcat^T + V_lo . Bcat^T with V[t] =
//          [v(t, u0) | ... ] (zero where t did not select the slot's adapter)
//          and Bcat[n] = [B_u0[n] | ...], TMEM double buffered.
//          Warp-specialised: 8 producer warps gather V rows, y_base rows and
//          Bcat with cp.async into a 3-4 deep ring, one thread issues the
//          MMAs, and 8 epilogue warps compute y = y_base + D2 for their row
//          and half in shared memory, round once to bf16 and store: a warp
//          whose 32 rows all hold tokens by TMA tile::scatter4 (four token
//          rows per copy), others by coalesced 128-byte row segments.  Loads,
//          MMAs and stores of different tiles overlap.
//
// Every mbarrier wait is bounded by the global timer (1 s); on expiry the CTA
// records APR_ERR_TIMEOUT, drains its copies and frees its TMEM.
#include <memory>

#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int TB_M = 128;          // rows per tile (= kSetTile)
constexpr int TB_BK = 64;          // input columns per shrink stage
constexpr int TB_MAXN1 = 256;      // shrink accumulator columns
constexpr int TB_MAXK2 = 64;       // k * R16 handled by the expand
constexpr int TB_NT = 128;         // output columns per expand tile
constexpr int TB_CW = 1024;        // output columns per expand item
constexpr int SH_WORKERS = 256;    // shrink: warps 0-7 load and run the epilogue, warp 8 issues MMAs
constexpr int SH_BLOCK = SH_WORKERS + 32;
constexpr int EX_PROD = 256;       // expand: warps 0-7 load
constexpr int EX_EPI = 256;        // expand: warps 8-15 run the epilogue
constexpr int EX_BLOCK = EX_PROD + EX_EPI + 32;   // warp 16 issues MMAs
constexpr int SMEM_BUDGET = 200 * 1024;

struct TcPlan {
  CUtensorMap ymap[APR_MAX_PROJ];    // expand: y of each projection as rows for tile::scatter4 stores
  CUtensorMap atmpl[APR_MAX_PROJ][APR_MAX_RANK / 8];   // shrink: A_e of rank 8 (j + 1), [r, d_in], 64 x R16 boxes
  SgmmArgs a;
  int R16;                           // rank slot per adapter
  int K2;                            // k * R16
  int pg;                            // projections per shrink item
  int npg;                           // shrink items per pair tile
  int stages;                        // shrink pipeline depth
  int ny;                            // expand ring depth
  int mixed;                         // expand over mixed tiles (<= 4 adapters, K2 = 4 * R16) instead of set tiles
  int ytma;                          // expand stores y rows with tile::scatter4 (else plain stores)
  int vpair;                         // shrink writes v by pair id, bf16 only ([proj][q][R16]) instead of
                                     // by plan position as bf16 hi | lo ([proj][pair position][2 * R16])
  size_t vprep_off;                  // scratch: V rows
  size_t amaps_off;                  // scratch: each shrink CTA's A tensor maps [CTA][projection]
  int cc_before[APR_MAX_PROJ + 1];   // expand: prefix of 1024-column items per projection
};

static_assert(TB_MAXK2 == kTensorMaxK2, "tensor scratch sizing");

// ---------------------------------------------------------------- shrink

struct ShSmem {
  int stage_bytes, stages;
  size_t bar, meta, mapbuf, total;
};
__host__ __device__ inline ShSmem sh_smem(int n1max, int stages) {
  ShSmem L;
  L.stage_bytes = TB_M * 128 + n1max * 128;
  L.stages = stages;
  L.bar = (size_t)stages * L.stage_bytes;
  L.meta = L.bar + (size_t)(2 * stages + 1) * 8;
  L.mapbuf = (L.meta + 3 * TB_M * 4 + 16 + TB_MAXN1 * 8 + 127) / 128 * 128;
  L.total = L.mapbuf + APR_MAX_PROJ * 128 + 1024;
  return L;
}

__global__ void __launch_bounds__(SH_BLOCK, 1) tc_shrink_kernel(const __grid_constant__ TcPlan P) {
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool worker = tid < SH_WORKERS;
  const int K = a.k, R16 = P.R16, S = P.stages;
  const ShSmem L = sh_smem(P.pg * R16, S);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  const uint32_t bar_full = smem_u32(bars), bar_empty = smem_u32(bars + S), bar_d1 = smem_u32(bars + 2 * S);
  int* s_tok = reinterpret_cast<int*>(smem + L.meta);
  float* s_g = reinterpret_cast<float*>(s_tok + TB_M);
  volatile int* s_flags = reinterpret_cast<volatile int*>(s_g + TB_M);      // [0] tmem [1] bad
  int* s_pair = reinterpret_cast<int*>(smem + L.meta + 2 * TB_M * 4 + 16 + TB_MAXN1 * 8);
  const uint32_t sbase = smem_u32(smem);

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(bar_full + 8 * i, SH_WORKERS + 1);   // the x copies of every worker, the A boxes' bytes
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_d1, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(const_cast<int*>(s_flags)), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)s_flags[0];

  pdl_wait();
  pdl_trigger();

  const WsLayout W = ws_layout(a.T, a.k, a.E);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  const PairTile* qtiles = ws_at<PairTile>(a.ws, W.qtiles);
  __nv_bfloat16* vprep = ws_at<__nv_bfloat16>(a.ws, P.vprep_off);
  const long nitems = (long)hdr->n_qtiles * P.npg;
  const long npairs = (long)a.T * K;
  const __nv_bfloat16* __restrict__ x = reinterpret_cast<const __nv_bfloat16*>(a.x);
  const int d_in = a.d_in, nk = d_in / TB_BK;
  uint32_t gchunk = 0, nitem = 0;
  bool abort = false;

  // items are taken from a work counter (after one static item per CTA), so CTAs that
  // draw small tiles take more of them
  auto fetch_next = [&]() {
    if (tid == 0) s_flags[2] = (int)gridDim.x + (int)atomicAdd(&hdr->sched, 1u);
  };
  for (long item = blockIdx.x; item < nitems;) {
    const PairTile tile = qtiles[item / P.npg];
    const int q0 = (int)(item % P.npg) * P.pg;
    const int nq = min(P.pg, a.nproj - q0);
    const int N1 = nq * R16;
    const int e = tile.e;
    if (tid < TB_M) {
      int tok = -1, q = -1;
      float g = 0.f;
      if (tid < tile.len) {
        q = a.perm[tile.start + tid];
        tok = q / K;
        g = a.gate[q];
      }
      s_tok[tid] = tok;
      s_pair[tid] = q;
      s_g[tid] = g;
      if (tid == 0) {
        const int r = (e >= 0 && e < a.E) ? a.ranks[e] : 0;
        bool bad = r < 8 || r > R16 || (r & 7);
        for (int qi = 0; qi < nq && !bad; ++qi) {
          const void* A = a.proj[q0 + qi].A[e];
          bad = !A || (reinterpret_cast<uintptr_t>(A) & 15);
        }
        s_flags[1] = bad ? 1 : 0;
        if (bad) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e);
      }
    }
    __syncthreads();
    if (s_flags[1] || tile.len <= 0 || abort) {
      fetch_next();
      __syncthreads();
      item = s_flags[2];
      continue;
    }
    // the item's A tensor maps (one per projection: the template for rank r_e with A_e's address;
    // rows past r_e are zeros by the map's bounds).  This CTA's maps are rewritten only after the
    // previous item's copies have all landed (its epilogue waited for the MMAs).
    CUtensorMap* am = ws_at<CUtensorMap>(a.ws, P.amaps_off) + (size_t)blockIdx.x * APR_MAX_PROJ;
    if (warp == 0) {
      const int re = a.ranks[e];
      for (int qi = 0; qi < nq; ++qi)
        tmap_build(am + qi, sbase + (uint32_t)L.mapbuf + qi * 128, &P.atmpl[q0 + qi][re / 8 - 1], a.proj[q0 + qi].A[e]);
      if (lane == 0)
        for (int qi = 0; qi < nq; ++qi) tmap_acquire(am + qi);
    }
    const uint32_t g0 = gchunk;
    if (worker) {
      // this thread's copies of every stage of the item, fixed across the stages: four 16-byte
      // pieces of x rows (source advanced by 64 columns per stage; a null source is a missing pair)
      const __nv_bfloat16* xs[TB_M * 8 / SH_WORKERS];
      uint32_t xo[TB_M * 8 / SH_WORKERS];
#pragma unroll
      for (int m = 0; m < TB_M * 8 / SH_WORKERS; ++m) {   // x rows: 8 lanes per 128-byte row segment
        const int w = tid + m * SH_WORKERS;
        const int row = w >> 3, q = w & 7;
        const int tk = s_tok[row];
        xs[m] = tk >= 0 ? x + (size_t)tk * d_in + q * 8 : nullptr;
        xo[m] = (uint32_t)row * 128 + (uint32_t)((q ^ (row & 7)) << 4);
      }
      for (int c = 0; c < nk && !abort; ++c) {
        const uint32_t g = g0 + c, s = g % S;
        if (g >= (uint32_t)S && !mbar_wait(bar_empty + 8 * s, ((g / S) - 1) & 1)) { abort = true; break; }
        const uint32_t st_base = sbase + s * L.stage_bytes;
        const size_t col = (size_t)c * TB_BK;
        // A rows: one box of 64 columns x R16 rows per projection, issued by thread 0
        if (tid == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)(N1 * 128));
          for (int qi = 0; qi < nq; ++qi)
            tma_load_2d(st_base + TB_M * 128 + (uint32_t)(qi * R16) * 128, am + qi, (int)col, 0, bar_full + 8 * s);
        }
#pragma unroll
        for (int m = 0; m < TB_M * 8 / SH_WORKERS; ++m)
          if (xs[m])
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(st_base + xo[m]), "l"(xs[m] + col)
                         : "memory");
        cp_async_arrive(bar_full + 8 * s);
      }
      // gate -> V rows (bf16 hi | lo) at the pair's plan position
      if (!abort && !mbar_wait(bar_d1, nitem & 1)) abort = true;
      tc_fence_after();
      if (!abort) {
        const int row = tid & (TB_M - 1), half = tid >> 7;      // the two warpgroups split the columns
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const bool valid = row < tile.len;
        const float gg = s_g[row];
        for (int c0 = half * 16; c0 < N1; c0 += 32) {
          float v[16];
          tmem_ld16(lane_addr + (uint32_t)c0, v);
          const int qi = c0 / R16, rr = c0 - qi * R16;
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a0 = v[2 * i] * gg, a1 = v[2 * i + 1] * gg;
            const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            const float2 hf = __bfloat1622float2(h);
            hi[i] = *reinterpret_cast<const uint32_t*>(&h);
            lo[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
          }
          if (valid && P.vpair) {
            __nv_bfloat16* dst = vprep + ((size_t)(q0 + qi) * npairs + s_pair[row]) * R16 + rr;
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
          } else if (valid) {
            __nv_bfloat16* dst = vprep + ((size_t)(q0 + qi) * npairs + tile.start + row) * (2 * R16) + rr;
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            reinterpret_cast<uint4*>(dst + R16)[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            reinterpret_cast<uint4*>(dst + R16)[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
          }
        }
      }
    } else if (lane == 0) {
      const uint32_t id = idesc_bf16(TB_M, N1);
      for (int c = 0; c < nk && !abort; ++c) {
        const uint32_t g = g0 + c, s = g % S;
        if (!mbar_wait(bar_full + 8 * s, (g / S) & 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t xs = sbase + s * L.stage_bytes, as = xs + TB_M * 128;
#pragma unroll
        for (int kk = 0; kk < TB_BK / 16; ++kk)
          mma_bf16(tmem, desc_k_sw128(xs + kk * 32), desc_k_sw128(as + kk * 32), id, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_empty + 8 * s);
      }
      if (!abort) mma_commit(bar_d1);
    }
    gchunk = g0 + nk;
    ++nitem;
    fetch_next();
    tc_fence_before();
    abort = __syncthreads_or(abort);
    tc_fence_after();
    item = s_flags[2];
  }
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- expand

struct ExSmem {
  int K2, ny;
  size_t vbuf, y, b, tok, bar, total;
};
__host__ __device__ inline ExSmem ex_smem(int K2, int ny) {
  ExSmem L;
  L.K2 = K2;
  L.ny = ny;
  L.vbuf = (size_t)2 * TB_M * K2 * 2;                 // one V buffer: hi then lo
  L.y = 2 * L.vbuf;                                   // ring of y tiles [2 halves][128 rows][128 B]
  L.b = L.y + (size_t)ny * TB_M * 256;                // ring of Bcat tiles [128][K2] bf16
  L.tok = L.b + (size_t)ny * TB_NT * K2 * 2;          // [2][128] token of each row
  L.bar = L.tok + 2 * TB_M * 4;
  L.total = L.bar + (size_t)(2 * ny + 12) * 8 + 16 + 1024;
  return L;
}

__global__ void __launch_bounds__(EX_BLOCK, 1) tc_expand_kernel(const __grid_constant__ TcPlan P) {
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.k, R16 = P.R16, K2 = P.K2, NY = P.ny;
  const ExSmem L = ex_smem(K2, NY);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  const uint32_t bar_tfull = smem_u32(bars);                  // [NY] tile operands landed
  const uint32_t bar_tempty = smem_u32(bars + NY);            // [NY] tile slot stored out
  const uint32_t bar_vfull = smem_u32(bars + 2 * NY);         // [2]  V of an item landed
  const uint32_t bar_vempty = smem_u32(bars + 2 * NY + 2);    // [2]  V of an item consumed by the MMAs
  const uint32_t bar_d2full = smem_u32(bars + 2 * NY + 4);    // [2]  accumulator ready
  const uint32_t bar_d2empty = smem_u32(bars + 2 * NY + 6);   // [2]  accumulator read
  const uint32_t bar_mfull = smem_u32(bars + 2 * NY + 8);     // [2]  row tokens of an item written
  const uint32_t bar_mempty = smem_u32(bars + 2 * NY + 10);   // [2]  item finished by the epilogue
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(bars + 2 * NY + 12);
  int* s_tok = reinterpret_cast<int*>(smem + L.tok);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t SBO = (uint32_t)(K2 / 8) * 128;              // next 8-row group of a K-major operand

  if (tid == 0) {
    for (int i = 0; i < NY; ++i) {
      mbar_init(bar_tfull + 8 * i, EX_PROD);
      mbar_init(bar_tempty + 8 * i, EX_EPI);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_vfull + 8 * i, EX_PROD);
      mbar_init(bar_vempty + 8 * i, 1);
      mbar_init(bar_d2full + 8 * i, 1);
      mbar_init(bar_d2empty + 8 * i, EX_EPI);
      mbar_init(bar_mfull + 8 * i, EX_PROD);
      mbar_init(bar_mempty + 8 * i, EX_EPI);
    }
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
  if (blockIdx.x == 0 && tid == 0) hdr->sched = 0;      // this call's shrink is complete
  const int* tok_order = ws_at<int>(a.ws, W.tok_order);
  const int* inv = ws_at<int>(a.ws, W.inv);
  const SetTile* stiles = ws_at<SetTile>(a.ws, W.stiles);
  const MixTile* mtiles = ws_at<MixTile>(a.ws, W.mtiles);
  const __nv_bfloat16* vprep = ws_at<__nv_bfloat16>(a.ws, P.vprep_off);
  const long npairs = (long)a.T * K;
  const int ipt = P.cc_before[a.nproj];
  const int nsl = P.mixed ? kMixAdapters : K;                  // adapter slots of the contraction
  const long nitems = (long)(P.mixed ? hdr->n_mtiles : hdr->n_stiles) * ipt;
  // each CTA takes a contiguous block of items, so consecutive items mostly share a tile (its
  // tokens and adapters stay loaded) and a projection (its V stays loaded)
  const long ibeg = (long)blockIdx.x * nitems / gridDim.x, iend = (long)(blockIdx.x + 1) * nitems / gridDim.x;
  auto item_at = [&](int i) -> long { return ibeg + i < iend ? ibeg + i : nitems; };
  // item -> (set tile, projection, first column, 128-column tiles)
  auto item_shape = [&](long it, int& st, int& p, int& n0, int& ntl, int& d_out) {
    st = (int)(it / ipt);
    const int loc = (int)(it - (long)st * ipt);
    p = 0;
    while (p + 1 < a.nproj && loc >= P.cc_before[p + 1]) ++p;
    d_out = a.proj[p].d_out;
    n0 = (loc - P.cc_before[p]) * TB_CW;
    ntl = (min(TB_CW, d_out - n0) + TB_NT - 1) / TB_NT;
  };
  bool abort = false;

  if (tid < EX_PROD) {
    // ---------------------------------------------------- producer
    const int ptid = tid;
    uint32_t gp = 0;
    int mcnt = -1, vcnt = -1, st_prev = -1, p_prev = -1;
    int tstart = 0, tlen = 0, tok = -1, su[kMixAdapters] = {-1, -1, -1, -1}, rs[kMixAdapters] = {0, 0, 0, 0};
    int ej[2] = {-2, -2};
    bool bad = false;
    const int prow = ptid & (TB_M - 1), phalf = ptid >> 7;
    const __nv_bfloat16* Bs[kMixAdapters] = {nullptr, nullptr, nullptr, nullptr};
    for (int i = 0; item_at(i) < nitems && !abort; ++i) {
      int st, p, n0, ntl, d_out;
      item_shape(item_at(i), st, p, n0, ntl, d_out);
      const bool newM = st != st_prev, newV = newM || p != p_prev;
      st_prev = st;
      p_prev = p;
      if (newM) {
        // the tile's tokens and its adapter slots (ascending; -1: an empty slot)
        const int mb = (++mcnt) & 1;
        if (mcnt >= 2 && !mbar_wait(bar_mempty + 8 * mb, ((mcnt >> 1) - 1) & 1)) { abort = true; break; }
        for (int q = 0; q < kMixAdapters; ++q) { su[q] = -1; rs[q] = 0; }
        if (P.mixed) {
          const MixTile mt = mtiles[st];
          tstart = mt.start;
          tlen = mt.len;
          for (int q = 0; q < kMixAdapters; ++q) su[q] = q < mt.nu ? mt.u[q] : -1;
        } else {
          const SetTile tile = stiles[st];
          tstart = tile.start;
          tlen = tile.len;
          const int t0 = tok_order[tile.start];
          int e0 = a.idx[(size_t)t0 * K], e1 = K == 2 ? a.idx[(size_t)t0 * K + 1] : -1;
          if (K == 2 && e1 < e0) { const int te = e0; e0 = e1; e1 = te; }
          su[0] = e0;
          su[1] = e1;
        }
        bad = false;
        for (int q = 0; q < nsl; ++q) {
          if (su[q] < 0) continue;
          if (su[q] >= a.E) { bad = true; continue; }
          rs[q] = a.ranks[su[q]];
          bad |= rs[q] < 8 || rs[q] > R16 || (rs[q] & 7);
        }
        if (bad && ptid == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, su[0]);
        tok = (!bad && prow < tlen) ? tok_order[tstart + prow] : -1;
        ej[0] = ej[1] = -2;
        if (tok >= 0)
          for (int j = 0; j < K && j < 2; ++j) ej[j] = a.idx[(size_t)tok * K + j];
        if (phalf == 0) s_tok[mb * TB_M + prow] = tok;
        asm volatile("bar.sync 1, %0;" ::"n"(EX_PROD) : "memory");     // every row's token is in shared memory
        mbar_arrive(bar_mfull + 8 * mb);
      }
      if (newV) {
        // V rows: slot q of row `prow` = v of its pair on adapter su[q] (hi or lo half), else zero
        const int vb = (++vcnt) & 1;
        if (vcnt >= 2 && !mbar_wait(bar_vempty + 8 * vb, ((vcnt >> 1) - 1) & 1)) { abort = true; break; }
        const uint32_t vbase = sbase + (uint32_t)(vb * L.vbuf) + (uint32_t)phalf * (TB_M * K2 * 2);
        for (int q = 0; q < nsl; ++q) {
          const __nv_bfloat16* src = nullptr;
          if (tok >= 0 && su[q] >= 0) {
            const int j = ej[0] == su[q] ? 0 : (ej[1] == su[q] ? 1 : -1);
            if (j >= 0) src = vprep + ((size_t)p * npairs + inv[(size_t)tok * K + j]) * (2 * R16) + phalf * R16;
          }
          for (int c = 0; c < R16 / 8; ++c) {
            const int kq = q * (R16 / 8) + c;
            const uint32_t off = (uint32_t)(prow >> 3) * SBO + (uint32_t)kq * 128 + (uint32_t)(prow & 7) * 16;
            if (src)
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(vbase + off), "l"(src + c * 8) : "memory");
            else
              st_shared_zero16(vbase + off);
          }
        }
        fence_proxy_async();
        cp_async_arrive(bar_vfull + 8 * vb);
        for (int q = 0; q < kMixAdapters; ++q)
          Bs[q] = (!bad && q < nsl && su[q] >= 0) ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[su[q]]) : nullptr;
      }
      const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].y_base);
      for (int t = 0; t < ntl; ++t, ++gp) {
        const uint32_t slot = gp % NY;
        if (gp >= (uint32_t)NY && !mbar_wait(bar_tempty + 8 * slot, ((gp / NY) - 1) & 1)) { abort = true; break; }
        const int c0 = n0 + t * TB_NT;
        const uint32_t ybuf = sbase + (uint32_t)L.y + slot * (TB_M * 256);
#pragma unroll 4
        for (int m = 0; m < TB_M * 16 / EX_PROD; ++m) {   // y_base rows: 8 lanes per 128-byte half-row segment
          const int w = ptid + m * EX_PROD;
          const int row = w >> 4, hs = (w >> 3) & 1, q = w & 7;
          const int tk = s_tok[(mcnt & 1) * TB_M + row];
          const int col = c0 + hs * 64 + q * 8;
          if (tk >= 0 && col < d_out)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ybuf + (uint32_t)hs * (TB_M * 128) +
                                                                            (uint32_t)row * 128 +
                                                                            (uint32_t)((q ^ (row & 7)) << 4)),
                         "l"(yb + (size_t)tk * d_out + col)
                         : "memory");
        }
        // Bcat: real chunks by cp.async; zero chunks (past a rank, an empty slot, past d_out) by
        // plain stores when the slot's previous content may differ (the item's first tiles, the edge)
        const uint32_t bbuf = sbase + (uint32_t)L.b + slot * (uint32_t)(TB_NT * K2 * 2);
        const int cpr = K2 / 8, cps = R16 / 8;
        const bool rezero = t < NY || c0 + TB_NT > d_out;
        for (int w = ptid; w < TB_NT * cpr; w += EX_PROD) {
          const int n = w / cpr, kq = w - n * cpr;
          const int sa = kq / cps, cq = kq - sa * cps;
          const __nv_bfloat16* B = Bs[sa];
          const int re = rs[sa];
          const bool ok = B != nullptr && c0 + n < d_out && cq * 8 < re;
          const uint32_t dst = bbuf + (uint32_t)(n >> 3) * SBO + (uint32_t)kq * 128 + (uint32_t)(n & 7) * 16;
          if (ok)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(B + (size_t)(c0 + n) * re + cq * 8)
                         : "memory");
          else if (rezero)
            st_shared_zero16(dst);
        }
        if (rezero) fence_proxy_async();
        cp_async_arrive(bar_tfull + 8 * slot);
      }
    }
  } else if (tid < EX_PROD + EX_EPI) {
    // ---------------------------------------------------- epilogue
    const int eid = tid - EX_PROD;
    const int row = eid & (TB_M - 1), half = eid >> 7;
    const int wrow0 = (warp & 3) * 32;
    uint32_t g = 0;
    int mcnt = -1, st_prev = -1, tok = -1;
    bool live = true;
    for (int i = 0; item_at(i) < nitems && !abort; ++i) {
      int st, p, n0, ntl, d_out;
      item_shape(item_at(i), st, p, n0, ntl, d_out);
      if (st != st_prev) {
        const int mb = (++mcnt) & 1;
        if (!mbar_wait(bar_mfull + 8 * mb, (mcnt >> 1) & 1)) { abort = true; break; }
        tok = s_tok[mb * TB_M + row];
        live = __any_sync(0xffffffffu, tok >= 0);       // a warp whose 32 rows are all empty skips the work
      }
      st_prev = st;
      __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.proj[p].y);
      for (int t = 0; t < ntl; ++t, ++g) {
        const uint32_t slot = g % NY, b = g & 1;
        if (!mbar_wait(bar_tfull + 8 * slot, (g / NY) & 1)) { abort = true; break; }
        if (!mbar_wait(bar_d2full + 8 * b, (g >> 1) & 1)) { abort = true; break; }
        tc_fence_after();
        const int c0 = n0 + t * TB_NT;
        const int ncols = min(TB_NT, d_out - c0);
        unsigned char* ytile = smem + L.y + (size_t)slot * (TB_M * 256);
        unsigned char* yhalf = ytile + (size_t)half * (TB_M * 128);
        unsigned char* yrow = yhalf + (size_t)row * 128;
        const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + b * 128 + (uint32_t)half * 64;
#pragma unroll
        for (int c16 = 0; c16 < 4 && live; ++c16) {
          float v[16];
          tmem_ld16(taddr + (uint32_t)(c16 * 16), v);
          if (tok >= 0) {
            uint4* p0 = reinterpret_cast<uint4*>(yrow + (((2 * c16) ^ (row & 7)) << 4));
            uint4* p1 = reinterpret_cast<uint4*>(yrow + (((2 * c16 + 1) ^ (row & 7)) << 4));
            uint4 u0 = *p0, u1 = *p1;
            __nv_bfloat162* h0 = reinterpret_cast<__nv_bfloat162*>(&u0);
            __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&u1);
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const float2 f0 = __bfloat1622float2(h0[k2]);
              const float2 f1 = __bfloat1622float2(h1[k2]);
              h0[k2] = __floats2bfloat162_rn(f0.x + v[2 * k2], f0.y + v[2 * k2 + 1]);
              h1[k2] = __floats2bfloat162_rn(f1.x + v[8 + 2 * k2], f1.y + v[8 + 2 * k2 + 1]);
            }
            *p0 = u0;
            *p1 = u1;
          }
        }
        tc_fence_before();
        mbar_arrive(bar_d2empty + 8 * b);
        __syncwarp();
        // the warp's 32 rows x 128 bytes.  A warp whose 32 rows all hold tokens stores them four
        // at a time with TMA tile::scatter4 (lane 0 issues; the map clips columns past d_out);
        // other warps use plain stores, 8 lanes per row segment
        bool used_tma = false;
        if (live) {
          const int q = lane & 7;
          const int col = half * 64 + q * 8;
          const bool tma = P.ytma && __all_sync(0xffffffffu, tok >= 0) && half * 64 < ncols;
          if (tma) {
            fence_proxy_async();                          // the RMW above is visible to the TMA engine
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int t0 = __shfl_sync(0xffffffffu, tok, 4 * it), t1 = __shfl_sync(0xffffffffu, tok, 4 * it + 1);
              const int t2 = __shfl_sync(0xffffffffu, tok, 4 * it + 2), t3 = __shfl_sync(0xffffffffu, tok, 4 * it + 3);
              if (lane == 0)
                tma_scatter4(&P.ymap[p], c0 + half * 64, t0, t1, t2, t3,
                             smem_u32(yhalf + (size_t)(wrow0 + 4 * it) * 128));
            }
            used_tma = true;
          } else {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rr = 4 * it + (lane >> 3);
              const int tk = __shfl_sync(0xffffffffu, tok, rr);
              const int r = wrow0 + rr;
              if (tk >= 0 && col < ncols) {
                const uint4 val = *reinterpret_cast<const uint4*>(yhalf + (size_t)r * 128 + ((q ^ (r & 7)) << 4));
                __stcs(reinterpret_cast<uint4*>(y + (size_t)tk * d_out + c0 + col), val);
              }
            }
          }
        }
        if (used_tma && lane == 0) {
          bulk_commit();
          bulk_wait_read_all();                            // the slot may be refilled once the copies read it
        }
        __syncwarp();
        mbar_arrive(bar_tempty + 8 * slot);
      }
      if (abort) break;
      bool last = item_at(i + 1) >= nitems;
      if (!last) {
        int st2, p2, n02, ntl2, d2;
        item_shape(item_at(i + 1), st2, p2, n02, ntl2, d2);
        last = st2 != st;
      }
      if (last) mbar_arrive(bar_mempty + 8 * (mcnt & 1));    // this tile's tokens are no longer read
    }
    if (lane == 0) bulk_wait_all();                          // every y row written before the CTA ends
  } else if (lane == 0) {
    // ---------------------------------------------------- MMA issue
    const uint32_t id = idesc_bf16(TB_M, TB_NT);
    uint32_t g = 0;
    int vcnt = -1, st_prev = -1, p_prev = -1;
    for (int i = 0; item_at(i) < nitems && !abort; ++i) {
      int st, p, n0, ntl, d_out;
      item_shape(item_at(i), st, p, n0, ntl, d_out);
      if (st != st_prev || p != p_prev) {
        ++vcnt;
        if (!mbar_wait(bar_vfull + 8 * (vcnt & 1), (vcnt >> 1) & 1)) { abort = true; break; }
      }
      st_prev = st;
      p_prev = p;
      const uint32_t vh = sbase + (uint32_t)((vcnt & 1) * L.vbuf), vl = vh + (uint32_t)(TB_M * K2 * 2);
      for (int t = 0; t < ntl; ++t, ++g) {
        const uint32_t slot = g % NY, b = g & 1;
        if (!mbar_wait(bar_tfull + 8 * slot, (g / NY) & 1)) { abort = true; break; }
        if (g >= 2 && !mbar_wait(bar_d2empty + 8 * b, ((g >> 1) - 1) & 1)) { abort = true; break; }
        tc_fence_after();
        const uint32_t bb = sbase + (uint32_t)L.b + slot * (uint32_t)(TB_NT * K2 * 2);
        const uint32_t dcol = tmem + b * 128;
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(vh + kk * 256, 128, SBO), desc_k_plain(bb + kk * 256, 128, SBO), id, kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(vl + kk * 256, 128, SBO), desc_k_plain(bb + kk * 256, 128, SBO), id, 1u);
        mma_commit(bar_d2full + 8 * b);
      }
      if (abort) break;
      bool last = item_at(i + 1) >= nitems;
      if (!last) {
        int st2, p2, n02, ntl2, d2;
        item_shape(item_at(i + 1), st2, p2, n02, ntl2, d2);
        last = st2 != st || p2 != p;
      }
      if (last) mma_commit(bar_vempty + 8 * (vcnt & 1));     // this V is no longer read
    }
  }
  abort = __syncthreads_or(abort);
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- host side

bool sgmm_tensor_supported(const SgmmArgs& a, int dtype) {
  if (sgmm_ragged_supported(a, dtype)) return true;
  if (dtype != APR_BF16) return false;
  if (a.k < 1 || a.k > 2) return false;
  if (a.k * round16i(a.max_rank) > TB_MAXK2) return false;
  if (a.d_in % TB_BK != 0) return false;
  for (int p = 0; p < a.nproj; ++p)
    if (a.proj[p].d_out % 16 != 0) return false;
  return true;
}

// Shrink plan fields shared by both expands: projections per item, pipeline depth, the A
// tensor-map templates (one per projection and rank) and where each CTA writes its maps.
static cudaError_t shrink_plan(TcPlan& t, const SgmmArgs& a, size_t v_off, size_t amaps_off, int vpair) {
  t.a = a;
  t.R16 = round16i(a.max_rank);
  t.amaps_off = amaps_off;
  for (int p = 0; p < a.nproj; ++p)
    for (int r = 8; r <= t.R16; r += 8) {
      const cudaError_t err = cached_box_map(&t.atmpl[p][r / 8 - 1], a.x, r, a.d_in, (long)a.d_in * 2, 64, t.R16, true);
      if (err != cudaSuccess) return err;
    }
  t.pg = TB_MAXN1 / t.R16;
  if (t.pg > a.nproj) t.pg = a.nproj;
  t.npg = (a.nproj + t.pg - 1) / t.pg;
  const int n1max = t.pg * t.R16;
  t.stages = (int)((SMEM_BUDGET - 4096) / (TB_M * 128 + n1max * 128));
  if (t.stages > 8) t.stages = 8;
  t.vprep_off = v_off;
  t.vpair = vpair;
  return cudaSuccess;
}

static cudaError_t launch_shrink(const TcPlan& t, cudaStream_t s) {
  const SgmmArgs& a = t.a;
  const size_t sm1 = sh_smem(t.pg * t.R16, t.stages).total;
  static SmemLimit lim;
  cudaError_t err;
  if ((err = lim.ensure((const void*)tc_shrink_kernel, sm1)) != cudaSuccess) return err;
  const int nsm = device_sm_count();
  // tile counts are bounded by the plan's maxima; the kernel loops over the real ones
  const long max_q = max_qtiles(a.T, a.k, a.E);
  int g1 = (int)(max_q * t.npg < nsm ? max_q * t.npg : nsm);
  if (g1 > kShrinkMaxCtas) g1 = kShrinkMaxCtas;
  return launch_pdl(tc_shrink_kernel, dim3(g1), dim3(SH_BLOCK), sm1, s, t);
}

cudaError_t launch_tc_shrink_pairs(const SgmmArgs& a, size_t v_off, cudaStream_t s) {
  std::unique_ptr<TcPlan> t(new TcPlan);
  memset(t.get(), 0, sizeof(TcPlan));
  cudaError_t err;
  if ((err = shrink_plan(*t, a, v_off, v_off + bank_vc_bytes(a.T, a.k, a.max_rank), 1)) != cudaSuccess) return err;
  return launch_shrink(*t, s);
}

cudaError_t launch_sgmm_tensor(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  std::unique_ptr<TcPlan> tp(new TcPlan);
  TcPlan& t = *tp;
  memset(&t, 0, sizeof(t));
  cudaError_t err;
  if ((err = shrink_plan(t, a, scratch_off, scratch_off + tc_vc_bytes(a.T, a.k, a.max_rank), 0)) != cudaSuccess)
    return err;
  t.mixed = (a.k <= 2 && kMixAdapters * t.R16 <= TB_MAXK2) ? 1 : 0;
  t.K2 = (t.mixed ? kMixAdapters : a.k) * t.R16;
  t.ny = t.K2 <= 32 ? 4 : 3;
  t.ytma = 1;
  for (int p = 0; p < a.nproj && t.ytma; ++p)
    t.ytma = encode_row_map(&t.ymap[p], a.proj[p].y, a.T, a.proj[p].d_out) == cudaSuccess;
  t.cc_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) t.cc_before[p + 1] = t.cc_before[p] + (a.proj[p].d_out + TB_CW - 1) / TB_CW;

  // the set and mixed tiles of the plan, on the first gathered call after it
  if ((err = launch_gather_plan(a.idx, a.T, a.k, a.E, a.ws, s)) != cudaSuccess) return err;
  const size_t sm2 = ex_smem(t.K2, t.ny).total;
  static SmemLimit lim2;
  if ((err = lim2.ensure((const void*)tc_expand_kernel, sm2)) != cudaSuccess) return err;
  const int nsm = device_sm_count();
  const long max_s = (long)a.T + (a.T + TB_M - 1) / TB_M;
  const int g2 = (int)(max_s * t.cc_before[a.nproj] < nsm ? max_s * t.cc_before[a.nproj] : nsm);
  if ((err = launch_shrink(t, s)) != cudaSuccess) return err;
  return launch_pdl(tc_expand_kernel, dim3(g2), dim3(EX_BLOCK), sm2, s, t);
}

}  // namespace apr
