// SGMM on the 5th-generation tensor cores (tcgen05) for long segments
// (prefill, many tenants).  AdaFuse summary (gist.science), Resumen tecnico
// §2.B: the segmented gather product applies the selected low-rank adapters to
// the tokens gathered per adapter in one batched product, fused into the add
// onto the base projection output.
//
// The routing plan orders the tokens by their adapter set; a set tile is a run
// of <= 128 tokens sharing the same k <= 2 adapters {e0 < e1}.  Two persistent
// kernels, one CTA per SM:
//
//  shrink  item = one set tile and a group of projections (all of them when
//          nproj * k * R16 <= 256; R16 = max rank rounded up to 16).
//          D1[128 x N1] = X_tile . [A_{q,e0} ; A_{q,e1} ...]^T on tcgen05
//          (kind::f16, bf16 in, fp32 in TMEM): x rows are gathered once per
//          tile, 64 columns per stage, with 16-byte cp.async into 128B-swizzled
//          K-major stages, A rows likewise; the copies complete on the stage's
//          mbarrier, one thread of the MMA warp issues the MMAs and commits
//          them to the stage's "empty" barrier.  The epilogue reads D1 back
//          (one TMEM lane per token), scales by the token's gates and stores
//          v as bf16 hi + lo halves (~16 mantissa bits) in the token's row of
//          the plan order: V[q][pos][hi: k*R16 | lo: k*R16].
//  expand  item = (set tile, projection, 1024 output columns), 128-column
//          tiles: D2[128 x 128] = V_hi . Bcat^T + V_lo . Bcat^T with
//          Bcat[n] = [B_e0[n] | B_e1[n]], TMEM double buffered.  Eight warps
//          gather the tile's y_base rows and Bcat with cp.async into a 4-deep
//          ring (three tiles ahead, across item boundaries), then run the
//          epilogue: y = y_base + D2 for their row and half, rounded once to
//          bf16, written back through shared memory so each warp stores whole
//          128-byte row segments.
//
// Every mbarrier wait is bounded by the global timer (1 s); on expiry the CTA
// records APR_ERR_TIMEOUT, drains its copies and frees its TMEM.
#include "apr_internal.cuh"
#include "tc_ptx.cuh"

namespace apr {

constexpr int TB_M = 128;          // tokens per set tile (= kSetTile)
constexpr int TB_BK = 64;          // input columns per shrink stage
constexpr int TB_MAXN1 = 256;      // shrink accumulator columns
constexpr int TB_MAXK2 = 64;       // k * R16 handled by the expand
constexpr int TB_NT = 128;         // output columns per expand tile
constexpr int TB_CW = 1024;        // output columns per expand item
constexpr int SH_WORKERS = 128;    // shrink: warps 0-3 load and run the epilogue, warp 4 issues MMAs
constexpr int SH_BLOCK = SH_WORKERS + 32;
constexpr int EX_WORKERS = 256;    // expand: warps 0-7 load and run the epilogue, warp 8 issues MMAs
constexpr int EX_BLOCK = EX_WORKERS + 32;
constexpr int SMEM_BUDGET = 200 * 1024;

struct TileInfo {        // a set tile and its adapters, written by the shrink for the expand
  int start, len, e0, e1;
};

struct TcPlan {
  SgmmArgs a;
  int R16;                           // rank slot per adapter
  int K2;                            // k * R16
  int pg;                            // projections per shrink item
  int npg;                           // shrink items per set tile
  int stages;                        // shrink pipeline depth
  int ny;                            // expand ring depth
  size_t vprep_off;                  // scratch: V rows [proj][pos][2 * K2] bf16
  size_t tinfo_off;                  // scratch: TileInfo [set tiles]
  int cc_before[APR_MAX_PROJ + 1];   // expand: prefix of 1024-column items per projection
};

static_assert(sizeof(TileInfo) == 16 && TB_MAXK2 == kTensorMaxK2, "tensor scratch sizing");

// ---------------------------------------------------------------- shrink

struct ShSmem {
  int stage_bytes, stages;
  size_t bar, meta, total;
};
__host__ __device__ inline ShSmem sh_smem(int n1max, int stages) {
  ShSmem L;
  L.stage_bytes = TB_M * 128 + n1max * 128;
  L.stages = stages;
  L.bar = (size_t)stages * L.stage_bytes;
  L.meta = L.bar + (size_t)(2 * stages + 1) * 8;
  L.total = L.meta + 3 * TB_M * 4 + 16 + TB_MAXN1 * 8 + 1024;
  return L;
}

__global__ void __launch_bounds__(SH_BLOCK, 1) tc_shrink_kernel(const __grid_constant__ TcPlan P) {
  const SgmmArgs& a = P.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool worker = tid < SH_WORKERS;
  const int K = a.k, R16 = P.R16, K2 = P.K2, S = P.stages;
  const ShSmem L = sh_smem(P.pg * K2, S);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  const uint32_t bar_full = smem_u32(bars), bar_empty = smem_u32(bars + S), bar_d1 = smem_u32(bars + 2 * S);
  int* s_tok = reinterpret_cast<int*>(smem + L.meta);
  float* s_g0 = reinterpret_cast<float*>(s_tok + TB_M);
  float* s_g1 = s_g0 + TB_M;
  volatile int* s_flags = reinterpret_cast<volatile int*>(s_g1 + TB_M);     // [0] tmem [1] e0 [2] e1 [3] bad
  const __nv_bfloat16** s_arow = reinterpret_cast<const __nv_bfloat16**>(smem + L.meta + 3 * TB_M * 4 + 16);
  const uint32_t sbase = smem_u32(smem);

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(bar_full + 8 * i, SH_WORKERS);
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
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const int* tok_order = ws_at<int>(a.ws, W.tok_order);
  const SetTile* stiles = ws_at<SetTile>(a.ws, W.stiles);
  TileInfo* tinfo = ws_at<TileInfo>(a.ws, P.tinfo_off);
  __nv_bfloat16* vprep = ws_at<__nv_bfloat16>(a.ws, P.vprep_off);
  const int nst = hdr->n_stiles;
  const long nitems = (long)nst * P.npg;
  const __nv_bfloat16* __restrict__ x = reinterpret_cast<const __nv_bfloat16*>(a.x);
  const int d_in = a.d_in, nk = d_in / TB_BK;
  uint32_t gchunk = 0, nitem = 0;
  bool abort = false;

  for (long item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int st = (int)(item / P.npg), q0 = (int)(item % P.npg) * P.pg;
    const int nq = min(P.pg, a.nproj - q0);
    const int N1 = nq * K2;
    const SetTile tile = stiles[st];
    if (worker) {
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
        s_flags[1] = e0;
        s_flags[2] = e1;
        bool bad = tile.len > 0 && (e0 < 0 || e0 >= a.E || (K == 2 && (e1 < 0 || e1 >= a.E)));
        if (!bad && tile.len > 0) {
          const int r0 = a.ranks[e0], r1 = K == 2 ? a.ranks[e1] : 8;
          bad = r0 < 8 || r0 > R16 || (r0 & 7) || r1 < 8 || r1 > R16 || (r1 & 7);
        }
        s_flags[3] = bad ? 1 : 0;
        if (bad) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e0);
        if (q0 == 0) tinfo[st] = TileInfo{tile.start, bad ? 0 : tile.len, e0, e1};
      }
    }
    __syncthreads();
    if (s_flags[3] || tile.len <= 0 || abort) {
      __syncthreads();
      continue;
    }
    const int e0 = s_flags[1], e1 = s_flags[2];
    // source row of every A row of the item (null: a zero row)
    if (worker) {
      for (int j = tid; j < N1; j += SH_WORKERS) {
        const int qi = j / K2, rem = j - qi * K2, slot = rem / R16, rr = rem - slot * R16;
        const int e = slot == 0 ? e0 : e1;
        const int re = a.ranks[e];
        s_arow[j] = rr < re ? reinterpret_cast<const __nv_bfloat16*>(a.proj[q0 + qi].A[e]) + (size_t)rr * d_in : nullptr;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(SH_WORKERS) : "memory");
    }
    const uint32_t g0 = gchunk;
    if (worker) {
      for (int c = 0; c < nk && !abort; ++c) {
        const uint32_t g = g0 + c, s = g % S;
        if (g >= (uint32_t)S && !mbar_wait(bar_empty + 8 * s, ((g / S) - 1) & 1)) { abort = true; break; }
        const uint32_t st_base = sbase + s * L.stage_bytes;
#pragma unroll
        for (int m = 0; m < 8; ++m) {          // x rows: 8 lanes per 128-byte row segment
          const int w = tid + m * SH_WORKERS;
          const int row = w >> 3, q = w & 7;
          const int tk = s_tok[row];
          if (tk >= 0)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(st_base + (uint32_t)row * 128 +
                                                                            (uint32_t)((q ^ (row & 7)) << 4)),
                         "l"(x + (size_t)tk * d_in + (size_t)c * TB_BK + q * 8)
                         : "memory");
        }
        const uint32_t abase = st_base + TB_M * 128;
        for (int w = tid; w < N1 * 8; w += SH_WORKERS) {
          const int j = w >> 3, q = w & 7;
          const __nv_bfloat16* src = s_arow[j];
          cp_async16_zfill(abase + (uint32_t)j * 128 + (uint32_t)((q ^ (j & 7)) << 4),
                           src ? (const void*)(src + (size_t)c * TB_BK + q * 8) : (const void*)x, src != nullptr);
        }
        cp_async_arrive(bar_full + 8 * s);
      }
      // gates -> V rows (bf16 hi | lo) in plan order
      if (!abort && !mbar_wait(bar_d1, nitem & 1)) abort = true;
      tc_fence_after();
      if (!abort) {
        const int row = tid;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const bool valid = row < tile.len;
        const float ga = s_g0[row], gb = s_g1[row];
        for (int c0 = 0; c0 < N1; c0 += 16) {
          float v[16];
          tmem_ld16(lane_addr + (uint32_t)c0, v);
          const int qi = c0 / K2, rem = c0 - qi * K2;
          const float gg = rem < R16 ? ga : gb;
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a0 = v[2 * i] * gg, a1 = v[2 * i + 1] * gg;
            const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            const float2 hf = __bfloat1622float2(h);
            hi[i] = *reinterpret_cast<const uint32_t*>(&h);
            lo[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(vprep + ((size_t)(q0 + qi) * a.T + tile.start + row) * (2 * K2) + rem);
            dst[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            dst[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            uint4* dlo = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + K2);
            dlo[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            dlo[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
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
    tc_fence_before();
    abort = __syncthreads_or(abort);
    tc_fence_after();
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
  size_t vbuf, y, b, bar, total;
};
__host__ __device__ inline ExSmem ex_smem(int K2, int ny) {
  ExSmem L;
  L.K2 = K2;
  L.ny = ny;
  L.vbuf = (size_t)2 * TB_M * K2 * 2;                 // one V buffer: hi then lo
  L.y = 2 * L.vbuf;                                   // ring of y tiles [128 rows][256 B]
  L.b = L.y + (size_t)ny * TB_M * 256;                // ring of Bcat tiles [128][K2] bf16
  L.bar = L.b + (size_t)ny * TB_NT * K2 * 2;
  L.total = L.bar + (size_t)(2 * ny + 8) * 8 + 16 + 1024;
  return L;
}

struct ExItem {
  int start, len, p, n0, ntl, d_out, tok;
  const __nv_bfloat16* B0;
  const __nv_bfloat16* B1;
  int r0, r1;
};

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
  const uint32_t bar_vfull = smem_u32(bars + NY);             // [2]  V of an item landed
  const uint32_t bar_vempty = smem_u32(bars + NY + 2);        // [2]  V of an item consumed by the MMAs
  const uint32_t bar_d2full = smem_u32(bars + NY + 4);        // [2]  accumulator ready
  const uint32_t bar_d2empty = smem_u32(bars + NY + 6);       // [2]  accumulator read
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(bars + 2 * NY + 8);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t SBO = (uint32_t)(K2 / 8) * 128;              // next 8-row group of a K-major operand

  if (tid == 0) {
    for (int i = 0; i < NY; ++i) mbar_init(bar_tfull + 8 * i, EX_WORKERS);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_vfull + 8 * i, EX_WORKERS);
      mbar_init(bar_vempty + 8 * i, 1);
      mbar_init(bar_d2full + 8 * i, 1);
      mbar_init(bar_d2empty + 8 * i, EX_WORKERS);
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
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const int* tok_order = ws_at<int>(a.ws, W.tok_order);
  const TileInfo* tinfo = ws_at<TileInfo>(a.ws, P.tinfo_off);
  const __nv_bfloat16* vprep = ws_at<__nv_bfloat16>(a.ws, P.vprep_off);
  const int ipt = P.cc_before[a.nproj];
  const long nitems = (long)hdr->n_stiles * ipt;
  auto item_at = [&](int i) -> long { return (long)blockIdx.x + (long)i * gridDim.x; };
  // item -> (set tile, projection, first column, tiles)
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

  if (tid < EX_WORKERS) {
    const int row = tid & (TB_M - 1), half = tid >> 7;
    auto load_item = [&](int i, ExItem& I) {
      int st;
      item_shape(item_at(i), st, I.p, I.n0, I.ntl, I.d_out);
      const TileInfo ti = tinfo[st];
      I.start = ti.start;
      I.len = ti.len;
      I.tok = row < ti.len ? tok_order[ti.start + row] : -1;
      I.B0 = I.B1 = nullptr;
      I.r0 = I.r1 = 0;
      if (ti.len > 0) {
        I.B0 = reinterpret_cast<const __nv_bfloat16*>(a.proj[I.p].B[ti.e0]);
        I.r0 = a.ranks[ti.e0];
        if (K == 2) {
          I.B1 = reinterpret_cast<const __nv_bfloat16*>(a.proj[I.p].B[ti.e1]);
          I.r1 = a.ranks[ti.e1];
        }
      }
    };
    // V rows of item i (this thread: row `row`, half hi/lo) into V buffer i & 1
    auto issue_v = [&](int i, const ExItem& I) {
      const uint32_t buf = sbase + (uint32_t)((i & 1) * L.vbuf) + (uint32_t)half * (TB_M * K2 * 2);
      const bool valid = row < I.len;
      const __nv_bfloat16* src = vprep + ((size_t)I.p * a.T + I.start + row) * (2 * K2) + half * K2;
      for (int q = 0; q < K2 / 8; ++q)
        cp_async16_zfill(buf + (uint32_t)(row >> 3) * SBO + (uint32_t)q * 128 + (uint32_t)(row & 7) * 16,
                         valid ? (const void*)(src + q * 8) : (const void*)vprep, valid);
      cp_async_arrive(bar_vfull + 8 * (i & 1));
    };
    // y_base rows and Bcat of tile t of item I into ring slot `slot`
    auto issue_tile = [&](const ExItem& I, int t, uint32_t slot) {
      const int n0 = I.n0 + t * TB_NT;
      const uint32_t ybuf = sbase + (uint32_t)L.y + slot * (TB_M * 256);
      if (I.tok >= 0) {
        const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.proj[I.p].y_base) +
                                   (size_t)I.tok * I.d_out + n0 + half * 64;
        const uint32_t dst = ybuf + (uint32_t)row * 256 + (uint32_t)half * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const bool ok = n0 + half * 64 + q * 8 < I.d_out;
          cp_async16_zfill(dst + (uint32_t)((q ^ (row & 7)) << 4), ok ? (const void*)(src + q * 8) : (const void*)src, ok);
        }
      }
      const uint32_t bbuf = sbase + (uint32_t)L.b + slot * (uint32_t)(TB_NT * K2 * 2);
      const int cpr = K2 / 8, cps = R16 / 8;
      for (int w = tid; w < TB_NT * cpr; w += EX_WORKERS) {
        const int n = w / cpr, kq = w - n * cpr;
        const int slot_a = kq / cps, cq = kq - slot_a * cps;
        const __nv_bfloat16* B = slot_a == 0 ? I.B0 : I.B1;
        const int re = slot_a == 0 ? I.r0 : I.r1;
        const bool ok = B != nullptr && n0 + n < I.d_out && cq * 8 < re;
        cp_async16_zfill(bbuf + (uint32_t)(n >> 3) * SBO + (uint32_t)kq * 128 + (uint32_t)(n & 7) * 16,
                         ok ? (const void*)(B + (size_t)(n0 + n) * re + cq * 8) : (const void*)vprep, ok);
      }
      cp_async_arrive(bar_tfull + 8 * slot);
    };

    ExItem prod, cons;
    int prod_i = 0, prod_t = 0, cons_i = 0, cons_t = 0;
    uint32_t gp = 0, gc = 0;
    bool prod_live = item_at(0) < nitems;
    if (prod_live) {
      load_item(0, prod);
      issue_v(0, prod);
    }
    cons = prod;
    while (!abort) {
      // ------------------------------------------------ producer: up to NY - 1 tiles ahead
      while (prod_live && gp < gc + (uint32_t)(NY - 1)) {
        if (prod_t == prod.ntl) {
          if (prod_i + 1 > cons_i + 1) break;                 // at most one item ahead of the epilogue
          if (item_at(prod_i + 1) >= nitems) { prod_live = false; break; }
          ++prod_i;
          prod_t = 0;
          load_item(prod_i, prod);
          if (prod_i == cons_i) cons = prod;
          if (prod_i >= 2 && !mbar_wait(bar_vempty + 8 * (prod_i & 1), ((prod_i >> 1) - 1) & 1)) { abort = true; break; }
          issue_v(prod_i, prod);
        }
        issue_tile(prod, prod_t, gp % NY);
        ++gp;
        ++prod_t;
      }
      if (abort || gc == gp) break;
      // ------------------------------------------------ epilogue of tile gc
      const uint32_t slot = gc % NY, b = gc & 1;
      if (!mbar_wait(bar_tfull + 8 * slot, (gc / NY) & 1)) { abort = true; break; }
      if (!mbar_wait(bar_d2full + 8 * b, (gc >> 1) & 1)) { abort = true; break; }
      tc_fence_after();
      const int n0 = cons.n0 + cons_t * TB_NT;
      const int ncols = min(TB_NT, cons.d_out - n0);
      unsigned char* yrow = smem + L.y + (size_t)slot * (TB_M * 256) + (size_t)row * 256 + half * 128;
      const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + b * 128 + (uint32_t)half * 64;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float v[16];
        tmem_ld16(taddr + (uint32_t)(c16 * 16), v);
        if (cons.tok >= 0) {
          uint4* p0 = reinterpret_cast<uint4*>(yrow + (((2 * c16) ^ (row & 7)) << 4));
          uint4* p1 = reinterpret_cast<uint4*>(yrow + (((2 * c16 + 1) ^ (row & 7)) << 4));
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
      mbar_arrive(bar_d2empty + 8 * b);
      __syncwarp();
      // the warp's 32 rows x 128 bytes: 8 lanes per row segment
      {
        __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.proj[cons.p].y);
        const int wrow0 = (warp & 3) * 32;
        const int q = lane & 7;
        const int col = half * 64 + q * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3);
          const int tk = __shfl_sync(0xffffffffu, cons.tok, rr);
          const int r = wrow0 + rr;
          if (tk >= 0 && col < ncols) {
            const uint4 val = *reinterpret_cast<const uint4*>(smem + L.y + (size_t)slot * (TB_M * 256) + (size_t)r * 256 +
                                                              half * 128 + ((q ^ (r & 7)) << 4));
            __stcs(reinterpret_cast<uint4*>(y + (size_t)tk * cons.d_out + n0 + col), val);
          }
        }
      }
      __syncwarp();
      ++gc;
      if (++cons_t == cons.ntl) {
        ++cons_i;
        cons_t = 0;
        if (prod_i == cons_i) cons = prod;
      }
    }
  } else if (lane == 0) {
    // ---------------------------------------------------- MMA issue
    const uint32_t id = idesc_bf16(TB_M, TB_NT);
    uint32_t g = 0;
    for (int i = 0; item_at(i) < nitems && !abort; ++i) {
      int st, p, n0, ntl, d_out;
      item_shape(item_at(i), st, p, n0, ntl, d_out);
      if (!mbar_wait(bar_vfull + 8 * (i & 1), (i >> 1) & 1)) { abort = true; break; }
      const uint32_t vh = sbase + (uint32_t)((i & 1) * L.vbuf), vl = vh + (uint32_t)(TB_M * K2 * 2);
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
      if (!abort) mma_commit(bar_vempty + 8 * (i & 1));
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
  if (dtype != APR_BF16) return false;
  if (a.k < 1 || a.k > 2) return false;
  if (a.k * round16i(a.max_rank) > TB_MAXK2) return false;
  if (a.d_in % TB_BK != 0) return false;
  for (int p = 0; p < a.nproj; ++p)
    if (a.proj[p].d_out % 16 != 0) return false;
  return true;
}

cudaError_t launch_sgmm_tensor(const SgmmArgs& a, size_t scratch_off, cudaStream_t s) {
  TcPlan t;
  memset(&t, 0, sizeof(t));
  t.a = a;
  t.R16 = round16i(a.max_rank);
  t.K2 = a.k * t.R16;
  t.pg = TB_MAXN1 / t.K2;
  if (t.pg > a.nproj) t.pg = a.nproj;
  t.npg = (a.nproj + t.pg - 1) / t.pg;
  const int n1max = t.pg * t.K2;
  t.stages = (int)((SMEM_BUDGET - 4096) / (TB_M * 128 + n1max * 128));
  if (t.stages > 8) t.stages = 8;
  t.ny = t.K2 <= 32 ? 4 : 3;
  t.vprep_off = scratch_off;
  t.tinfo_off = scratch_off + align_up(tc_vprep_bytes(a.T, t.K2));   // layout as in tc_scratch_bytes
  t.cc_before[0] = 0;
  for (int p = 0; p < a.nproj; ++p) t.cc_before[p + 1] = t.cc_before[p] + (a.proj[p].d_out + TB_CW - 1) / TB_CW;

  const size_t sm1 = sh_smem(n1max, t.stages).total, sm2 = ex_smem(t.K2, t.ny).total;
  static size_t conf1 = 0, conf2 = 0;
  cudaError_t err;
  if (sm1 > conf1) {
    if ((err = cudaFuncSetAttribute(tc_shrink_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1)) != cudaSuccess)
      return err;
    conf1 = sm1;
  }
  if (sm2 > conf2) {
    if ((err = cudaFuncSetAttribute(tc_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2)) != cudaSuccess)
      return err;
    conf2 = sm2;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // set tiles <= T + ceil(T / 128): the kernels loop over the real count
  const long max_tiles = (long)a.T + (a.T + TB_M - 1) / TB_M;
  const int g1 = (int)(max_tiles * t.npg < nsm ? max_tiles * t.npg : nsm);
  const int g2 = (int)(max_tiles * t.cc_before[a.nproj] < nsm ? max_tiles * t.cc_before[a.nproj] : nsm);
  if ((err = launch_pdl(tc_shrink_kernel, dim3(g1), dim3(SH_BLOCK), sm1, s, t)) != cudaSuccess) return err;
  return launch_pdl(tc_expand_kernel, dim3(g2), dim3(EX_BLOCK), sm2, s, t);
}

}  // namespace apr
