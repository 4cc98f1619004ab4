// SGMM on the 5th-generation tensor cores (tcgen05) for long segments
// (prefill).  AdaFuse summary (gist.science), Resumen tecnico §2.B: the
// segmented gather product applies the selected low-rank adapters to the
// tokens gathered per adapter in one batched product, fused into the add onto
// the base projection output, with prefetching and tiling.
//
// The routing plan orders tokens by their adapter set; a work item is one
// set tile (<= 128 tokens that share the same k <= 2 adapters {e0, e1}) and
// one projection.  Per item, in one CTA of 128 threads (1 CTA per SM, TMEM
// fully owned):
//
//  shrink  D1[128 x N1] = X_tile[128 x d_in] . [A_e0 ; A_e1]^T on tcgen05
//          (kind::f16, bf16 in, fp32 accumulate in TMEM), N1 = k * R16 where
//          R16 is the rank rounded up to 16 (zero rows pad the smaller ranks).
//          The gathered x rows and the A rows are staged with 16-byte cp.async
//          into 128B-swizzled K-major tiles, 3 stages in flight, one elected
//          thread issues the MMAs and commits each stage to an mbarrier.
//  gate    D1 is read back with tcgen05.ld (one TMEM lane per token), scaled
//          by the token's gates and split into bf16 hi + lo parts (so the
//          expand keeps ~16 mantissa bits of v), written to shared memory as
//          the K-major A operand of the expand.
//  expand  for every 128-column tile of d_out: D2[128 x 128] = V_hi.Bcat^T +
//          V_lo.Bcat^T with Bcat[n] = [B_e0[n] | B_e1[n]] (K2 = N1), TMEM
//          double buffered.  The epilogue adds y_base (fetched with bulk
//          async copies one tile ahead, completion on an mbarrier), rounds to
//          bf16 once and writes each token row back with a bulk async store.
//
// Every mbarrier wait is bounded by the global timer (1 s); on expiry the CTA
// records APR_ERR_TIMEOUT, drains its own bulk copies and frees its TMEM.
#include "apr_internal.cuh"

namespace apr {

constexpr int TC_THREADS = 128;
constexpr int TC_BM = 128;       // tokens per tile (= kSetTile)
constexpr int TC_BK = 64;        // input columns per stage (one 128-byte swizzle row)
constexpr int TC_STAGES = 3;
constexpr int TC_MAXN1 = 64;     // k * R16
constexpr int TC_NT = 128;       // output columns per expand tile
constexpr int TC_YSTRIDE = TC_NT * 2 + 16;   // bytes per staged y row (padding against bank conflicts)
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr uint32_t TC_D2_COL = 128;           // D2 buffers at columns 128 and 256

struct TcSmem {
  static constexpr size_t X = 0;                                              // 3 x 16 KB
  static constexpr size_t A = X + (size_t)TC_STAGES * TC_BM * 128;            // 3 x 8 KB
  static constexpr size_t VH = A + (size_t)TC_STAGES * TC_MAXN1 * 128;        // 16 KB
  static constexpr size_t VL = VH + (size_t)TC_BM * TC_MAXN1 * 2;             // 16 KB
  static constexpr size_t BB = VL + (size_t)TC_BM * TC_MAXN1 * 2;             // 2 x 16 KB
  static constexpr size_t Y = BB + 2 * (size_t)TC_NT * TC_MAXN1 * 2;          // 2 x 34 KB
  static constexpr size_t BAR = Y + 2 * (size_t)TC_BM * TC_YSTRIDE;           // mbarriers
  static constexpr size_t META = BAR + 16 * 8;
  static constexpr size_t TOTAL = META + 3 * TC_BM * 4 + 64;
  static constexpr size_t ALLOC = TOTAL + 1024;                               // for 1024-byte alignment
};
static_assert(TcSmem::ALLOC <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after about one second of global time.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (globaltimer() - t0 > 1000000000ull) return false;
    __nanosleep(32);
  }
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptors (tcgen05 format, version 1).
// K-major, 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                 // leading offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;       // stride offset: next 8-row group
  d |= (uint64_t)1u << 46;                 // descriptor version
  d |= (uint64_t)2u << 61;                 // SWIZZLE_128B
  return d;
}
// K-major, no swizzle: 8x16-byte core matrices; `lbo` to the next one along K,
// `sbo` to the next 8-row group.
__device__ __forceinline__ uint64_t desc_k_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- the kernel

struct TcArgs {
  SgmmArgs a;
  int R16;     // rank slot per adapter (multiple of 16)
  int N1;      // k * R16
};

__global__ void __launch_bounds__(TC_THREADS, 1) sgmm_tc_kernel(TcArgs args) {
  const SgmmArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int K = a.k, R16 = args.R16, N1 = args.N1, K2 = N1;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TcSmem::BAR);
  // barriers: [0..2] stage MMA done, [3..4] expand MMA done, [5..6] y_base arrived
  const uint32_t bar_stage = smem_u32(bars);
  const uint32_t bar_mma2 = smem_u32(bars + 3);
  const uint32_t bar_y = smem_u32(bars + 5);
  int* s_tok = reinterpret_cast<int*>(smem + TcSmem::META);
  float* s_g0 = reinterpret_cast<float*>(s_tok + TC_BM);
  float* s_g1 = s_g0 + TC_BM;
  volatile int* s_flags = reinterpret_cast<volatile int*>(s_g1 + TC_BM);   // [0] tmem base, [1] abort, [2..3] set
  const uint32_t sX = smem_u32(smem + TcSmem::X);
  const uint32_t sA = smem_u32(smem + TcSmem::A);
  const uint32_t sVH = smem_u32(smem + TcSmem::VH);
  const uint32_t sVL = smem_u32(smem + TcSmem::VL);
  const uint32_t sB = smem_u32(smem + TcSmem::BB);
  unsigned char* sYp = smem + TcSmem::Y;
  const uint32_t sY = smem_u32(sYp);

  if (tid == 0) {
    for (int i = 0; i < TC_STAGES; ++i) mbar_init(bar_stage + 8 * i, 1);
    for (int i = 0; i < 2; ++i) mbar_init(bar_mma2 + 8 * i, 1);
    for (int i = 0; i < 2; ++i) mbar_init(bar_y + 8 * i, TC_THREADS);
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

  const WsLayout L = ws_layout(a.T, a.k, a.E);
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const int* tok_order = ws_at<int>(a.ws, L.tok_order);
  const SetTile* stiles = ws_at<SetTile>(a.ws, L.stiles);
  const int nst = hdr->n_stiles;
  const long nitems = (long)nst * a.nproj;
  const __nv_bfloat16* __restrict__ x = reinterpret_cast<const __nv_bfloat16*>(a.x);
  const int d_in = a.d_in;
  const int nk = d_in / TC_BK;
  const uint32_t id1 = idesc_bf16(TC_BM, N1);
  const uint32_t id2 = idesc_bf16(TC_BM, TC_NT);
  const uint32_t sbo_v = (uint32_t)(K2 / 8) * 128;   // V and Bcat: next 8-row group
  uint32_t ph_stage = 0;                              // bit s: parity of stage barrier s
  uint32_t ph_mma2 = 0, ph_y = 0;
  bool abort = false;

  for (long item = blockIdx.x; item < nitems && !abort; item += gridDim.x) {
    const int st = (int)(item / a.nproj);
    const int p = (int)(item % a.nproj);
    const SetTile tile = stiles[st];
    const int len = tile.len;
    const int d_out = a.proj[p].d_out;
    // tokens, their adapter set (sorted) and gates in that order
    {
      int tok = -1, e0 = 0, e1 = 0;
      float g0 = 0.f, g1 = 0.f;
      if (tid < len) {
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
      }
    }
    __syncthreads();
    const int e0 = s_flags[2], e1 = s_flags[3];
    int rk[2] = {0, 0};
    bool bad = (e0 < 0 || e0 >= a.E || (K == 2 && (e1 < 0 || e1 >= a.E)));
    if (!bad) {
      rk[0] = a.ranks[e0];
      rk[1] = K == 2 ? a.ranks[e1] : 0;
      if (rk[0] <= 0 || rk[0] > R16 || (rk[0] & 7) || (K == 2 && (rk[1] <= 0 || rk[1] > R16 || (rk[1] & 7))))
        bad = true;
    }
    if (bad) {
      if (tid == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_TC, e0);
      __syncthreads();
      continue;
    }
    const __nv_bfloat16* Aj[2];
    Aj[0] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].A[e0]);
    Aj[1] = K == 2 ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].A[e1]) : Aj[0];
    const int my_tok = s_tok[tid];

    // ------------------------------------------------------------ shrink
    for (int c = 0; c < nk + TC_STAGES - 1 && !abort; ++c) {
      if (c < nk && !abort) {
        const int s = c % TC_STAGES;
        if (c >= TC_STAGES) {
          if (!mbar_wait(bar_stage + 8 * s, (ph_stage >> s) & 1)) abort = true;
          ph_stage ^= 1u << s;
        }
        // x row of this thread's token: 8 x 16 bytes into the swizzled row
        const uint32_t xrow = sX + (uint32_t)s * TC_BM * 128 + (uint32_t)tid * 128;
        if (my_tok >= 0) {
          const __nv_bfloat16* src = x + (size_t)my_tok * d_in + (size_t)c * TC_BK;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(xrow + ((q ^ (tid & 7)) << 4)),
                         "l"(src + q * 8)
                         : "memory");
          }
        }
        // A rows: row j of [A_e0 ; A_e1] (rank slots of R16 rows, zero padded)
        const uint32_t abase = sA + (uint32_t)s * TC_MAXN1 * 128;
        for (int w = tid; w < N1 * 8; w += TC_THREADS) {
          const int j = w >> 3, q = w & 7;
          const int slot = j / R16, r = j % R16;
          const uint32_t dst = abase + (uint32_t)j * 128 + ((q ^ (j & 7)) << 4);
          if (r < rk[slot]) {
            const __nv_bfloat16* src = Aj[slot] + (size_t)r * d_in + (size_t)c * TC_BK + q * 8;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
          } else {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0) : "memory");
          }
        }
      }
      cp_async_commit();
      const int m = c - (TC_STAGES - 1);
      if (m >= 0) {
        cp_async_wait<TC_STAGES - 1>();
        fence_proxy_async();
        abort = __syncthreads_or(abort);
        if (abort) break;
        if (tid == 0) {
          tc_fence_after();
          const int s = m % TC_STAGES;
          const uint32_t xs = sX + (uint32_t)s * TC_BM * 128;
          const uint32_t as = sA + (uint32_t)s * TC_MAXN1 * 128;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)
            mma_bf16(tmem, desc_k_sw128(xs + kk * 32), desc_k_sw128(as + kk * 32), id1, (m > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_stage + 8 * s);
        }
      }
    }
    // every stage with an outstanding commit: wait (keeps parities in step)
    for (int s = 0; s < TC_STAGES && s < nk; ++s) {
      if (!abort && !mbar_wait(bar_stage + 8 * s, (ph_stage >> s) & 1)) abort = true;
      ph_stage ^= 1u << s;
    }
    abort = __syncthreads_or(abort);
    tc_fence_after();
    if (abort) break;

    // ------------------------------------------------------------ gates -> V (bf16 hi + lo)
    {
      const int row = tid;                       // TMEM lane = token row
      const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
      const float ga = s_g0[row], gb = s_g1[row];
      for (int c0 = 0; c0 < N1; c0 += 16) {
        float v[16];
        tmem_ld16(lane_addr + (uint32_t)c0, v);
        const float g = (c0 / R16) == 0 ? ga : gb;
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a0 = v[2 * i] * g, a1 = v[2 * i + 1] * g;
          const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
          const float2 hf = __bfloat1622float2(h);
          hi[i] = *reinterpret_cast<const uint32_t*>(&h);
          lo[i] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
        }
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const int kc8 = (c0 >> 3) + h8;          // core matrix index along K
          const uint32_t off = (uint32_t)(row >> 3) * sbo_v + (uint32_t)kc8 * 128 + (uint32_t)(row & 7) * 16;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sVH + off), "r"(hi[4 * h8]),
                       "r"(hi[4 * h8 + 1]), "r"(hi[4 * h8 + 2]), "r"(hi[4 * h8 + 3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sVL + off), "r"(lo[4 * h8]),
                       "r"(lo[4 * h8 + 1]), "r"(lo[4 * h8 + 2]), "r"(lo[4 * h8 + 3])
                       : "memory");
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------------------------ expand
    const __nv_bfloat16* Bj[2];
    Bj[0] = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e0]);
    Bj[1] = K == 2 ? reinterpret_cast<const __nv_bfloat16*>(a.proj[p].B[e1]) : Bj[0];
    const __nv_bfloat16* __restrict__ yb = reinterpret_cast<const __nv_bfloat16*>(a.proj[p].y_base);
    __nv_bfloat16* __restrict__ y = reinterpret_cast<__nv_bfloat16*>(a.proj[p].y);
    const int nnt = (d_out + TC_NT - 1) / TC_NT;

    auto issue_tile = [&](int nt, int b) {
      const int n0 = nt * TC_NT;
      const int ncols = min(TC_NT, d_out - n0);
      // Bcat rows n0..n0+127: K2 / 8 chunks of 16 bytes per row
      const uint32_t bbase = sB + (uint32_t)b * TC_NT * TC_MAXN1 * 2;
      const int cpr = K2 / 8;
      for (int w = tid; w < TC_NT * cpr; w += TC_THREADS) {
        const int n = w / cpr, q = w % cpr;
        const int slot = q / (R16 / 8), cq = q % (R16 / 8);
        const uint32_t dst = bbase + (uint32_t)(n >> 3) * sbo_v + (uint32_t)q * 128 + (uint32_t)(n & 7) * 16;
        if (n < ncols && cq * 8 < rk[slot]) {
          const __nv_bfloat16* src = Bj[slot] + (size_t)(n0 + n) * rk[slot] + cq * 8;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0) : "memory");
        }
      }
      // y_base row of this thread's token (the previous store from this buffer row must be read out)
      bulk_wait_read_all();
      const uint32_t bytes = my_tok >= 0 ? (uint32_t)ncols * 2 : 0u;
      mbar_arrive_expect_tx(bar_y + 8 * b, bytes);
      if (bytes) bulk_load(sY + (uint32_t)b * TC_BM * TC_YSTRIDE + (uint32_t)tid * TC_YSTRIDE,
                           yb + (size_t)my_tok * d_out + n0, bytes, bar_y + 8 * b);
    };

    issue_tile(0, 0);
    cp_async_commit();
    for (int nt = 0; nt < nnt; ++nt) {
      const int b = nt & 1;
      const int n0 = nt * TC_NT;
      const int ncols = min(TC_NT, d_out - n0);
      if (nt + 1 < nnt) issue_tile(nt + 1, b ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
      fence_proxy_async();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t bb = sB + (uint32_t)b * TC_NT * TC_MAXN1 * 2;
        const uint32_t dcol = tmem + TC_D2_COL + (uint32_t)b * TC_NT;
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(sVH + kk * 256, 128, sbo_v), desc_k_plain(bb + kk * 256, 128, sbo_v), id2,
                   kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < K2 / 16; ++kk)
          mma_bf16(dcol, desc_k_plain(sVL + kk * 256, 128, sbo_v), desc_k_plain(bb + kk * 256, 128, sbo_v), id2, 1u);
        mma_commit(bar_mma2 + 8 * b);
      }
      if (!mbar_wait(bar_mma2 + 8 * b, (ph_mma2 >> b) & 1)) abort = true;
      ph_mma2 ^= 1u << b;
      tc_fence_after();
      if (!mbar_wait(bar_y + 8 * b, (ph_y >> b) & 1)) abort = true;
      ph_y ^= 1u << b;
      abort = __syncthreads_or(abort);
      if (abort) break;
      // epilogue: y = y_base + D2, one rounding, back into the staged row, then a bulk store
      {
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + TC_D2_COL + (uint32_t)b * TC_NT;
        unsigned char* yrow = sYp + (size_t)b * TC_BM * TC_YSTRIDE + (size_t)tid * TC_YSTRIDE;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[16];
          tmem_ld16(lane_addr + (uint32_t)c0, v);
          if (my_tok >= 0) {
            uint4* pr = reinterpret_cast<uint4*>(yrow + c0 * 2);
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
        if (my_tok >= 0) {
          fence_proxy_async();
          bulk_store(y + (size_t)my_tok * d_out + n0,
                     sY + (uint32_t)b * TC_BM * TC_YSTRIDE + (uint32_t)tid * TC_YSTRIDE, (uint32_t)ncols * 2);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncthreads();
    }
    cp_async_wait_all();
    __syncthreads();
  }
  if (abort && tid == 0) report(a.ws, APR_ERR_TIMEOUT, K_TC, (int)blockIdx.x);
  cp_async_wait_all();
  bulk_wait_all();
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

cudaError_t launch_sgmm_tensor(const SgmmArgs& a, cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    cudaError_t err = cudaFuncSetAttribute(sgmm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)TcSmem::ALLOC);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  TcArgs t;
  t.a = a;
  t.R16 = round16(a.max_rank);
  t.N1 = a.k * t.R16;
  // upper bound on items: set tiles <= T (one per token at worst); the kernel loops over the real count
  long max_items = (long)((a.T + TC_BM - 1) / TC_BM + a.T) * a.nproj;
  int grid = nsm;
  if (max_items < grid) grid = (int)max_items;
  return launch_pdl(sgmm_tc_kernel, dim3(grid), dim3(TC_THREADS), TcSmem::ALLOC, s, t);
}

}  // namespace apr
