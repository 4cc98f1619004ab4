// Batch-1 merge on the 5th-generation tensor cores (tcgen05).
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include <map>
#include <tuple>

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

// In-place merge and exact unmerge (AdaFuse summary §2.B steps 3 and 5: merge, run,
// unmerge for the next token).  The merge writes w' = rn(w + d) over w and, per element, the
// distance from w to u = rn(w' - d), the value the unmerge will recompute, counted in
// representable bf16 steps (keys that order the bit patterns like the values).  The unmerge
// recomputes d (the same tensor-core product, bit for bit), forms u and steps back by the
// stored distance.  Distances outside [-126, 127] become escapes: the exact bits go to a list
// written back after the unmerge; when the list is full the element is left unmerged (code
// -127) and the merge reports APR_ERR_WORKSPACE, so restoration stays exact either way.
constexpr int MERGE_OUT_OF_PLACE = 0, MERGE_IN_PLACE = 1, UNMERGE_IN_PLACE = 2;
constexpr int8_t kCodeEscape = -128, kCodeKept = -127;

struct MergeEscapes {                  // device, caller-owned (apr_merge_escape_bytes)
  unsigned int count;                  // escapes met (may exceed the capacity: those were kept)
  int k;                               // the merge's routing, checked by the unmerge
  int e[APR_MAX_K];
  float g[APR_MAX_K];
  int pad[14];
  // then the capacity's entries {weight, element, bits}, 3 x 32 bits each
};
static_assert(sizeof(MergeEscapes) == 128, "escape header is 128 bytes");

// key: positive values b ^ 0x8000, negative ones ~b (16 bits), so keys ascend with the values
__device__ __forceinline__ int bf16_key(uint32_t b) {
  return (int)((b ^ 0x8000u ^ ((uint32_t)((int32_t)(b << 16) >> 31) & 0x7FFFu)) & 0xFFFFu);
}
__device__ __forceinline__ uint32_t bf16_from_key(int key) {
  const uint32_t k = (uint32_t)key & 0xFFFFu;
  return k ^ (0xFFFFu ^ (((k >> 15) & 1u) * 0x7FFFu));
}
__device__ __forceinline__ float bf16_val(uint32_t b) { return __uint_as_float(b << 16); }
// bytes of x picked by the selector nibbles; a nibble with bit 3 set gives the picked byte's sign
// replicated (PTX prmt, default mode)
__device__ __forceinline__ uint32_t prmt_sext(uint32_t x, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(x), "r"(sel));
  return r;
}
// the same key and its inverse on the two 16-bit halves of a word
__device__ __forceinline__ uint32_t bf16_key2(uint32_t x) {
  return x ^ 0x80008000u ^ (((x >> 15) & 0x00010001u) * 0x7FFFu);
}
__device__ __forceinline__ uint32_t bf16_from_key2(uint32_t k) {
  return k ^ (0xFFFFFFFFu ^ (((k >> 15) & 0x00010001u) * 0x7FFFu));
}
__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 h) { return *reinterpret_cast<const uint32_t*>(&h); }

template <int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1) merge_tc_kernel(const apr_merge_proj* __restrict__ projs,
                                                                 int nproj, int E, int r, int R16,
                                                                 const int32_t* __restrict__ idx,
                                                                 const float* __restrict__ gate, int k,
                                                                 void* ws, MergeEscapes* esc, long esc_cap) {
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
  if (MODE == MERGE_IN_PLACE && blockIdx.x == 0 && tid == 0 && !s_flags[1]) {
    esc->k = k;
    for (int j = 0; j < k; ++j) {
      esc->e[j] = s_e[j];
      esc->g[j] = s_g[j];
    }
  }
  if (MODE == UNMERGE_IN_PLACE && tid == 0) {
    // the unmerge must recompute the merge's delta exactly: the same adapters and gates
    bool same = esc->k == k;
    for (int j = 0; j < k && same; ++j) same = esc->e[j] == s_e[j] && esc->g[j] == s_g[j];
    if (!same && !s_flags[1]) s_flags[1] = 2;
  }
  __syncthreads();
  bool abort = false;
  if (s_flags[1]) {
    if (tid == 0 && blockIdx.x == 0)
      report(ws, s_flags[1] == 2 ? APR_ERR_INVALID_ARG : APR_ERR_DEVICE_INDEX, K_MERGE, 0);
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
      const __nv_bfloat16* Wt = reinterpret_cast<const __nv_bfloat16*>(pj.W);
      // out of place: W' to Wp; in place: back over W, with the residual codes in Wp (int8)
      __nv_bfloat16* Wp = MODE == MERGE_OUT_OF_PLACE ? reinterpret_cast<__nv_bfloat16*>(pj.Wp)
                                                     : const_cast<__nv_bfloat16*>(Wt);
      int8_t* Rc = MODE == MERGE_OUT_OF_PLACE ? nullptr : reinterpret_cast<int8_t*>(pj.Wp);
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
        // unmerge: this row's residual codes of the tile, loaded now so that their latency passes
        // under the MMA's
        uint4 tile_codes[MODE == UNMERGE_IN_PLACE ? 8 : 1];
        if (MODE == UNMERGE_IN_PLACE) {
          const uint4* rt = reinterpret_cast<const uint4*>(Rc + ((size_t)(row0 / TC_BM) * nct + ct) * 8 * 2048) + tid;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            tile_codes[q] = (q * 16 < ncols && tid < nrows) ? rt[q * 128] : make_uint4(0, 0, 0, 0);
        }
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
              if (MODE == MERGE_OUT_OF_PLACE) {
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
              } else {
                // residual codes, tile-major: [strip][column tile][16-column chunk][row][16 bytes],
                // so a warp's 32 rows of one chunk are 512 contiguous bytes
                unsigned int* hw = reinterpret_cast<unsigned int*>(pr);       // 8 x bf16 pairs
                uint4* rc = reinterpret_cast<uint4*>(Rc + (((size_t)(row0 / TC_BM) * nct + ct) * 8 + (cc >> 4)) * 2048) + tid;
                uint4 cw = make_uint4(0, 0, 0, 0);
                uint32_t* cwd = reinterpret_cast<uint32_t*>(&cw);
                uint32_t bf16_orig[16];                                       // W bits (escapes)
                if (MODE == MERGE_IN_PLACE) {
#pragma unroll
                  for (int i = 0; i < 16; ++i) bf16_orig[i] = (hw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
                  // common path on bf16 pairs; elements whose distance does not fit a code are
                  // marked and settled below, one warp-wide counter update per chunk
                  uint32_t esc_mask = 0;
#pragma unroll
                  for (int i = 0; i < 16; i += 2) {
                    const uint32_t w2 = hw[i >> 1];
                    const uint32_t m2 = bf16x2_bits(__floats2bfloat162_rn(bf16_val(w2 & 0xFFFFu) + v[i],
                                                                          bf16_val(w2 >> 16) + v[i + 1]));
                    const uint32_t u2 = bf16x2_bits(__floats2bfloat162_rn(bf16_val(m2 & 0xFFFFu) - v[i],
                                                                          bf16_val(m2 >> 16) - v[i + 1]));
                    const uint32_t kw = bf16_key2(w2), ku = bf16_key2(u2);
                    const int dl = (int)(kw & 0xFFFFu) - (int)(ku & 0xFFFFu);
                    const int dh = (int)(kw >> 16) - (int)(ku >> 16);
                    esc_mask |= ((uint32_t)(dl + 126) > 253u ? 1u : 0u) << i;
                    esc_mask |= ((uint32_t)(dh + 126) > 253u ? 1u : 0u) << (i + 1);
                    const uint32_t pair = ((uint32_t)dl & 0xFFu) | (((uint32_t)dh & 0xFFu) << 8);
                    cwd[i >> 2] |= pair << (16 * ((i >> 1) & 1));
                    hw[i >> 1] = m2;
                  }
                  if (ncols - cc < 16) esc_mask &= (1u << (ncols - cc)) - 1u;   // columns past the weight
                  const unsigned int act = __activemask();
                  const unsigned int want = __ballot_sync(act, esc_mask != 0);
                  if (want) {
                    const int leader = __ffs(want) - 1;
                    unsigned int base = 0;
                    const unsigned int before = __popc(esc_mask);
                    // exclusive scan of the active lanes' escape counts (rarely taken)
                    unsigned int offs = 0, total_w = 0;
                    for (int l = 0; l < 32; ++l) {
                      const unsigned int n_l = __shfl_sync(act, before, l);
                      if ((act >> l) & 1u) {
                        total_w += n_l;
                        if (l < lane) offs += n_l;
                      }
                    }
                    if (lane == leader) base = atomicAdd(&esc->count, total_w);
                    base = __shfl_sync(act, base, leader);
                    int8_t* code = reinterpret_cast<int8_t*>(&cw);
                    for (int i = 0; i < 16; ++i) {
                      if (!((esc_mask >> i) & 1u)) continue;
                      const uint32_t wb = bf16_orig[i];
                      const unsigned int slot = base + offs++;
                      if ((long)slot < esc_cap) {
                        unsigned int* ent = reinterpret_cast<unsigned int*>(esc + 1) + 3 * (size_t)slot;
                        ent[0] = (unsigned int)lo;
                        ent[1] = (unsigned int)((size_t)(row0 + tid) * pj.d_in + c0 + cc + i);
                        ent[2] = wb;
                        code[i] = kCodeEscape;
                      } else {
                        code[i] = kCodeKept;                           // no room: left unmerged
                        hw[i >> 1] = (hw[i >> 1] & ~(0xFFFFu << (16 * (i & 1)))) | (wb << (16 * (i & 1)));
                        report(ws, APR_ERR_WORKSPACE, K_MERGE, lo);
                      }
                    }
                  }
                  *rc = cw;
                } else {
#pragma unroll
                  for (int q = 0; q < 8; ++q)
                    if (q == (cc >> 4)) cw = tile_codes[q];
                  // bytes 0x80 / 0x81 (escape / kept) anywhere in the chunk take the slow path
                  uint32_t special = 0;
#pragma unroll
                  for (int q = 0; q < 4; ++q) special |= __vcmpeq4(cwd[q], 0x80808080u) | __vcmpeq4(cwd[q], 0x81818181u);
                  if (!__any_sync(__activemask(), special != 0)) {
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                      const uint32_t w2 = hw[i >> 1];
                      const uint32_t u2 = bf16x2_bits(__floats2bfloat162_rn(bf16_val(w2 & 0xFFFFu) - v[i],
                                                                            bf16_val(w2 >> 16) - v[i + 1]));
                      // the two codes sign-extended to 16-bit halves, added to the keys of u
                      const uint32_t c2 = prmt_sext(cwd[i >> 2], ((i >> 1) & 1) ? 0xB3A2u : 0x9180u);
                      hw[i >> 1] = bf16_from_key2(__vadd2(bf16_key2(u2), c2));
                    }
                  } else {
                    // a chunk of this warp holds an escape or a kept element: element by element
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                      const uint32_t w2 = hw[i >> 1];
                      const uint32_t u2 = bf16x2_bits(__floats2bfloat162_rn(bf16_val(w2 & 0xFFFFu) - v[i],
                                                                            bf16_val(w2 >> 16) - v[i + 1]));
                      uint32_t out = 0;
#pragma unroll
                      for (int h = 0; h < 2; ++h) {
                        const int8_t c = reinterpret_cast<const int8_t*>(&cw)[i + h];
                        const uint32_t wb = (w2 >> (16 * h)) & 0xFFFFu, ub = (u2 >> (16 * h)) & 0xFFFFu;
                        const uint32_t rb = c == kCodeKept ? wb : (c == kCodeEscape ? ub : bf16_from_key(bf16_key(ub) + c));
                        out |= rb << (16 * h);
                      }
                      hw[i >> 1] = out;
                    }
                  }
                }
              }
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

cudaError_t encode_box_map(CUtensorMap* m, const void* base, long rows, long cols, long pitch_bytes, int box_cols,
                           int box_rows, bool swizzle128) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? cudaSuccess
             : cudaErrorInvalidValue;
}

// Tensor-map templates depend only on shapes, so they are encoded once per shape (the address is
// a placeholder the kernels replace on the device).
cudaError_t cached_box_map(CUtensorMap* m, const void* placeholder, long rows, long cols, long pitch_bytes,
                           int box_cols, int box_rows, bool swizzle128) {
  using Key = std::tuple<long, long, long, int, int, int>;
  static std::mutex mu;
  static std::map<Key, CUtensorMap> cache;
  const Key key{rows, cols, pitch_bytes, box_cols, box_rows, swizzle128 ? 1 : 0};
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *m = it->second;
    return cudaSuccess;
  }
  cudaError_t err = encode_box_map(m, placeholder, rows, cols, pitch_bytes, box_cols, box_rows, swizzle128);
  if (err == cudaSuccess) cache.emplace(key, *m);
  return err;
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

// The unmerge's last step: every escaped element gets its exact bits back (unless the routing
// is not the merge's, in which case the unmerge itself refused and wrote nothing).
__global__ void __launch_bounds__(256) merge_escape_kernel(const apr_merge_proj* __restrict__ projs,
                                                           const MergeEscapes* esc, long esc_cap,
                                                           const int32_t* __restrict__ idx,
                                                           const float* __restrict__ gate, int k) {
  pdl_wait();
  pdl_trigger();
  bool same = esc->k == k;
  for (int j = 0; j < k && same; ++j) same = esc->e[j] == idx[j] && esc->g[j] == gate[j];
  if (!same) return;
  const long n = min((long)esc->count, esc_cap);
  const unsigned int* ent = reinterpret_cast<const unsigned int*>(esc + 1);
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const unsigned int p = ent[3 * i], el = ent[3 * i + 1], bits = ent[3 * i + 2];
    reinterpret_cast<unsigned short*>(const_cast<void*>(projs[p].W))[el] = (unsigned short)bits;
  }
}

size_t merge_escape_bytes(long capacity) { return sizeof(MergeEscapes) + (size_t)12 * (size_t)capacity; }
size_t merge_residual_bytes(int d_out, int d_in) {
  return (size_t)((d_out + TC_BM - 1) / TC_BM) * (size_t)((d_in + MT_BN - 1) / MT_BN) * TC_BM * MT_BN;
}

cudaError_t launch_merge_inplace(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                 const float* gate, int k, void* escapes, long capacity, bool unmerge, void* ws,
                                 cudaStream_t s) {
  const size_t smem = MtSmem::fixed_bytes() + sizeof(int) * ((size_t)nproj + 1);
  static SmemLimit lim1, lim2;
  cudaError_t err;
  MergeEscapes* esc = reinterpret_cast<MergeEscapes*>(escapes);
  const int nsm = device_sm_count();
  if (!unmerge) {
    if ((err = lim1.ensure((const void*)merge_tc_kernel<MERGE_IN_PLACE>, smem)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(esc, 0, sizeof(MergeEscapes), s)) != cudaSuccess) return err;
    return launch_pdl(merge_tc_kernel<MERGE_IN_PLACE>, dim3(nsm), dim3(TC_THREADS), smem, s, projs, nproj, E, r,
                      round16(r), idx, gate, k, ws, esc, capacity);
  }
  if ((err = lim2.ensure((const void*)merge_tc_kernel<UNMERGE_IN_PLACE>, smem)) != cudaSuccess) return err;
  if ((err = launch_pdl(merge_tc_kernel<UNMERGE_IN_PLACE>, dim3(nsm), dim3(TC_THREADS), smem, s, projs, nproj, E, r,
                        round16(r), idx, gate, k, ws, esc, capacity)) != cudaSuccess)
    return err;
  return launch_pdl(merge_escape_kernel, dim3(nsm), dim3(256), 0, s, projs, (const MergeEscapes*)esc, capacity, idx,
                    gate, k);
}

bool merge_tensor_supported(int k, int r, int nproj) {
  return k * round16(r) <= TC_MAXN1 && nproj <= MT_MAXPROJ;
}

cudaError_t launch_merge_tensor(const apr_merge_proj* projs, int nproj, int E, int r, const int32_t* idx,
                                const float* gate, int k, void* ws, cudaStream_t s) {
  const size_t smem = MtSmem::fixed_bytes() + sizeof(int) * ((size_t)nproj + 1);
  static SmemLimit limit;
  cudaError_t err = limit.ensure((const void*)merge_tc_kernel<MERGE_OUT_OF_PLACE>, smem);
  if (err != cudaSuccess) return err;
  const int nsm = device_sm_count();
  return launch_pdl(merge_tc_kernel<MERGE_OUT_OF_PLACE>, dim3(nsm), dim3(TC_THREADS), smem, s, projs, nproj, E, r,
                    round16(r), idx, gate, k, ws, (MergeEscapes*)nullptr, 0L);
}

}  // namespace apr
