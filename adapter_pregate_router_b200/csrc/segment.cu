// Segments of the segmented gather product (AdaFuse summary, gist.science,
// Resumen tecnico §2.B: SGMM gathers the tokens of each adapter and runs one
// batched product).  One CTA of 1024 threads builds, bit-exactly and
// deterministically:
//   seg_off [E+1]  exclusive prefix sum of the per-adapter pair counts
//   perm    [T*k]  pair ids q = t*k+j grouped by adapter, ascending q inside
//                  a segment (stable counting sort)
// and the routing plan in the workspace:
//   inv      [T*k] sorted position of pair q
//   tiles    pair tiles (<= kPairTile pairs of one adapter) for the shrink
//   tok_order[T]   tokens ordered by their sorted adapter tuple (LSD radix of
//                  k stable counting sorts), so that tokens sharing an adapter
//                  set are contiguous
//   qtiles         tiles of <= 128 pairs of one adapter (tensor-core shrink)
// The top-2 gathered tensor-core expand also needs, built on demand by the
// first such call after the plan (gather_plan_kernel; no other path pays):
//   set tiles      runs of <= kSetTile tokens with one adapter set
//   mixed tiles    runs of <= 128 consecutive plan tokens whose adapters
//                  number <= 4 (k <= 2), built by one thread walking the set
//                  tiles in order
// The histograms use shared-memory atomics (order-free counts).  The order-
// dependent steps (the stable scatters of the pairs and of the tokens, the set
// tiles) run over blocks of 1024 consecutive items, all 32 warps at once: a
// warp ranks equal keys by lane with __match_any_sync, the per-key counts of
// the 32 warps are scanned across warps in shared memory, and a per-key base
// carries from one block to the next, so the result is unique.  idx and the
// token order are staged in shared memory when they fit.
#include <climits>

#include "apr_internal.cuh"

namespace apr {

constexpr int SEG_THREADS = 1024;
constexpr int MIX_CHUNK = 1024;      // set tiles staged per pass of the mixed-tile walk

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive scan of one value per thread over the whole block; *total gets the sum.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[nwarps - 1];
  __syncthreads();
  return before;
}

// Inclusive max over the block (one value per thread).
__device__ int block_inclusive_max(int v, int* warp_vals) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x = max(x, y);
  }
  if (lane == 31) warp_vals[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? warp_vals[lane] : INT_MIN;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s = max(s, y);
    }
    warp_vals[lane] = s;
  }
  __syncthreads();
  const int r = warp > 0 ? max(warp_vals[warp - 1], x) : x;
  __syncthreads();
  return r;
}

// Stable rank of one block of up to 1024 items (thread i holds item i of the
// block, key in [0, E) when valid): returns base[key] + the number of earlier
// items of this block with the same key, and advances base[key] by the block's
// count of that key.  cnt is a [32][E] table of zeros on entry and on exit.
__device__ int block_stable_rank(int key, bool valid, int E, int* base, uint16_t* cnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? key : -1);
  const int intra = __popc(peers & lanemask_lt());
  if (valid && lane == __ffs(peers) - 1) cnt[warp * E + key] = (uint16_t)__popc(peers);
  __syncthreads();
  int run = 0;
  if (tid < E) {                           // this key's count in each warp -> exclusive prefix over warps
#pragma unroll 8
    for (int w = 0; w < 32; ++w) {
      const int c = cnt[w * E + tid];
      cnt[w * E + tid] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
  const int pos = valid ? base[key] + cnt[warp * E + key] + intra : -1;
  __syncthreads();
  if (tid < E) {
    base[tid] += run;
#pragma unroll 8
    for (int w = 0; w < 32; ++w) cnt[w * E + tid] = 0;
  }
  __syncthreads();
  return pos;
}

// The p-th smallest adapter of token t (its tuple sorted ascending).
__device__ __forceinline__ int sorted_key(const int32_t* idx, int t, int k, int p) {
  if (k == 1) return idx[t];
  if (k == 2) {
    const int a0 = idx[2 * (size_t)t], a1 = idx[2 * (size_t)t + 1];
    return p == 0 ? min(a0, a1) : max(a0, a1);
  }
  int a[APR_MAX_K];
#pragma unroll
  for (int j = 0; j < APR_MAX_K; ++j) a[j] = j < k ? idx[(size_t)t * k + j] : 0x7FFFFFFF;
#pragma unroll
  for (int i = 1; i < APR_MAX_K; ++i) {
#pragma unroll
    for (int j = APR_MAX_K - 1; j >= 1; --j) {
      if (j <= i && a[j - 1] > a[j]) {
        const int tmp = a[j];
        a[j] = a[j - 1];
        a[j - 1] = tmp;
      }
    }
  }
  int r = a[0];
#pragma unroll
  for (int j = 1; j < APR_MAX_K; ++j)
    if (j == p) r = a[j];
  return r;
}

__device__ __forceinline__ bool same_set(const int32_t* idx, int t0, int t1, int k) {
  for (int p = 0; p < k; ++p)
    if (sorted_key(idx, t0, k, p) != sorted_key(idx, t1, k, p)) return false;
  return true;
}

// Dynamic shared memory: hist [E], base [E] (int), cnt [32][E] (uint16), and
// with STAGE idx [T*k], two token arrays [T] (int).
__host__ __device__ inline size_t seg_smem_fixed(int E) {
  return (sizeof(int) * 2 * (size_t)E + sizeof(uint16_t) * 32 * (size_t)E + 15) / 16 * 16;
}
__host__ __device__ inline size_t seg_smem_stage(int T, int k) { return sizeof(int) * ((size_t)T * k + 2 * (size_t)T); }

template <bool STAGE>
__global__ void __launch_bounds__(SEG_THREADS) segment_kernel(const int32_t* __restrict__ idx_g, int T,
                                                              int k, int E,
                                                              int32_t* __restrict__ seg_off,
                                                              int32_t* __restrict__ perm, void* ws) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char seg_smem[];
  int* hist = reinterpret_cast<int*>(seg_smem);                   // [E]
  int* base = hist + E;                                           // [E]
  uint16_t* cnt = reinterpret_cast<uint16_t*>(base + E);          // [32][E]
  int* stage = reinterpret_cast<int*>(seg_smem + seg_smem_fixed(E));
  __shared__ int warp_sums[32];
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int n = T * k;
  const WsLayout L = ws_layout(T, k, E);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  int* inv = ws_at<int>(ws, L.inv);
  int* tok_order = ws_at<int>(ws, L.tok_order);
  int* tok_tmp = ws_at<int>(ws, L.tok_tmp);
  PairTile* ptiles = ws_at<PairTile>(ws, L.ptiles);
  SetTile* stiles = ws_at<SetTile>(ws, L.stiles);
  const int32_t* idx = STAGE ? stage : idx_g;
  int* tok_a = STAGE ? stage + n : tok_tmp;
  int* tok_b = STAGE ? stage + n + T : tok_order;

  // 0. zero the rank table, stage idx
  for (int i = tid; i < 32 * E; i += SEG_THREADS) cnt[i] = 0;
  if (STAGE)
    for (int q = tid; q < n; q += SEG_THREADS) stage[q] = idx_g[q];
  // 1. counts and validation
  for (int e = tid; e < E; e += SEG_THREADS) hist[e] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int q = tid; q < n; q += SEG_THREADS) {
    const int e = idx[q];
    if (e < 0 || e >= E) {
      bad = 1;
    } else {
      atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  if (bad) {
    for (int e = tid; e <= E; e += SEG_THREADS) seg_off[e] = 0;
    if (tid == 0) {
      report(ws, APR_ERR_DEVICE_INDEX, K_SEGMENT, 0);
      hdr->n_ptiles = 0;
      hdr->n_stiles = 0;
      hdr->n_qtiles = 0;
      hdr->n_mtiles = 0;
      hdr->gplan = 1;                  // the empty plan needs no gathered tiles
    }
    return;
  }
  // 2. segment offsets
  int total;
  {
    const int c = tid < E ? hist[tid] : 0;
    const int off = block_exclusive_scan(c, warp_sums, &total);
    if (tid < E) {
      base[tid] = off;
      seg_off[tid] = off;
    }
    if (tid == 0) seg_off[E] = total;
  }
  __syncthreads();
  // 3. shrink pair tiles: ceil(count / kPairTile) per adapter, in adapter order
  {
    const int c = tid < E ? hist[tid] : 0;
    const int nt = (c + kPairTile - 1) / kPairTile;
    int ntiles;
    const int toff = block_exclusive_scan(nt, warp_sums, &ntiles);
    if (tid < E) {
      const int s0 = base[tid];
      for (int i = 0; i < nt; ++i) {
        PairTile p;
        p.e = tid;
        p.start = s0 + i * kPairTile;
        p.len = min(kPairTile, c - i * kPairTile);
        p.pad = 0;
        ptiles[toff + i] = p;
      }
    }
    if (tid == 0) {
      hdr->n_ptiles = ntiles;
      hdr->sched = 0;
      hdr->T = T;
      hdr->k = k;
      hdr->E = E;
    }
  }
  __syncthreads();
  // 3b. tensor-core pair tiles: ceil(count / kSetTile) per adapter, in adapter order
  {
    PairTile* qtiles = ws_at<PairTile>(ws, L.qtiles);
    const int c = tid < E ? hist[tid] : 0;
    const int nt = (c + kSetTile - 1) / kSetTile;
    int ntiles;
    const int toff = block_exclusive_scan(nt, warp_sums, &ntiles);
    if (tid < E) {
      const int s0 = base[tid];
      for (int i = 0; i < nt; ++i) {
        PairTile p;
        p.e = tid;
        p.start = s0 + i * kSetTile;
        p.len = min(kSetTile, c - i * kSetTile);
        p.pad = 0;
        qtiles[toff + i] = p;
      }
    }
    if (tid == 0) hdr->n_qtiles = ntiles;
  }
  __syncthreads();
  // 4. stable scatter of the pairs, 1024 at a time
  for (int q0 = 0; q0 < n; q0 += SEG_THREADS) {
    const int q = q0 + tid;
    const bool valid = q < n;
    const int pos = block_stable_rank(valid ? idx[q] : 0, valid, E, base, cnt);
    if (valid) {
      perm[pos] = q;
      inv[q] = pos;
    }
  }
  // 5. tokens ordered by sorted adapter tuple: LSD, k stable counting sorts
  int* src = tok_a;
  int* dst = tok_b;
  for (int i = tid; i < T; i += SEG_THREADS) src[i] = i;
  for (int p = k - 1; p >= 0; --p) {
    for (int e = tid; e < E; e += SEG_THREADS) hist[e] = 0;
    __syncthreads();
    for (int i = tid; i < T; i += SEG_THREADS) atomicAdd(&hist[sorted_key(idx, i, k, p)], 1);
    __syncthreads();
    {
      const int c = tid < E ? hist[tid] : 0;
      int tot;
      const int off = block_exclusive_scan(c, warp_sums, &tot);
      if (tid < E) base[tid] = off;
    }
    __syncthreads();
    for (int i0 = 0; i0 < T; i0 += SEG_THREADS) {
      const int i = i0 + tid;
      const bool valid = i < T;
      const int t = valid ? src[i] : 0;
      const int pos = block_stable_rank(valid ? sorted_key(idx, t, k, p) : 0, valid, E, base, cnt);
      if (valid) dst[pos] = t;
    }
    int* tmp = src;
    src = dst;
    dst = tmp;
  }
  // src holds the final order; the plan keeps it in tok_order
  if (src != tok_order) {
    for (int i = tid; i < T; i += SEG_THREADS) tok_order[i] = src[i];
  }
  // the gathered expand's set and mixed tiles are built on demand (gather_plan_kernel)
  if (tid == 0) hdr->gplan = 0;
}

// Set tiles and mixed tiles of the current plan, the tiles of the gathered tensor-core expand
// only: built by the first call that needs them after the plan (the header flag makes later calls
// of the same plan return at once), so the other paths do not pay for them.
template <bool STAGE>
__global__ void __launch_bounds__(SEG_THREADS) gather_plan_kernel(const int32_t* __restrict__ idx_g, int T, int k,
                                                                  int E, void* ws) {
  pdl_wait();
  pdl_trigger();
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  if (*reinterpret_cast<volatile int*>(&hdr->gplan)) return;
  extern __shared__ __align__(16) unsigned char gp_smem[];
  __shared__ int warp_sums[32];
  __shared__ int carry[2];
  const int tid = threadIdx.x;
  const int n = T * k;
  const WsLayout L = ws_layout(T, k, E);
  const int* tok_order = ws_at<int>(ws, L.tok_order);
  SetTile* stiles = ws_at<SetTile>(ws, L.stiles);
  int* stage = reinterpret_cast<int*>(gp_smem);
  if (STAGE) {
    for (int q = tid; q < n; q += SEG_THREADS) stage[q] = idx_g[q];
    for (int i = tid; i < T; i += SEG_THREADS) stage[n + i] = tok_order[i];
    __syncthreads();
  }
  const int32_t* idx = STAGE ? stage : idx_g;
  const int* order = STAGE ? stage + n : tok_order;
  // 6. set tiles: runs of equal adapter sets, split into <= kSetTile tokens.  A run starts
  //    where the set changes; a tile starts at a run start or every kSetTile tokens into a run.
  if (tid == 0) {
    carry[0] = 0;  // start of the current run
    carry[1] = 0;  // tiles written
  }
  __syncthreads();
  for (int i0 = 0; i0 < T; i0 += SEG_THREADS) {
    const int i = i0 + tid;
    const bool valid = i < T;
    const bool head = valid && (i == 0 || !same_set(idx, order[i - 1], order[i], k));
    const int rs = max(block_inclusive_max(head ? i : -1, warp_sums), carry[0]);
    const bool tstart = valid && (head || ((i - rs) % kSetTile) == 0);
    int ntot;
    const int off = block_exclusive_scan(tstart ? 1 : 0, warp_sums, &ntot);
    if (tstart) {
      SetTile st;
      st.start = i;
      st.len = 0;
      stiles[carry[1] + off] = st;
    }
    __syncthreads();
    if (tid == SEG_THREADS - 1) {
      carry[0] = rs;
      carry[1] += ntot;
    }
    __syncthreads();
  }
  const int nst = carry[1];
  for (int j = tid; j < nst; j += SEG_THREADS) {
    const int end = (j + 1 < nst) ? stiles[j + 1].start : T;
    stiles[j].len = end - stiles[j].start;
  }
  if (tid == 0) hdr->n_stiles = nst;
  // 7. mixed tiles (k <= 2): consecutive set-ordered tokens, <= kSetTile of them, whose
  //    adapters number <= kMixAdapters; greedy over the set tiles, one thread walking chunks
  //    of the set tiles staged in shared memory.
  __syncthreads();
  if (k > 2) {
    if (tid == 0) {
      hdr->n_mtiles = 0;
      hdr->gplan = 1;
    }
    return;
  }
  {
    MixTile* mtiles = ws_at<MixTile>(ws, L.mtiles);
    __shared__ int4 s_st[MIX_CHUNK];       // start, len, a0, a1 of a chunk of set tiles
    __shared__ MixTile s_cur;
    __shared__ int s_nm;
    if (tid == 0) {
      s_cur.start = 0;
      s_cur.len = 0;
      s_cur.nu = 0;
      s_nm = 0;
    }
    for (int c0 = 0; c0 < nst; c0 += MIX_CHUNK) {
      __syncthreads();
      for (int j = tid; j < MIX_CHUNK && c0 + j < nst; j += SEG_THREADS) {
        const SetTile st = stiles[c0 + j];
        const int t0 = order[st.start];
        const int a0 = sorted_key(idx, t0, k, 0);
        const int a1 = k == 2 ? sorted_key(idx, t0, k, 1) : -1;
        s_st[j] = make_int4(st.start, st.len, a0, a1);
      }
      __syncthreads();
      if (tid == 0) {
        // the open tile: start, length and its adapters u0 < u1 < u2 < u3 (INT_MAX: unused),
        // all in registers
        int cstart = s_cur.start, clen = s_cur.len, nu = s_cur.nu;
        int u0 = nu > 0 ? s_cur.u[0] : INT_MAX, u1 = nu > 1 ? s_cur.u[1] : INT_MAX;
        int u2 = nu > 2 ? s_cur.u[2] : INT_MAX, u3 = nu > 3 ? s_cur.u[3] : INT_MAX;
        int nm = s_nm;
        const int n = min(MIX_CHUNK, nst - c0);
        for (int j = 0; j < n; ++j) {
          const int4 t = s_st[j];
          int remaining = t.y, pos = t.x;
          // adapters of this set not yet in the tile (a1 < 0 when k == 1)
          const bool new0 = t.z != u0 && t.z != u1 && t.z != u2 && t.z != u3;
          const bool new1 = t.w >= 0 && t.w != t.z && t.w != u0 && t.w != u1 && t.w != u2 && t.w != u3;
          const int add = (int)new0 + (int)new1;
          while (remaining > 0) {
            const bool fits = clen == 0 || (nu + add <= kMixAdapters && clen < kSetTile);
            if (!fits) {                          // close the tile; this set opens the next one
              MixTile mt;
              mt.start = cstart;
              mt.len = clen;
              mt.nu = nu;
              mt.pad = 0;
              mt.u[0] = u0; mt.u[1] = u1; mt.u[2] = u2; mt.u[3] = u3;
              for (int q = nu; q < kMixAdapters; ++q) mt.u[q] = 0;
              mtiles[nm++] = mt;
              clen = 0;
              nu = 0;
              u0 = u1 = u2 = u3 = INT_MAX;
            }
            if (clen == 0) {
              cstart = pos;
              // a fresh tile holds exactly this set's adapters
              nu = 0;
              u0 = u1 = u2 = u3 = INT_MAX;
            }
            if (clen == 0 || new0 || new1) {
              // sorted insert of the set's adapters not yet present (branch-free over 4 registers)
              const int vs[2] = {t.z, t.w};
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int v = vs[q];
                const bool present = v == u0 || v == u1 || v == u2 || v == u3;
                if (v >= 0 && !present) {
                  const int n3 = min(u3, max(u2, v)), n2 = min(u2, max(u1, v)), n1 = min(u1, max(u0, v));
                  u0 = min(u0, v);
                  u1 = n1;
                  u2 = n2;
                  u3 = n3;
                  ++nu;
                }
              }
            }
            const int take = min(remaining, kSetTile - clen);
            clen += take;
            remaining -= take;
            pos += take;
          }
        }
        s_cur.start = cstart;
        s_cur.len = clen;
        s_cur.nu = nu;
        s_cur.u[0] = u0; s_cur.u[1] = u1; s_cur.u[2] = u2; s_cur.u[3] = u3;
        s_nm = nm;
      }
    }
    __syncthreads();
    if (tid == 0) {
      int nm = s_nm;
      if (s_cur.len > 0) mtiles[nm++] = s_cur;
      hdr->n_mtiles = nm;
      hdr->gplan = 1;
    }
  }
}


cudaError_t launch_gather_plan(const int32_t* idx, int T, int k, int E, void* ws, cudaStream_t s) {
  // idx and the token order go to shared memory when they fit beside the mixed-tile staging
  constexpr size_t kStageBudget = 200 * 1024;
  const size_t need = sizeof(int) * ((size_t)T * k + (size_t)T);
  static SmemLimit lim;
  cudaError_t err;
  if (need <= kStageBudget) {
    if ((err = lim.ensure((const void*)gather_plan_kernel<true>, need)) != cudaSuccess) return err;
    return launch_pdl(gather_plan_kernel<true>, dim3(1), dim3(SEG_THREADS), need, s, idx, T, k, E, ws);
  }
  return launch_pdl(gather_plan_kernel<false>, dim3(1), dim3(SEG_THREADS), 0, s, idx, T, k, E, ws);
}

cudaError_t launch_segment(const int32_t* idx, int T, int k, int E, int32_t* seg_off,
                           int32_t* perm, void* ws, cudaStream_t s) {
  // idx and the token arrays go to shared memory when they fit beside the fixed tables
  constexpr size_t kStageBudget = 200 * 1024;
  const size_t fixed = seg_smem_fixed(E);
  const bool stage = fixed + seg_smem_stage(T, k) <= kStageBudget;
  const size_t smem = fixed + (stage ? seg_smem_stage(T, k) : 0);
  // the limit is raised for every size (static and dynamic shared memory count against one limit)
  static SmemLimit lim[2];
  cudaError_t err;
  if (stage) {
    if ((err = lim[1].ensure((const void*)segment_kernel<true>, smem)) != cudaSuccess) return err;
    return launch_pdl(segment_kernel<true>, dim3(1), dim3(SEG_THREADS), smem, s, idx, T, k, E, seg_off, perm, ws);
  }
  if ((err = lim[0].ensure((const void*)segment_kernel<false>, smem)) != cudaSuccess) return err;
  return launch_pdl(segment_kernel<false>, dim3(1), dim3(SEG_THREADS), smem, s, idx, T, k, E, seg_off, perm, ws);
}

}  // namespace apr
