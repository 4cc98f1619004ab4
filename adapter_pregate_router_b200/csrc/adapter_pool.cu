// Adapter paging: a pool of adapters larger than the device memory set aside for
// them lives in pinned host memory, and a fixed number of device slots hold the
// ones the current step's routing selected.  The Chameleon page (7minutos.es)
// describes loading adapters on demand and keeping the popular ones resident
// (an adaptive adapter cache, as in S-LoRA); with token-level pre-gating the
// adapters of a step are known only once the router has run on the device, so
// here the paging runs on the device as well, between the router and the
// first SGMM call, with no host round trip (the step stays one CUDA graph):
//
//  1. pool_decide_kernel (one CTA): marks the adapters idx selects, refreshes
//     the last-use stamp of the resident ones, and gives every missing one a
//     slot: empty slots first, then the least recently used slots not needed
//     by this step.  It rewrites, for every adapter paged in, its entry in
//     each of the caller's pointer tables (the A and B tables that the SGMM
//     calls take) to the slot's copy.  More distinct adapters than slots is
//     an error (APR_ERR_WORKSPACE) and changes nothing.
//  2. pool_copy_kernel (all SMs): copies each paged-in adapter's bytes from its
//     mapped pinned host buffer into its slot, 16 bytes per load, over PCIe.
//
// State lives in caller-owned device memory (apr_adapter_pool_state_bytes).
#include "apr_internal.cuh"

namespace apr {

struct PoolHeader {
  int n_adapters, n_slots;
  int n_copy;                           // adapters this call pages in
  int pad0;
  unsigned long long step;              // page-in calls so far
  unsigned long long copies;            // adapters paged in so far
  int pad[8];
};
static_assert(sizeof(PoolHeader) == 64, "pool header is 64 bytes");

struct PoolView {
  PoolHeader* h;
  int* slot_of;                         // [n_adapters] slot or -1
  int* id_of;                           // [n_slots] adapter or -1
  unsigned long long* last_used;        // [n_slots] step of the last use (0: never)
  int* copy_id;                         // [n_slots] this call's (adapter, slot) pairs
  int* copy_slot;
};

__host__ __device__ inline size_t pool_state_bytes(int n_adapters, int n_slots) {
  return sizeof(PoolHeader) + align_up(sizeof(int) * (size_t)n_adapters) + align_up(sizeof(int) * (size_t)n_slots) +
         align_up(sizeof(unsigned long long) * (size_t)n_slots) + 2 * align_up(sizeof(int) * (size_t)n_slots);
}

__host__ __device__ inline PoolView pool_view(void* state, int n_adapters, int n_slots) {
  PoolView v;
  char* p = reinterpret_cast<char*>(state);
  v.h = reinterpret_cast<PoolHeader*>(p);
  p += sizeof(PoolHeader);
  v.slot_of = reinterpret_cast<int*>(p);
  p += align_up(sizeof(int) * (size_t)n_adapters);
  v.id_of = reinterpret_cast<int*>(p);
  p += align_up(sizeof(int) * (size_t)n_slots);
  v.last_used = reinterpret_cast<unsigned long long*>(p);
  p += align_up(sizeof(unsigned long long) * (size_t)n_slots);
  v.copy_id = reinterpret_cast<int*>(p);
  p += align_up(sizeof(int) * (size_t)n_slots);
  v.copy_slot = reinterpret_cast<int*>(p);
  return v;
}

struct PoolArgs {
  void* state;
  int n_adapters, n_slots;
  const int32_t* idx;                   // [T * k]
  int nq;                               // T * k
  const void* const* host_src;          // device array [n_adapters]: mapped pinned host buffers
  size_t adapter_bytes;                 // bytes of one adapter (a multiple of 16)
  char* pool;                           // device, n_slots * adapter_bytes
  const unsigned long long* offsets;    // device [ntab]: byte offset of table t's matrix in an adapter
  void* const* tables;                  // device [ntab]: each a device array [n_adapters] of pointers
  int ntab;
  void* ws;
};

constexpr int PD_THREADS = 1024;

// Every table entry of every adapter starts at slot 0's copy (zeros until something is paged
// in): the dense and bank SGMM kernels read the whole adapter bank and multiply the adapters a
// token did not select by a zero gate, so an entry must always point at finite adapter-shaped
// data inside the pool, never at nothing.
__global__ void __launch_bounds__(PD_THREADS, 1) pool_init_kernel(void* state, int n_adapters, int n_slots,
                                                                  char* pool, const unsigned long long* offsets,
                                                                  void* const* tables, int ntab) {
  PoolView v = pool_view(state, n_adapters, n_slots);
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nt = gridDim.x * blockDim.x;
  for (long w = tid; w < (long)ntab * n_adapters; w += nt) {
    const int t = (int)(w / n_adapters), e = (int)(w - (long)t * n_adapters);
    reinterpret_cast<void**>(tables[t])[e] = pool + offsets[t];
  }
  if (tid == 0) {
    v.h->n_adapters = n_adapters;
    v.h->n_slots = n_slots;
    v.h->n_copy = 0;
    v.h->step = 0;
    v.h->copies = 0;
  }
  for (int i = tid; i < n_adapters; i += nt) v.slot_of[i] = -1;
  for (int i = tid; i < n_slots; i += nt) {
    v.id_of[i] = -1;
    v.last_used[i] = 0;
  }
}

__global__ void __launch_bounds__(PD_THREADS, 1) pool_decide_kernel(const __grid_constant__ PoolArgs a) {
  extern __shared__ int sh[];
  int* needed = sh;                                  // [n_adapters] 0/1, then the missing ids' order
  int* cand = sh + a.n_adapters;                     // [n_slots] 1 if the slot may be taken
  __shared__ int s_nneed, s_nmiss, s_bad;
  const int tid = threadIdx.x;
  PoolView v = pool_view(a.state, a.n_adapters, a.n_slots);
  pdl_wait();                                        // idx comes from the router
  pdl_trigger();
  for (int i = tid; i < a.n_adapters; i += PD_THREADS) needed[i] = 0;
  if (tid == 0) {
    s_nneed = s_nmiss = 0;
    s_bad = v.h->n_adapters != a.n_adapters || v.h->n_slots != a.n_slots;
  }
  __syncthreads();
  for (int t = tid; t < a.ntab; t += PD_THREADS)
    if (a.offsets[t] % 16 != 0 || a.offsets[t] >= a.adapter_bytes) atomicExch(&s_bad, 1);
  for (int q = tid; q < a.nq; q += PD_THREADS) {
    const int e = a.idx[q];
    if (e < 0 || e >= a.n_adapters) {
      if (atomicExch(&s_bad, 2) == 0) report(a.ws, APR_ERR_DEVICE_INDEX, K_POOL, e);
    } else {
      needed[e] = 1;
    }
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      if (s_bad == 1) report(a.ws, APR_ERR_INVALID_ARG, K_POOL, 0);   // another pool's state, or an offset outside an adapter
      v.h->n_copy = 0;
    }
    return;
  }
  const unsigned long long step = v.h->step + 1;
  // needed adapters, the missing ones among them, and the slots a missing one may take
  for (int i = tid; i < a.n_adapters; i += PD_THREADS)
    if (needed[i]) {
      atomicAdd(&s_nneed, 1);
      if (v.slot_of[i] < 0) atomicAdd(&s_nmiss, 1);
    }
  for (int s = tid; s < a.n_slots; s += PD_THREADS) {
    const int id = v.id_of[s];
    cand[s] = id < 0 || !needed[id];
  }
  __syncthreads();
  const int nmiss = s_nmiss;
  if (s_nneed > a.n_slots) {
    if (tid == 0) {
      report(a.ws, APR_ERR_WORKSPACE, K_POOL, s_nneed);
      v.h->n_copy = 0;
    }
    return;
  }
  // the i-th missing adapter (ascending id) takes the candidate slot of rank i, candidates
  // ordered by (last use, slot): never-used and emptied slots (stamp 0) first
  for (int s = tid; s < a.n_slots; s += PD_THREADS) {
    if (!cand[s]) continue;
    const unsigned long long ls = v.last_used[s];
    int rank = 0;
    for (int o = 0; o < a.n_slots; ++o)
      if (cand[o] && (v.last_used[o] < ls || (v.last_used[o] == ls && o < s))) ++rank;
    if (rank < nmiss) {
      // the missing adapter of this rank: count missing ids below each candidate id
      int id = -1;
      for (int i = 0, r = 0; i < a.n_adapters; ++i)
        if (needed[i] && v.slot_of[i] < 0) {
          if (r == rank) { id = i; break; }
          ++r;
        }
      v.copy_id[rank] = id;
      v.copy_slot[rank] = s;
    }
  }
  __syncthreads();
  // apply: evict, map, stamp; refresh the stamps of the resident needed adapters
  for (int c = tid; c < nmiss; c += PD_THREADS) {
    const int id = v.copy_id[c], s = v.copy_slot[c];
    const int old = v.id_of[s];
    if (old >= 0) v.slot_of[old] = -1;
    v.id_of[s] = id;
  }
  __syncthreads();
  for (int c = tid; c < nmiss; c += PD_THREADS) v.slot_of[v.copy_id[c]] = v.copy_slot[c];
  __syncthreads();
  for (int i = tid; i < a.n_adapters; i += PD_THREADS)
    if (needed[i]) v.last_used[v.slot_of[i]] = step;
  // pointer tables of the paged-in adapters
  for (int w = tid; w < nmiss * a.ntab; w += PD_THREADS) {
    const int c = w / a.ntab, t = w - c * a.ntab;
    const int id = v.copy_id[c], s = v.copy_slot[c];
    reinterpret_cast<void**>(a.tables[t])[id] = a.pool + (size_t)s * a.adapter_bytes + a.offsets[t];
  }
  if (tid == 0) {
    v.h->n_copy = nmiss;
    v.h->step = step;
    v.h->copies += (unsigned long long)nmiss;
  }
}

// It never signals its dependents early: the SGMM kernels may read adapter weights (and the
// pointer tables) before their own dependency wait, so nothing after this kernel may start
// before its copies are complete.
__global__ void __launch_bounds__(256) pool_copy_kernel(const __grid_constant__ PoolArgs a) {
  pdl_wait();                                        // the decisions, and the slots' last readers
  PoolView v = pool_view(a.state, a.n_adapters, a.n_slots);
  const int n = v.h->n_copy;
  const size_t chunks = a.adapter_bytes / 16;
  const size_t total = (size_t)n * chunks;
  for (size_t w = (size_t)blockIdx.x * blockDim.x + threadIdx.x; w < total; w += (size_t)gridDim.x * blockDim.x) {
    const size_t c = w / chunks, o = w - c * chunks;
    const uint4* src = reinterpret_cast<const uint4*>(a.host_src[v.copy_id[c]]);
    uint4* dst = reinterpret_cast<uint4*>(a.pool + (size_t)v.copy_slot[c] * a.adapter_bytes);
    dst[o] = src[o];
  }
}

// ---------------------------------------------------------------- host side

size_t adapter_pool_state_bytes(int n_adapters, int n_slots) { return pool_state_bytes(n_adapters, n_slots); }

cudaError_t launch_pool_init(void* state, int n_adapters, int n_slots, void* pool, size_t pool_bytes,
                             const unsigned long long* offsets, void* const* tables, int ntab, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(pool, 0, pool_bytes, s);
  if (err != cudaSuccess) return err;
  count_launch();
  pool_init_kernel<<<4, PD_THREADS, 0, s>>>(state, n_adapters, n_slots, reinterpret_cast<char*>(pool), offsets,
                                            tables, ntab);
  return cudaGetLastError();
}

cudaError_t launch_pool_page_in(void* state, int n_adapters, int n_slots, const int32_t* idx, int nq,
                                const void* const* host_src, size_t adapter_bytes, void* pool,
                                const unsigned long long* offsets, void* const* tables, int ntab, void* ws,
                                cudaStream_t s) {
  PoolArgs a;
  a.state = state;
  a.n_adapters = n_adapters;
  a.n_slots = n_slots;
  a.idx = idx;
  a.nq = nq;
  a.host_src = host_src;
  a.adapter_bytes = adapter_bytes;
  a.pool = reinterpret_cast<char*>(pool);
  a.offsets = offsets;
  a.tables = tables;
  a.ntab = ntab;
  a.ws = ws;
  const size_t smem = sizeof(int) * ((size_t)n_adapters + (size_t)n_slots);
  static SmemLimit lim;
  cudaError_t err;
  if ((err = lim.ensure((const void*)pool_decide_kernel, smem)) != cudaSuccess) return err;
  if ((err = launch_pdl(pool_decide_kernel, dim3(1), dim3(PD_THREADS), smem, s, a)) != cudaSuccess) return err;
  return launch_pdl(pool_copy_kernel, dim3(2 * device_sm_count()), dim3(256), 0, s, a);
}

}  // namespace apr
