// Ring-buffer KV store: prefix store (a1), ring append with eviction and
// position bookkeeping (a2), window import/export and the visible-row dump.
//
// Cache update rule ("Formal verification of a sliding-window KV cache in
// Lean4", pnsm.cn blog, sections 3.3-3.4): a new entry fills slot
// (head + count) mod W while fewer than W entries are held, otherwise it
// overwrites the oldest slot `head` and head advances by one.  Over n tokens
// that is count' = min(W, count + n), head' = head + max(0, count + n - W)
// (mod W), and position p always lands in slot (head + p - base) mod W with
// base = next_pos - count the oldest held position.
#include "internal.h"
#include "sm100_ptx.cuh"

namespace ps {

namespace {

constexpr int kThreads = 256;

__global__ void k_meta_set(DevMeta* meta, int seq, DevMeta m) { meta[seq] = m; }

// Page-table updates of a paged cache: page_table[idx[i]] = phys[i].
struct PageSets {
  int32_t n;
  int32_t idx[kMaxPageSets];
  int32_t phys[kMaxPageSets];
};
__global__ void k_page_set(int32_t* page_table, PageSets u) {
  for (int i = threadIdx.x; i < u.n; i += blockDim.x) page_table[u.idx[i]] = u.phys[i];
}

// Prefix rows: input [P_s][Hkv][d] -> slab rows [0, P_s) of every head.
__global__ void k_prefix_store(CacheDev c, int vpr, int seq, const uint4* __restrict__ k,
                               const uint4* __restrict__ v, int P_s) {
  uint4* K = (uint4*)c.K;
  uint4* V = (uint4*)c.V;
  int64_t total = (int64_t)P_s * c.Hkv * vpr;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < total;
       x += (int64_t)gridDim.x * blockDim.x) {
    int vi = (int)(x % vpr);
    int64_t r = x / vpr;
    int g = (int)(r % c.Hkv);
    int64_t j = r / c.Hkv;
    size_t dst = (size_t)prefix_row(c, seq, g, j) * vpr + vi;
    K[dst] = k[x];
    V[dst] = v[x];
  }
}

// Append n tokens to each batch entry (grid.y = batch entry).  Every CTA of an
// entry reads the entry's bookkeeping before arriving on the entry's ticket;
// the last CTA to arrive commits the new bookkeeping and re-arms the ticket.
__global__ void k_ring_append(CacheDev c, int vpr, BatchIds ids, const uint4* __restrict__ k,
                              const uint4* __restrict__ v, int n) {
  const int b = blockIdx.y;
  const int s = ids.seq[b];
  const DevMeta m = c.meta[s];
  const int64_t W = c.W;
  const int64_t n_eff = n < W ? n : W;       // earlier tokens are overwritten in this call
  const int64_t i0 = n - n_eff;
  const int64_t base = m.next_pos - m.count;
  uint4* K = (uint4*)c.K;
  uint4* V = (uint4*)c.V;
  const int64_t total = n_eff * c.Hkv * vpr;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < total;
       x += (int64_t)gridDim.x * blockDim.x) {
    int vi = (int)(x % vpr);
    int64_t r = x / vpr;
    int g = (int)(r % c.Hkv);
    int64_t i = i0 + r / c.Hkv;
    int64_t p = m.next_pos + i;
    const int32_t slot = (int32_t)(((int64_t)m.head + (p - base)) % W);
    const int phys = ring_page(c, s, slot);
    size_t src = (((size_t)b * n + i) * c.Hkv + g) * vpr + vi;
    size_t dst = (size_t)ring_row(c, phys, g, slot) * vpr + vi;
    K[dst] = k[src];
    V[dst] = v[src];
    if (g == 0 && vi == 0) c.pos[pos_index(c, phys, slot)] = p;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int old = atomicAdd(&c.tickets[s], 1);
    if (old == (int)gridDim.x - 1) {
      DevMeta nm = m;
      int64_t cn = (int64_t)m.count + n;
      nm.count = (int32_t)(cn < W ? cn : W);
      int64_t adv = cn - W > 0 ? cn - W : 0;
      nm.head = (int32_t)(((int64_t)m.head + adv) % W);
      nm.next_pos = m.next_pos + n;
      c.meta[s] = nm;
      c.tickets[s] = 0;
    }
  }
}

// Import: rows i of [n][Hkv][d] hold positions next_pos - n + i, oldest at slot head.
__global__ void k_ring_import(CacheDev c, int vpr, int seq, DevMeta mn,
                              const uint4* __restrict__ k, const uint4* __restrict__ v, int n) {
  uint4* K = (uint4*)c.K;
  uint4* V = (uint4*)c.V;
  const int64_t W = c.W;
  const int64_t total = (int64_t)n * c.Hkv * vpr;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < total;
       x += (int64_t)gridDim.x * blockDim.x) {
    int vi = (int)(x % vpr);
    int64_t r = x / vpr;
    int g = (int)(r % c.Hkv);
    int64_t i = r / c.Hkv;
    const int32_t slot = (int32_t)(((int64_t)mn.head + i) % W);
    const int phys = ring_page(c, seq, slot);
    size_t dst = (size_t)ring_row(c, phys, g, slot) * vpr + vi;
    K[dst] = k[x];
    V[dst] = v[x];
    if (g == 0 && vi == 0) c.pos[pos_index(c, phys, slot)] = mn.next_pos - n + i;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int old = atomicAdd(&c.tickets[seq], 1);
    if (old == (int)gridDim.x - 1) {
      c.meta[seq] = mn;
      c.tickets[seq] = 0;
    }
  }
}

// Export the held window in logical order: entry i is slot (head + i) mod W.
__global__ void k_ring_export(CacheDev c, int vpr, int seq, uint4* __restrict__ k,
                              uint4* __restrict__ v, int64_t* __restrict__ pos,
                              int32_t* __restrict__ count_out) {
  const DevMeta m = c.meta[seq];
  const uint4* K = (const uint4*)c.K;
  const uint4* V = (const uint4*)c.V;
  const int64_t total = (int64_t)m.count * c.Hkv * vpr;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < total;
       x += (int64_t)gridDim.x * blockDim.x) {
    int vi = (int)(x % vpr);
    int64_t r = x / vpr;
    int g = (int)(r % c.Hkv);
    int64_t i = r / c.Hkv;
    const int32_t slot = (int32_t)(((int64_t)m.head + i) % c.W);
    const int phys = ring_page(c, seq, slot);
    size_t src = (size_t)ring_row(c, phys, g, slot) * vpr + vi;
    k[x] = K[src];
    v[x] = V[src];
    if (g == 0 && vi == 0) pos[i] = c.pos[pos_index(c, phys, slot)];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *count_out = m.count;
}

// The rows the attention kernels visit for a query at t, as positions.
__global__ void k_debug_visible(CacheDev c, int seq, int64_t t, int64_t* __restrict__ pos_out,
                                int32_t* __restrict__ n_out) {
  const DevMeta m = c.meta[seq];
  const SegSet s = build_segments(m, c.W, t);
  if (!s.ring_ok && threadIdx.x == 0) atomicOr(c.err, ERR_RING);
  int32_t j0 = 0;
  for (int i = 0; i < s.n; ++i) {
    for (int32_t r = threadIdx.x; r < s.len[i]; r += blockDim.x) {
      int64_t p;
      if (s.src[i] == 0) {
        p = s.row0[i] + r;  // prefix row j holds position j
      } else if (s.src[i] == 1) {
        const int32_t slot = (int32_t)(s.row0[i] + r);
        p = c.pos[pos_index(c, ring_page(c, seq, slot), slot)];
      } else {
        p = m.next_pos + s.row0[i] + r;
      }
      pos_out[j0 + r] = p;
    }
    j0 += s.len[i];
  }
  if (threadIdx.x == 0) *n_out = s.total;
}

// Test hook for the bounded waits every pipeline uses: one thread waits on an
// mbarrier that nothing ever arrives at, with the same helper and a short limit,
// and reports the time-out in the error word as the kernels do.
__global__ void k_debug_wait_timeout(CacheDev c, long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
    if (!ptx::mbar_wait_bounded(&bar, 0, &abort_flag, limit_cycles)) atomicOr(c.err, ERR_TIMEOUT);
  }
}

int grid_for(int64_t work, int cap) {
  int64_t g = (work + kThreads - 1) / kThreads;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return (int)g;
}

}  // namespace

cudaError_t launch_page_set(const CacheDev& c, const int32_t* idx, const int32_t* phys, int n,
                            cudaStream_t st) {
  for (int i0 = 0; i0 < n; i0 += kMaxPageSets) {
    PageSets u;
    u.n = n - i0 < kMaxPageSets ? n - i0 : kMaxPageSets;
    for (int i = 0; i < u.n; ++i) {
      u.idx[i] = idx[i0 + i];
      u.phys[i] = phys[i0 + i];
    }
    k_page_set<<<1, 256, 0, st>>>(c.page_table, u);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_meta_set(const CacheDev& c, int seq, const DevMeta& m, cudaStream_t st) {
  k_meta_set<<<1, 1, 0, st>>>(c.meta, seq, m);
  return cudaGetLastError();
}

cudaError_t launch_prefix_store(const CacheDev& c, int esize, int seq, const void* k,
                                const void* v, int P_s, cudaStream_t st) {
  int vpr = c.d * esize / 16;
  int64_t work = (int64_t)P_s * c.Hkv * vpr;
  if (work == 0) return cudaSuccess;
  k_prefix_store<<<grid_for(work, 4096), kThreads, 0, st>>>(c, vpr, seq, (const uint4*)k,
                                                            (const uint4*)v, P_s);
  return cudaGetLastError();
}

cudaError_t launch_ring_append(const CacheDev& c, int esize, const BatchIds& ids, int B,
                               const void* k, const void* v, int n, cudaStream_t st) {
  int vpr = c.d * esize / 16;
  int64_t n_eff = n < c.W ? n : c.W;
  int64_t work = n_eff * c.Hkv * vpr;
  dim3 grid(grid_for(work, 256), B);
  k_ring_append<<<grid, kThreads, 0, st>>>(c, vpr, ids, (const uint4*)k, (const uint4*)v, n);
  return cudaGetLastError();
}

cudaError_t launch_ring_import(const CacheDev& c, int esize, int seq, const DevMeta& m_new,
                               const void* k, const void* v, int n, cudaStream_t st) {
  int vpr = c.d * esize / 16;
  int64_t work = (int64_t)n * c.Hkv * vpr;
  k_ring_import<<<grid_for(work, 1024), kThreads, 0, st>>>(c, vpr, seq, m_new, (const uint4*)k,
                                                           (const uint4*)v, n);
  return cudaGetLastError();
}

cudaError_t launch_ring_export(const CacheDev& c, int esize, int seq, void* k, void* v,
                               int64_t* pos, int32_t* count_out, cudaStream_t st) {
  int vpr = c.d * esize / 16;
  int64_t work = (int64_t)c.W * c.Hkv * vpr;
  k_ring_export<<<grid_for(work, 1024), kThreads, 0, st>>>(c, vpr, seq, (uint4*)k, (uint4*)v,
                                                           pos, count_out);
  return cudaGetLastError();
}

cudaError_t launch_debug_visible(const CacheDev& c, int seq, int64_t t, int64_t* pos_out,
                                 int32_t* n_out, cudaStream_t st) {
  k_debug_visible<<<1, kThreads, 0, st>>>(c, seq, t, pos_out, n_out);
  return cudaGetLastError();
}

cudaError_t launch_debug_wait_timeout(const CacheDev& c, long long limit_cycles, cudaStream_t st) {
  k_debug_wait_timeout<<<1, 32, 0, st>>>(c, limit_cycles);
  return cudaGetLastError();
}

}  // namespace ps
