// Shared device-side definitions: cache layout, per-sequence bookkeeping and
// the derivation of the visible row ranges (the part of the path that turns a
// query position into the rows to stream, never addressing evicted rows).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace ps {

// Per-sequence bookkeeping kept in device memory (32 bytes).
//   The ring holds positions [next_pos - count, next_pos); the oldest sits in
//   slot `head`, position p in slot (head + (p - (next_pos - count))) mod W.
//   P is the pinned prefix length; prefix row j holds position j.
struct DevMeta {
  int64_t next_pos;
  int32_t P;
  int32_t head;
  int32_t count;
  int32_t owner;  // sequence whose slab holds the pinned prefix rows (itself unless shared)
  int32_t pad[2];
};
static_assert(sizeof(DevMeta) == 32, "DevMeta layout");

// Device view of one cache, passed to kernels by value.  Rows are d elements.
//   Prefix row j of (sequence, kv head g): K/V row prefix_row(seq, g, j).
//   Ring slot s of a sequence lives in ring page s / page_rows of that
//   sequence, at physical page phys = page_table[seq][s / page_rows] (the
//   sequence itself when page_table is NULL), row ring_row(phys, g, s).
//   An unpaged cache is the case page_rows = W with one page per sequence
//   inside its own slab [Hkv][P_max + W] (prefix rows, then ring rows); a paged
//   cache keeps its ring pages [nphys][Hkv][page_rows] in a pool after the
//   prefix slabs [S][Hkv][P_max] and maps them through page_table (the
//   block-table indirection of a paged cache).
//   pos[pos_index(phys, s)]: absolute position held by each ring slot.
struct CacheDev {
  DevMeta* meta;
  int32_t* tickets;     // [S] completion counters of the ring writers (0 at rest)
  int32_t* err;         // device error word (bit flags below)
  int64_t* pos;
  void* K;
  void* V;
  int32_t* page_table;  // [S][npg] physical page of each ring page; NULL: unpaged
  int32_t W, P_max, Hkv, d, S;
  int32_t page_rows;    // ring slots per page (W when unpaged)
  int32_t npg;          // ring pages per sequence (W / page_rows)
  int32_t nphys;        // physical ring pages (S when unpaged)
  int64_t pstride;      // rows from one (sequence, head) prefix slab to the next
  int64_t rstride;      // rows from one (page, head) ring slab to the next
  int64_t rbase;        // row of slot 0 of (page 0, head 0)
};

__host__ __device__ inline int64_t prefix_row(const CacheDev& c, int seq, int g, int64_t j) {
  return ((int64_t)seq * c.Hkv + g) * c.pstride + j;
}
// Ring slots lie in [0, W), so slot arithmetic is 32-bit; an unpaged cache
// (page_rows = W) needs no division at all.
__host__ __device__ inline int64_t ring_row(const CacheDev& c, int phys, int g, int32_t slot) {
  const int32_t in_page = c.page_table ? slot % c.page_rows : slot;
  return c.rbase + ((int64_t)phys * c.Hkv + g) * c.rstride + in_page;
}
__host__ __device__ inline int64_t pos_index(const CacheDev& c, int phys, int32_t slot) {
  const int32_t in_page = c.page_table ? slot % c.page_rows : slot;
  return (int64_t)phys * c.page_rows + in_page;
}
#ifdef __CUDACC__
// Physical page holding ring slot `slot` of sequence `seq` (a table read only
// for a paged cache).
__device__ __forceinline__ int ring_page(const CacheDev& c, int seq, int32_t slot) {
  return c.page_table ? c.page_table[(int64_t)seq * c.npg + slot / c.page_rows] : seq;
}
#endif

enum : int32_t {
  ERR_RING = 2,      // the ring does not hold the window a query needs
  ERR_BATCH = 4,     // a batch entry's position disagrees with the bookkeeping
  ERR_TIMEOUT = 8,   // a pipeline wait gave up (the kernel stopped early)
};

// Row ranges a query at position t reads, in visiting order (at most 4):
//   src 0: prefix rows [0, P) (row0 = 0);
//   src 1: ring segment from slot s0 up to the physical end of the ring (row0 = s0);
//   src 1: ring segment wrapping around from slot 0 (row0 = 0);
//   src 2: block rows (chunk queries): block row r holds position next_pos + r.
// Visible set (digest section 03, 0-indexed): [0, P) and [max(P, t-W+1), t].
struct SegSet {
  int32_t n;
  int32_t total;
  int32_t len[4];
  int64_t row0[4];  // first prefix row (src 0), ring slot (src 1) or block row (src 2)
  int32_t src[4];
  int32_t ring_ok;  // 0 if the window part below next_pos is not held by the ring
};

__host__ __device__ inline SegSet build_segments(const DevMeta& m, int32_t W, int64_t t) {
  SegSet s;
  s.n = 0;
  s.total = 0;
  s.ring_ok = 1;
  for (int i = 0; i < 4; ++i) { s.len[i] = 0; s.row0[i] = 0; s.src[i] = 0; }
  if (m.P > 0) {
    s.len[0] = m.P; s.row0[0] = 0; s.src[0] = 0; s.n = 1;
  }
  int64_t lo = t - (int64_t)W + 1;
  if (lo < m.P) lo = m.P;
  // ring part: positions [lo, min(t, next_pos - 1)]
  int64_t hi = t < m.next_pos - 1 ? t : m.next_pos - 1;
  int64_t base = m.next_pos - m.count;
  if (hi >= lo) {
    if (lo < base) {  // window reaches below what the ring holds
      s.ring_ok = 0;
      lo = base;
    }
    if (hi >= lo) {
      int64_t nw = hi - lo + 1;
      int64_t s0 = ((int64_t)m.head + (lo - base)) % W;
      int64_t lenA = nw < (int64_t)W - s0 ? nw : (int64_t)W - s0;
      s.len[s.n] = (int32_t)lenA; s.row0[s.n] = s0; s.src[s.n] = 1; s.n++;
      if (nw > lenA) {
        s.len[s.n] = (int32_t)(nw - lenA); s.row0[s.n] = 0; s.src[s.n] = 1; s.n++;
      }
    }
  }
  // block part: positions [max(lo, next_pos), t]
  int64_t blo = lo > m.next_pos ? lo : m.next_pos;
  if (t >= blo) {
    s.len[s.n] = (int32_t)(t - blo + 1); s.row0[s.n] = blo - m.next_pos; s.src[s.n] = 2; s.n++;
  }
  for (int i = 0; i < s.n; ++i) s.total += s.len[i];
  return s;
}

// Segment index and offset of logical row j (0 <= j < total).
__device__ __forceinline__ void seg_locate(const SegSet& s, int32_t j, int& si, int32_t& off) {
  si = 0;
  off = j;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    if (si == i && i + 1 < s.n && off >= s.len[i]) { off -= s.len[i]; si = i + 1; }
  }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// float -> bfloat16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f2bf(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

}  // namespace ps
