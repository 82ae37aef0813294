// Key-tile schedule of the tensor-core chunk kernel: which 128-row key tiles
// a query tile reads, in order (prefix rows, the ring window as at most two
// slot runs split at the physical wrap, then the block rows).  A ring run of
// a paged cache with pages of 128 rows or more is also cut at page edges.
// With smaller pages (8 to 64 rows, dividing 128) the run is tiled from the
// page edge at or below its first slot instead, so that every tile is whole
// pages; the rows before the run hold positions below KSched::rlo, which the
// kernel masks by position like the window's edge.  Host-callable so that it
// can be checked on the CPU.
#pragma once
#include <stdint.h>

#include "common.cuh"

namespace ps {

constexpr int kBN = 128;  // key rows per tile

// The key tiles of one query tile: up to 4 ranges, each tiled from its start;
// a ring range of a paged cache is also cut where it crosses into a new page
// (the first `first` rows, then 128-row tiles from that page boundary on).
struct KSched {
  int n;
  int ntiles;
  int64_t rlo;      // lowest position a ring or block tile presents as a key
  int src[4];       // 0: ring slot, 1: block row, 2: prefix row (owner's slab)
  int64_t row0[4];  // first ring slot / block row / prefix row of the range
  int64_t pos0[4];  // position of that row
  int32_t len[4];
  int32_t first[4];   // rows before the range's first page boundary (len if none)
  int32_t tfirst[4];  // tiles over those rows
  int32_t tbase[4];
};

struct KTile {
  int src;
  int64_t row, pos0;
  int valid;
};

// Pages smaller than a key tile (they divide it): ring tiles are whole pages.
__host__ __device__ __forceinline__ bool small_pages(int64_t page) { return page > 0 && page < kBN; }

// page: ring page size for a ring range of a paged cache (0: no page cuts)
__host__ __device__ __forceinline__ void add_range(KSched& s, int src, int64_t row0, int64_t pos0,
                                          int64_t len, int64_t page = 0) {
  if (len <= 0) return;
  if (small_pages(page)) {  // start at the page edge at or below row0 (a slot, below 2^28)
    const int32_t lead = (int32_t)row0 % (int32_t)page;
    row0 -= lead;
    pos0 -= lead;
    len += lead;
    page = 0;
  }
  int64_t first = len;
  if (page > 0) {  // a ring range: row0 is a slot, below 2^28
    const int64_t to_edge = page - (int32_t)row0 % (int32_t)page;
    first = to_edge < len ? to_edge : len;
  }
  const int32_t tfirst = (int32_t)((first + kBN - 1) / kBN);
  // stored through constant indices (a store at index s.n would put the
  // schedule in local memory instead of registers)
  auto put = [&](int k) {
    s.src[k] = src;
    s.row0[k] = row0;
    s.pos0[k] = pos0;
    s.len[k] = (int32_t)len;
    s.first[k] = (int32_t)first;
    s.tfirst[k] = tfirst;
    s.tbase[k] = s.ntiles;
  };
  if (s.n == 0) put(0);
  if (s.n == 1) put(1);
  if (s.n == 2) put(2);
  if (s.n == 3) put(3);
  s.ntiles += tfirst + (int32_t)((len - first + kBN - 1) / kBN);
  s.n++;
}

// Query positions [plo, phi]; the ring holds [next_pos - count, next_pos - 1] = [.., t0 - 1].
// Prompt queries (phi < P) read only the prefix rows [0, phi].
// page: ring page size of a paged cache (0 when unpaged).
__host__ __device__ __forceinline__ KSched make_sched(const DevMeta& m, int W, int page, int64_t t0,
                                             int64_t plo, int64_t phi, bool prompt) {
  KSched s;
  s.n = 0;
  s.ntiles = 0;
  s.rlo = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s.src[i] = 0; s.row0[i] = 0; s.pos0[i] = 0; s.len[i] = 0;
    s.first[i] = 0; s.tfirst[i] = 0; s.tbase[i] = 0;
  }
  if (prompt) {
    add_range(s, 2, 0, 0, phi + 1 < m.P ? phi + 1 : m.P);
    return s;
  }
  add_range(s, 2, 0, 0, m.P);  // pinned prefix
  int64_t lo = plo - W + 1;
  if (lo < m.P) lo = m.P;
  const int64_t base = m.next_pos - m.count;
  int64_t rlo = lo < base ? base : lo;  // never below what the ring holds
  s.rlo = rlo;  // block rows start at or above it too (base <= t0)
  if (t0 - 1 >= rlo) {
    const int64_t nw = t0 - rlo;
    int64_t s0 = (int64_t)m.head + (rlo - base);  // head < W, rlo - base < W: one wrap at most
    if (s0 >= W) s0 -= W;
    const int64_t lenA = nw < W - s0 ? nw : W - s0;
    add_range(s, 0, s0, rlo, lenA, page);
    add_range(s, 0, 0, rlo + lenA, nw - lenA, page);
  }
  const int64_t blo = lo > t0 ? lo : t0;
  add_range(s, 1, blo - t0, blo, phi - blo + 1);
  return s;
}

__host__ __device__ __forceinline__ KTile tile_of(const KSched& s, int j) {
  KTile t;
  t.src = s.src[0]; t.row = s.row0[0]; t.pos0 = s.pos0[0]; t.valid = 0;
  int k = 0;
#pragma unroll
  for (int q = 1; q < 4; ++q)
    if (q < s.n && j >= s.tbase[q]) k = q;
  int64_t off = 0, end = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q == k) {
      t.src = s.src[q];
      const int u = j - s.tbase[q];
      if (u < s.tfirst[q]) {  // before the range's first page boundary
        off = (int64_t)u * kBN;
        end = s.first[q];
      } else {
        off = s.first[q] + (int64_t)(u - s.tfirst[q]) * kBN;
        end = s.len[q];
      }
      t.row = s.row0[q] + off;
      t.pos0 = s.pos0[q] + off;
    }
  t.valid = (int)(end - off < kBN ? end - off : kBN);
  return t;
}

}  // namespace ps
