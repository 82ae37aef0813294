// Tile layout of the tensor-core decode kernel: where each visible row of one
// (batch entry, kv head) pair lands in the shared-memory tiles.
//
// The pair's visible rows come in runs, in visiting order: the pinned prefix
// rows [0, P), the ring window as at most two slot runs split at the physical
// wrap, and its newest row, position t, as a run of its own -- in a decode
// step that row is the appended token, read from the caller's buffer instead
// of its ring slot.  The rows are placed in a padded row space cut into 8-row
// atoms (a 128-byte-swizzle atom is 8 rows of 128 bytes; tensor-map copies
// land on atom boundaries): every run starts a new atom, and a prefix or ring
// row sits at the offset within its atom that its row or slot has modulo 8,
// so a copy of whole atoms starting at the 8-aligned row or slot below a
// piece brings it into place (the rows before and after it are padding,
// masked by the kernel).  A paged ring is cut into one piece per page; with
// pages a multiple of 8 rows every page edge falls on an atom boundary and
// the layout is the unpaged one, so paged and unpaged caches compute
// bit-identical results.  Smaller pages each start a new atom.  Tile j of the
// pair holds padded rows [j TR, (j + 1) TR).  No row outside the visible set
// is a valid row of any tile ("Prefix Sliding" digest, section 06: the prefix
// range and the window range are walked separately and the evicted middle is
// never visited).
//
// Chunk mode (a small block of queries routed off the 128-row tensor-core
// tile): a pair is one group of up to 8 consecutive queries of the block and
// one kv head; its runs are the union of the group's visible sets -- the
// prefix, the ring window of its first query, and the block's own rows (read
// from the caller's buffer) -- and a per-row query mask (dec_row_queries)
// cuts that union back to each query's set.
//
// Host-callable, so that the layout can be checked on the CPU.
#pragma once
#include <stdint.h>

#include "common.cuh"

namespace ps {

constexpr int32_t kPadRows = 8;

__host__ __device__ __forceinline__ int32_t pad8(int32_t x) { return (x + 7) & ~7; }

enum : int32_t {
  RUN_PREFIX = 0,  // prefix rows of the owner's slab, row0 = first prefix row
  RUN_RING = 1,    // ring slots of the sequence, row0 = first slot
  RUN_NEW = 2,     // the appended token (decode step), from the caller's buffer
  RUN_BLK = 3,     // chunk mode: rows of the caller's block, row0 = first block row
};

struct DecRuns {
  int32_t n;
  int32_t src[4];
  int32_t row0[4];    // first prefix row / ring slot of the run
  int32_t len[4];
  int32_t pstart[4];  // padded row of the run's first row
  int32_t padded;     // padded rows of the pair (a multiple of 8)
  int32_t rows;       // valid rows of the pair
  int32_t page;       // ring page rows of a paged cache, 0 when unpaged
  int32_t plg;        // log2(page) for a power-of-two page, else -1 (divisions)
  int32_t ring_ok;    // 0 if the window reaches below what the ring holds
  // chunk mode (dec_runs_chunk; a plain decode leaves qb0 = qd0 = qd1 = 0 and
  // no tile is query-dependent): the group's queries are at t0 + qi0 + k,
  // k < qnq; qlo = t0 + qi0 - W + 1; ring slot s holds position
  // rbase + (s - rhead) mod W.  Padded rows [qd0, qd1) and [qb0, padded) may
  // hold rows that not every query of the group sees.
  int64_t qlo, rbase;
  int32_t qi0, qnq, qW, rhead;
  int32_t qd0, qd1, qb0;
};

// log2 of a power-of-two page size, -1 otherwise; x mod page and x / page
// with shifts when it is one (the common sizes), divisions otherwise.
__host__ __device__ __forceinline__ int32_t page_log2(int32_t page) {
  if (page <= 0 || (page & (page - 1))) return -1;
#ifdef __CUDA_ARCH__
  return __ffs(page) - 1;
#else
  return __builtin_ctz((unsigned)page);
#endif
}
__host__ __device__ __forceinline__ int32_t pg_mod(int32_t x, int32_t page, int32_t lg) {
  return lg >= 0 ? (x & (page - 1)) : x % page;
}
__host__ __device__ __forceinline__ int32_t pg_div(int32_t x, int32_t page, int32_t lg) {
  return lg >= 0 ? (x >> lg) : x / page;
}

// Pages whose edges fall on atom boundaries keep the unpaged layout.
__host__ __device__ __forceinline__ bool page_aligned(int32_t page) {
  return page <= 0 || page % kPadRows == 0;
}

// Padded rows of a ring run of n slots from slot s placed from an atom
// boundary: one stretch at offset s mod 8, or for small pages one atom-started
// stretch per page.
__host__ __device__ __forceinline__ int32_t ring_run_padded(int32_t s, int32_t n, int32_t page) {
  if (page_aligned(page)) return pad8(s % kPadRows + n);
  int32_t f = page - s % page;
  if (f > n) f = n;
  const int32_t rest = n - f;
  const int32_t last = rest % page;
  return pad8(f) + (rest / page) * pad8(page) + (last ? pad8(last) : 0);
}

// Runs of the decode query at t = next_pos - 1, with m the ring state the
// query sees (in a decode step: the state after the append, whose token at
// position t is the RUN_NEW run).  Visible set (digest section 03, 0-indexed):
// the prefix [0, P) and the window [max(P, t - W + 1), t], which the ring holds
// as at most two slot runs split at the physical wrap.  Everything is computed
// in scalars and stored at constant indices, so that in device code the runs
// stay in registers.
__host__ __device__ __forceinline__ DecRuns dec_runs(const DevMeta& m, int32_t W, int64_t t,
                                                     int32_t page, bool step) {
  DecRuns r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.src[i] = 0; r.row0[i] = 0; r.len[i] = 0; r.pstart[i] = 0;
  }
  r.page = page;
  r.plg = page_log2(page);
  r.ring_ok = 1;
  // the window part: positions [lo, hi] of the ring, oldest at slot `head`
  const int64_t base = m.next_pos - m.count;
  int64_t lo = t - (int64_t)W + 1;
  if (lo < m.P) lo = m.P;
  const int64_t hi = t < m.next_pos - 1 ? t : m.next_pos - 1;
  int32_t s0 = 0, lenA = 0, lenB = 0;
  if (hi >= lo) {
    if (lo < base) {  // the window reaches below what the ring holds
      r.ring_ok = 0;
      lo = base;
    }
    if (hi >= lo) {
      const int64_t nw = hi - lo + 1;
      s0 = m.head + (int32_t)(lo - base);  // head < W and lo - base < W: one wrap at most
      if (s0 >= W) s0 -= W;
      lenA = (int32_t)(nw < (int64_t)(W - s0) ? nw : (int64_t)(W - s0));
      lenB = (int32_t)(nw - lenA);
    }
  }
  // The window's last row (position t, the last ring slot) always forms a
  // run of its own, after the others: in a decode step it is the appended
  // token, read from the caller's buffer; in a plain decode it is read from its
  // ring slot.  So a step and an append followed by a plain decode lay out
  // their tiles identically, and compute bit-identical results.
  const bool newest = lenA + lenB > 0;
  int32_t last_slot = 0;
  if (newest) {
    if (lenB > 0) {
      last_slot = lenB - 1;
      --lenB;
    } else {
      last_slot = s0 + lenA - 1;
      --lenA;
    }
  }
  r.qlo = 0; r.rbase = 0; r.qi0 = 0; r.qnq = 1; r.qW = W; r.rhead = 0;
  r.qd0 = 0; r.qd1 = 0; r.qb0 = 0;
  int32_t n = 0, padded = 0, rows = 0;
  auto add = [&](int32_t src, int32_t row0, int32_t len, int32_t pre, int32_t padlen) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k == n) {
        r.src[k] = src;
        r.row0[k] = row0;
        r.len[k] = len;
        r.pstart[k] = padded + pre;
      }
    }
    ++n;
    padded += padlen;
    rows += len;
  };
  if (m.P > 0) add(RUN_PREFIX, 0, m.P, 0, pad8(m.P));
  const bool al = page_aligned(page);
  if (lenA > 0) add(RUN_RING, s0, lenA, al ? s0 % kPadRows : 0, ring_run_padded(s0, lenA, page));
  if (lenB > 0) add(RUN_RING, 0, lenB, 0, ring_run_padded(0, lenB, page));
  if (newest) add(step ? RUN_NEW : RUN_RING, step ? 0 : last_slot, 1, 0, kPadRows);
  r.n = n;
  r.padded = padded;
  r.rows = rows;
  r.qb0 = padded;
  return r;
}

// Runs of a chunk-mode pair: the group of nq (1..8) queries at positions
// t0 + i0 + k of a block whose rows j sit at positions t0 + j in the caller's
// buffer, with m the ring state before the block (next_pos == t0).  Query i
// of the block sees (digest section 03, 0-indexed) the prefix [0, P), the ring
// rows at positions >= max(P, t0 + i - W + 1), and the block rows j with
// i - W + 1 <= j <= i.  The runs hold the union over the group: the prefix,
// the ring window of its first query as at most two slot runs, and block rows
// [max(0, i0 - W + 1), i0 + nq) as one run from an atom boundary.
__host__ __device__ __forceinline__ DecRuns dec_runs_chunk(const DevMeta& m, int32_t W, int64_t t0,
                                                           int32_t i0, int32_t nq, int32_t page) {
  DecRuns r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.src[i] = 0; r.row0[i] = 0; r.len[i] = 0; r.pstart[i] = 0;
  }
  r.page = page;
  r.plg = page_log2(page);
  r.ring_ok = 1;
  const int64_t base = m.next_pos - m.count;
  const int64_t qlo = t0 + i0 - (int64_t)W + 1;
  int64_t lo = qlo < m.P ? (int64_t)m.P : qlo;
  const int64_t hi = m.next_pos - 1;
  int32_t s0 = 0, lenA = 0, lenB = 0;
  if (hi >= lo) {
    if (lo < base) {
      r.ring_ok = 0;
      lo = base;
    }
    if (hi >= lo) {
      const int64_t nw = hi - lo + 1;
      s0 = m.head + (int32_t)(lo - base);
      if (s0 >= W) s0 -= W;
      lenA = (int32_t)(nw < (int64_t)(W - s0) ? nw : (int64_t)(W - s0));
      lenB = (int32_t)(nw - lenA);
    }
  }
  const int32_t jlo = i0 - W + 1 > 0 ? i0 - W + 1 : 0;
  const int32_t nblk = i0 + nq - jlo;
  int32_t n = 0, padded = 0, rows = 0;
  int32_t pA = 0, pB = 0;
  auto add = [&](int32_t src, int32_t row0, int32_t len, int32_t pre, int32_t padlen) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k == n) {
        r.src[k] = src;
        r.row0[k] = row0;
        r.len[k] = len;
        r.pstart[k] = padded + pre;
      }
    }
    ++n;
    padded += padlen;
    rows += len;
  };
  if (m.P > 0) add(RUN_PREFIX, 0, m.P, 0, pad8(m.P));
  const bool al = page_aligned(page);
  pA = padded;
  if (lenA > 0) add(RUN_RING, s0, lenA, al ? s0 % kPadRows : 0, ring_run_padded(s0, lenA, page));
  pB = padded;
  if (lenB > 0) add(RUN_RING, 0, lenB, 0, ring_run_padded(0, lenB, page));
  const int32_t pK = padded;
  add(RUN_BLK, jlo, nblk, 0, pad8(nblk));
  r.n = n;
  r.padded = padded;
  r.rows = rows;
  r.qlo = qlo;
  r.rbase = base;
  r.qi0 = i0;
  r.qnq = nq;
  r.qW = W;
  r.rhead = m.head;
  // Ring rows whose visibility differs within the group: positions
  // [lo, qlo + nq - 1), the window's first rows (run A, then run B).
  int64_t dep = qlo + nq - 1 - lo;
  if (dep < 0) dep = 0;
  if (dep > (int64_t)lenA + lenB) dep = (int64_t)lenA + lenB;
  r.qd0 = pA;
  r.qd1 = pA;
  if (dep > 0) {
    if (dep <= lenA) {
      r.qd1 = pA + ring_run_padded(s0, (int32_t)dep, page);
    } else {
      r.qd1 = pB + ring_run_padded(0, (int32_t)(dep - lenA), page);
    }
  }
  // Block rows: j > i0 (causal inside the block), and with a window shorter
  // than the group, j < i0 + nq - W.
  const int32_t jd = i0 + nq - W > jlo ? jlo : i0 + 1;
  r.qb0 = pK + (jd - jlo);
  return r;
}

// Queries of a chunk-mode group (bit k: query t0 + qi0 + k) that see the row
// `row` of a run of source src (prefix row, ring slot, or block row).
__host__ __device__ __forceinline__ uint32_t dec_row_queries(const DecRuns& r, int32_t src,
                                                             int32_t row) {
  int64_t lo_k = 0, hi_k = 7;  // queries k in [lo_k, hi_k] see the row
  if (src == RUN_RING) {
    int32_t off = row - r.rhead;
    if (off < 0) off += r.qW;
    hi_k = r.rbase + off - r.qlo;  // position >= qlo + k
  } else if (src == RUN_BLK) {
    const int32_t d = row - r.qi0;  // block row j <= i0 + k and j >= i0 + k - W + 1
    lo_k = d;
    hi_k = (int64_t)d + r.qW - 1;
  }
  if (lo_k < 0) lo_k = 0;
  if (hi_k > 7) hi_k = 7;
  if (hi_k < lo_k) return 0u;
  return ((2u << hi_k) - 1u) & ~((1u << lo_k) - 1u);
}

// True if the tile of padded rows [x0, x1) may hold a row that not every query
// of a chunk-mode group sees (never in a plain decode or a decode step).
__host__ __device__ __forceinline__ bool dec_tile_qdep(const DecRuns& r, int32_t x0, int32_t x1) {
  return (x0 < r.qd1 && x1 > r.qd0) || x1 > r.qb0;
}

__host__ __device__ __forceinline__ int32_t dec_tiles(const DecRuns& r, int32_t TR) {
  return (r.padded + TR - 1) / TR;
}

// True if the tile of padded rows [x0, x1) (x0 a multiple of 8) is a single
// whole piece: x1 - x0 == TR valid rows of one prefix or ring run (inside one
// page) from tile row 0.  Then *src is its source and *row its first prefix
// row or ring slot (a multiple of 8, since row and tile row agree modulo 8).
__host__ __device__ __forceinline__ bool dec_range_whole(const DecRuns& r, int32_t TR, int32_t x0,
                                                         int32_t x1, int32_t* src, int32_t* row) {
  bool whole = false;
  if (x1 - x0 != TR) return false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k < r.n && r.src[k] <= RUN_RING && x0 >= r.pstart[k] &&
        x0 + TR <= r.pstart[k] + r.len[k]) {
      const int32_t rw = r.row0[k] + (x0 - r.pstart[k]);
      const int32_t pg = r.src[k] == RUN_RING ? r.page : 0;
      if (pg <= 0 || pg_mod(rw, pg, r.plg) + TR <= pg) {
        whole = true;
        *src = r.src[k];
        *row = rw;
      }
    }
  }
  return whole;
}

// Calls f(src, row, smem_row, n) for the pieces of the tile of padded rows
// [x0, x1) (x0 a multiple of 8, x1 - x0 <= TR): n valid rows starting at
// prefix row / ring slot `row` (RUN_NEW: row 0), placed at tile row smem_row.  The atoms [smem_row & ~7, pad8(smem_row + n)) of a piece hold
// no row of any other piece; a copy of them starts at row or slot
// row - (smem_row & 7), which lies in the same page as `row`.  A ring piece
// never crosses the physical wrap or a page edge.  (The runs are visited with
// constant indices so that, in device code, everything stays in registers.)
template <typename F>
__host__ __device__ __forceinline__ void dec_range_pieces(const DecRuns& r, int32_t x0, int32_t x1,
                                                          F&& f) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k >= r.n) continue;
    const int32_t src = r.src[k], ps = r.pstart[k], len = r.len[k], row0 = r.row0[k];
    const int32_t pg = src == RUN_RING ? r.page : 0;
    if (page_aligned(pg)) {
      const int32_t a = x0 > ps ? x0 : ps;
      const int32_t b = x1 < ps + len ? x1 : ps + len;
      int32_t row = row0 + (a - ps);
      for (int32_t x = a; x < b;) {  // one piece, or one per page edge crossed
        int32_t n = b - x;
        if (pg > 0) {
          const int32_t to_edge = pg - pg_mod(row, pg, r.plg);
          if (n > to_edge) n = to_edge;
        }
        f(src, row, x - x0, n);
        x += n;
        row += n;
      }
    } else {
      // small pages: the first (partial) page, then page after page, each
      // from its own atom
      const int32_t f0 = pg - pg_mod(row0, pg, r.plg);
      const int32_t first = f0 < len ? f0 : len;
      const int32_t step = pad8(pg);
      int32_t pos = ps, row = row0, n = first;
      if (x0 > ps + pad8(first)) {  // jump over the pages that end before the tile
        const int32_t skip = (x0 - ps - pad8(first)) / step;
        pos = ps + pad8(first) + skip * step;
        row = row0 + first + skip * pg;
        n = len - (row - row0) < pg ? len - (row - row0) : pg;
      }
      while (row - row0 < len && pos < x1) {
        const int32_t lo = x0 > pos ? x0 : pos;
        const int32_t hi = x1 < pos + n ? x1 : pos + n;
        if (hi > lo) f(src, row + (lo - pos), lo - x0, hi - lo);
        pos += pad8(n);
        row += n;
        n = len - (row - row0) < pg ? len - (row - row0) : pg;
      }
    }
  }
}

// Tile j of the pair: padded rows [j TR, (j + 1) TR).
__host__ __device__ __forceinline__ bool dec_tile_whole(const DecRuns& r, int32_t TR, int32_t j,
                                                        int32_t* src, int32_t* row) {
  return dec_range_whole(r, TR, j * TR, j * TR + TR, src, row);
}
template <typename F>
__host__ __device__ __forceinline__ void dec_tile_pieces(const DecRuns& r, int32_t TR, int32_t j,
                                                         F&& f) {
  dec_range_pieces(r, j * TR, j * TR + TR, f);
}

// Cluster split: the padded rows [*x0, *x1) of CTA `rank` of `csize` that
// share one pair -- equal shares to within 8 rows, each starting on an atom.
__host__ __device__ __forceinline__ void dec_cluster_share(const DecRuns& r, int rank, int csize,
                                                           int32_t* x0, int32_t* x1) {
  *x0 = (int32_t)(((int64_t)r.padded * rank / csize) & ~(int64_t)(kPadRows - 1));
  *x1 = rank + 1 == csize
            ? r.padded
            : (int32_t)(((int64_t)r.padded * (rank + 1) / csize) & ~(int64_t)(kPadRows - 1));
}

}  // namespace ps
