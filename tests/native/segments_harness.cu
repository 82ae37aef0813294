// Host-side harness for the library's visible-range derivation and cache
// addressing (prefix_sliding_window_ring_b200/csrc/common.cuh), compiled by
// the CPU tests and run without a GPU.  It prints, for each case read from
// stdin, the positions the derived row ranges visit, so the test can compare
// them with the oracle's visible set.
//
// Input lines:  seg P W head count next_pos t
//               addr S Hkv P_max W page_rows nphys   (prints the address checks)
#include <stdio.h>
#include <string.h>

#include <vector>

#include "common.cuh"

using ps::CacheDev;
using ps::DevMeta;
using ps::SegSet;

static void seg_case(int P, int W, int head, int count, long long next_pos, long long t) {
  DevMeta m;
  memset(&m, 0, sizeof(m));
  m.next_pos = next_pos;
  m.P = P;
  m.head = head;
  m.count = count;
  const SegSet s = ps::build_segments(m, W, t);
  const long long base = next_pos - count;
  printf("ok %d total %d :", s.ring_ok, s.total);
  for (int i = 0; i < s.n; ++i)
    for (int r = 0; r < s.len[i]; ++r) {
      long long p;
      if (s.src[i] == 0) p = s.row0[i] + r;                                // prefix row = position
      else if (s.src[i] == 1) p = base + ((s.row0[i] + r - head) % W + W) % W;  // ring slot
      else p = next_pos + s.row0[i] + r;                                   // block row
      printf(" %lld", p);
    }
  printf("\n");
}

// Every (sequence, head, prefix row) and (page, head, slot) maps to its own
// K/V row inside the cache, and every (page, slot) to its own position entry.
static void addr_case(int S, int Hkv, int P_max, int W, int page_rows, int nphys) {
  CacheDev c;
  memset(&c, 0, sizeof(c));
  c.W = W; c.P_max = P_max; c.Hkv = Hkv; c.S = S;
  const bool paged = page_rows > 0;
  int32_t dummy = 0;
  c.page_table = paged ? &dummy : nullptr;  // only tested for non-NULL by the helpers
  c.page_rows = paged ? page_rows : W;
  c.npg = paged ? W / page_rows : 1;
  c.nphys = paged ? nphys : S;
  c.pstride = paged ? P_max : (long long)P_max + W;
  c.rstride = paged ? page_rows : (long long)P_max + W;
  c.rbase = paged ? (long long)S * Hkv * P_max : P_max;
  const long long rows = paged ? (long long)S * Hkv * P_max + (long long)nphys * Hkv * page_rows
                               : (long long)S * Hkv * (P_max + W);
  std::vector<int> hit(rows, 0);
  long long bad = 0;
  for (int s = 0; s < S; ++s)
    for (int g = 0; g < Hkv; ++g)
      for (int j = 0; j < P_max; ++j) {
        const long long r = ps::prefix_row(c, s, g, j);
        if (r < 0 || r >= rows) ++bad; else ++hit[r];
      }
  std::vector<int> phit((long long)c.nphys * c.page_rows, 0);
  // a ring slot s of physical page ph: every slot of the page (s % page_rows)
  for (int ph = 0; ph < c.nphys; ++ph)
    for (int k = 0; k < c.page_rows; ++k) {
      const int slot = (paged ? (ph % c.npg) * c.page_rows : 0) + k;  // a slot that lands on row k
      for (int g = 0; g < Hkv; ++g) {
        const long long r = ps::ring_row(c, ph, g, slot);
        if (r < 0 || r >= rows) ++bad; else ++hit[r];
      }
      const long long pi = ps::pos_index(c, ph, slot);
      if (pi < 0 || pi >= (long long)phit.size()) ++bad; else ++phit[pi];
    }
  long long twice = 0, unused = 0;
  for (int h : hit) { if (h > 1) ++twice; if (h == 0) ++unused; }
  for (int h : phit) { if (h != 1) ++twice; }
  printf("rows %lld out_of_range %lld shared %lld unused %lld\n", rows, bad, twice, unused);
}

int main() {
  char kind[16];
  while (scanf("%15s", kind) == 1) {
    if (!strcmp(kind, "seg")) {
      int P, W, head, count;
      long long next_pos, t;
      if (scanf("%d %d %d %d %lld %lld", &P, &W, &head, &count, &next_pos, &t) != 6) return 2;
      seg_case(P, W, head, count, next_pos, t);
    } else if (!strcmp(kind, "addr")) {
      int S, Hkv, P_max, W, page_rows, nphys;
      if (scanf("%d %d %d %d %d %d", &S, &Hkv, &P_max, &W, &page_rows, &nphys) != 6) return 2;
      addr_case(S, Hkv, P_max, W, page_rows, nphys);
    } else {
      return 2;
    }
  }
  return 0;
}
