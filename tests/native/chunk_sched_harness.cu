// Host-side harness for the tensor-core chunk kernel's key-tile schedule
// (prefix_sliding_window_ring_b200/csrc/chunk_sched.cuh), compiled by the CPU
// tests and run without a GPU.  For each case read from stdin it prints the
// lowest ring or block key position (rlo) and the key tiles a query tile
// reads: source, first row, first position, rows.
//
// Input lines:  P W head count next_pos t0 plo phi prompt page
#include <stdio.h>
#include <string.h>

#include "chunk_sched.cuh"

int main() {
  int P, W, head, count, prompt, page;
  long long next_pos, t0, plo, phi;
  while (scanf("%d %d %d %d %lld %lld %lld %lld %d %d", &P, &W, &head, &count, &next_pos, &t0,
               &plo, &phi, &prompt, &page) == 10) {
    ps::DevMeta m;
    memset(&m, 0, sizeof(m));
    m.next_pos = next_pos;
    m.P = P;
    m.head = head;
    m.count = count;
    const ps::KSched s = ps::make_sched(m, W, page, t0, plo, phi, prompt != 0);
    printf("%d %lld", s.ntiles, (long long)s.rlo);
    for (int j = 0; j < s.ntiles; ++j) {
      const ps::KTile t = ps::tile_of(s, j);
      printf(" %d,%lld,%lld,%d", t.src, (long long)t.row, (long long)t.pos0, t.valid);
    }
    printf("\n");
  }
  return 0;
}
