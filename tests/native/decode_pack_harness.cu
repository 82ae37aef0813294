// Host-side harness for the tensor-core decode kernel's tile layout
// (prefix_sliding_window_ring_b200/csrc/decode_pack.cuh), compiled by the CPU
// tests and run without a GPU.  For each case read from stdin it prints the
// pair's tiles and, per tile, its pieces: source, first prefix row / ring
// slot, tile row, valid rows.
//
// Input lines:  P W head count next_pos t page step TR csize
// Output line:  ntiles rows padded ring_ok, then per tile "|" and its pieces
//               src,row,smem_row,n.  With csize > 0 the tiles are those of the
//               cluster shares of ranks 0 .. csize-1, in order, each share's
//               tiles starting at its first padded row.
#include <stdio.h>
#include <string.h>

#include "decode_pack.cuh"

int main() {
  int P, W, head, count, page, step, TR, csize;
  long long next_pos, t;
  while (scanf("%d %d %d %d %lld %lld %d %d %d %d", &P, &W, &head, &count, &next_pos, &t, &page,
               &step, &TR, &csize) == 10) {
    ps::DevMeta m;
    memset(&m, 0, sizeof(m));
    m.next_pos = next_pos;
    m.P = P;
    m.head = head;
    m.count = count;
    const ps::DecRuns r = ps::dec_runs(m, W, t, page, step != 0);
    int nt = 0;
    const int C = csize > 0 ? csize : 1;
    for (int rank = 0; rank < C; ++rank) {
      int x0 = 0, x1 = r.padded;
      if (csize > 0) ps::dec_cluster_share(r, rank, csize, &x0, &x1);
      if (x1 > x0) nt += (x1 - x0 + TR - 1) / TR;
    }
    printf("%d %d %d %d", nt, r.rows, r.padded, r.ring_ok);
    for (int rank = 0; rank < C; ++rank) {
      int xs = 0, xe = r.padded;
      if (csize > 0) ps::dec_cluster_share(r, rank, csize, &xs, &xe);
      for (int x0 = xs; x0 < xe; x0 += TR) {
        const int x1 = x0 + TR < xe ? x0 + TR : xe;
        printf(" |");
        int wsrc = -1, wrow = -1;
        const bool whole = ps::dec_range_whole(r, TR, x0, x1, &wsrc, &wrow);
        ps::dec_range_pieces(r, x0, x1, [&](int src, long long row, int sr, int n) {
          printf(" %d,%lld,%d,%d", src, row, sr, n);
        });
        if (whole) printf(" W%d,%d", wsrc, wrow);
      }
    }
    printf("\n");
  }
  return 0;
}
