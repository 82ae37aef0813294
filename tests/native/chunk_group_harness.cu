// Host-side harness for the chunk mode of the tensor-core decode kernel
// (prefix_sliding_window_ring_b200/csrc/decode_pack.cuh: dec_runs_chunk,
// dec_row_queries, dec_tile_qdep), compiled by the CPU tests and run without a
// GPU.  For each case read from stdin it prints the pair's tiles and, per
// tile, its pieces with the query mask of every row as the kernel applies it:
// the row's dec_row_queries bits on a query-dependent tile, all queries
// otherwise (prefix rows: all queries).
//
// Input lines:  P W head count t0 i0 nq page TR csize
// Output line:  ntiles rows padded ring_ok, then per tile "|" and its pieces
//               src,row,smem_row,n,m0:m1:...  (one mask per row, in decimal),
//               with csize > 0 the tiles of the cluster shares in rank order.
#include <stdio.h>
#include <string.h>

#include "decode_pack.cuh"

int main() {
  int P, W, head, count, i0, nq, page, TR, csize;
  long long t0;
  while (scanf("%d %d %d %d %lld %d %d %d %d %d", &P, &W, &head, &count, &t0, &i0, &nq, &page,
               &TR, &csize) == 10) {
    ps::DevMeta m;
    memset(&m, 0, sizeof(m));
    m.next_pos = t0;
    m.P = P;
    m.head = head;
    m.count = count;
    const ps::DecRuns r = ps::dec_runs_chunk(m, W, t0, i0, nq, page);
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
        const bool dep = ps::dec_tile_qdep(r, x0, x1);
        int wsrc = -1, wrow = -1;
        const bool whole = !dep && ps::dec_range_whole(r, TR, x0, x1, &wsrc, &wrow);
        printf(" |");
        ps::dec_range_pieces(r, x0, x1, [&](int src, int row, int sr, int n) {
          printf(" %d,%d,%d,%d,", src, row, sr, n);
          for (int k = 0; k < n; ++k) {
            const unsigned q = (dep && src != ps::RUN_PREFIX) ? ps::dec_row_queries(r, src, row + k)
                                                              : 0xffu;
            printf(k ? ":%u" : "%u", q);
          }
        });
        if (whole) printf(" W%d,%d", wsrc, wrow);
      }
    }
    printf("\n");
  }
  return 0;
}
