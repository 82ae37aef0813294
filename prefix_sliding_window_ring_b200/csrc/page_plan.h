// Host-side page planning of a paged ring (no CUDA): which ring pages of a
// sequence a write touches, and which physical pages from the pool they get.
// Plain C++ so that it can be checked on the CPU.
#pragma once
#include <stdint.h>

#include <vector>

namespace ps {

struct PageShape {
  int64_t W;          // ring slots per sequence
  int64_t page_rows;  // slots per page (W % page_rows == 0)
  int64_t npg;        // pages per sequence, W / page_rows
};

// Ring slots [slot0, slot0 + n) (mod W; only the last W of them if n > W) of
// sequence `seq` are about to be written.  Every ring page they touch that
// has no physical page yet (pages[p] < 0) gets the last page of `avail`, and
// the page-table entry to set is recorded in (idx, phys), idx = seq * npg + p.
// Returns false if `avail` runs out; the caller works on copies of `pages`
// and `avail` and keeps them only on success, so a failure changes nothing.
inline bool plan_pages(const PageShape& sh, int seq, std::vector<int32_t>& pages, int64_t slot0,
                       int64_t n, std::vector<int32_t>& avail, std::vector<int32_t>& idx,
                       std::vector<int32_t>& phys) {
  if (n <= 0) return true;
  const int64_t W = sh.W, pr = sh.page_rows;
  int64_t s = ((slot0 % W) + W) % W;
  for (int64_t left = n < W ? n : W; left > 0;) {
    const int64_t page = s / pr;
    const int64_t chunk = pr - s % pr < left ? pr - s % pr : left;
    if (pages[page] < 0) {
      if (avail.empty()) return false;
      pages[page] = avail.back();
      avail.pop_back();
      idx.push_back((int32_t)(seq * sh.npg + page));
      phys.push_back(pages[page]);
    }
    left -= chunk;
    s = (s + chunk) % W;
  }
  return true;
}

}  // namespace ps
