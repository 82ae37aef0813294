// Host-side harness for the paged ring's page planning
// (prefix_sliding_window_ring_b200/csrc/page_plan.h), compiled by the CPU
// tests.  One case per input line:
//   W page_rows seq slot0 n | pages[0..npg) | avail...
// Output per case:  ok | pages after | avail after | idx:phys ...
#include <stdio.h>

#include <iostream>
#include <sstream>
#include <string>
#include <vector>

#include "page_plan.h"

int main() {
  std::string line;
  while (std::getline(std::cin, line)) {
    if (line.empty()) continue;
    std::stringstream ss(line);
    long long W, pr, slot0, n;
    int seq;
    std::string bar;
    ss >> W >> pr >> seq >> slot0 >> n >> bar;
    const long long npg = W / pr;
    std::vector<int32_t> pages(npg), avail, idx, phys;
    for (long long i = 0; i < npg; ++i) ss >> pages[i];
    ss >> bar;
    int32_t a;
    while (ss >> a) avail.push_back(a);
    const ps::PageShape sh{W, pr, npg};
    const bool ok = ps::plan_pages(sh, seq, pages, slot0, n, avail, idx, phys);
    std::cout << (ok ? 1 : 0) << " |";
    for (int32_t p : pages) std::cout << ' ' << p;
    std::cout << " |";
    for (int32_t p : avail) std::cout << ' ' << p;
    std::cout << " |";
    for (size_t i = 0; i < idx.size(); ++i) std::cout << ' ' << idx[i] << ':' << phys[i];
    std::cout << '\n';
  }
  return 0;
}
