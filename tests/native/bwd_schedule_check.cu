// Host-side check of the backward's work decomposition and dQ ordering, using
// the kernel header's own decode_item / BwdItem (nothing is launched).
//
// For every shape given on the command line (ntiles, heads, causal, head
// group) it checks:
//  1. every (key tile j, query tile i) pair of every head is visited exactly
//     once (causal: only i >= j);
//  2. for each (head, query tile, sum), the positions of its contributors are
//     0, 1, ..., count-1: one fixed total order, whose first entry stores;
//  3. the contributor just before (i, j) in that order belongs to an item that
//     is fetched earlier (smaller item index) and visits tile i one step
//     (non-causal) or two steps (causal) earlier in its own sequence, so the
//     earliest unfinished item never waits and items that start together do
//     not wait on each other;
//  4. sum_contributors (the counts the finishing step waits for) equals the
//     number of contributors of every sum, empty sums included.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <tuple>
#include <vector>

#include "../../exact_attention_119_b200/csrc/bwd_kernels.cuh"

int check(int ntiles, int heads, bool causal, int group) {
  // (bh, i, chain) -> list of (pos, item, step, j)
  std::map<std::tuple<int, int, int>, std::vector<std::tuple<int, int, int, int>>> sums;
  std::map<std::tuple<int, int, int>, int> visits;  // (bh, j, i) -> count
  const int total = heads * ntiles;
  for (int item = 0; item < total; ++item) {
    const fa::BwdItem w = fa::decode_item(item, ntiles, causal, heads, group);
    if (w.bh < 0 || w.bh >= heads || w.j < 0 || w.j >= ntiles || w.T < 1 || w.T > ntiles) {
      std::printf("bad item %d: bh %d j %d T %d\n", item, w.bh, w.j, w.T);
      return 1;
    }
    for (int s = 0; s < w.T; ++s) {
      const int i = w.tile(s);
      if (i < 0 || i >= ntiles || (causal && i < w.j)) {
        std::printf("item %d step %d visits tile %d\n", item, s, i);
        return 1;
      }
      ++visits[{w.bh, w.j, i}];
      sums[{w.bh, i, w.chain(i)}].push_back({w.pos(i), item, s, w.j});
    }
  }
  for (int bh = 0; bh < heads; ++bh)
    for (int j = 0; j < ntiles; ++j)
      for (int i = 0; i < ntiles; ++i) {
        const int want = (!causal || i >= j) ? 1 : 0;
        const auto it = visits.find({bh, j, i});
        const int got = it == visits.end() ? 0 : it->second;
        if (got != want) {
          std::printf("head %d pair (i %d, j %d) visited %d times\n", bh, i, j, got);
          return 1;
        }
      }
  // 4. the finishing step's contributor counts match the sums, including the
  //    empty ones.
  for (int bh = 0; bh < heads; ++bh)
    for (int i = 0; i < ntiles; ++i)
      for (int c = 0; c < 2; ++c) {
        const auto it = sums.find({bh, i, c});
        const int got = it == sums.end() ? 0 : (int)it->second.size();
        if (got != fa::sum_contributors(i, ntiles, causal, c)) {
          std::printf("head %d tile %d sum %d: %d contributors, finishing step expects %d\n", bh, i, c, got,
                      fa::sum_contributors(i, ntiles, causal, c));
          return 1;
        }
      }
  for (auto& kv : sums) {
    auto& v = kv.second;
    std::vector<int> by_pos(v.size(), -1);
    for (size_t k = 0; k < v.size(); ++k) {
      const int p = std::get<0>(v[k]);
      if (p < 0 || p >= (int)v.size() || by_pos[p] != -1) {
        std::printf("sum (head %d, tile %d, chain %d): positions not a permutation\n", std::get<0>(kv.first),
                    std::get<1>(kv.first), std::get<2>(kv.first));
        return 1;
      }
      by_pos[p] = (int)k;
    }
    for (size_t p = 1; p < v.size(); ++p) {
      const auto& cur = v[by_pos[p]];
      const auto& prev = v[by_pos[p - 1]];
      // The predecessor is fetched earlier and visits the tile `lag` steps
      // earlier: one for the non-causal sums, two for the causal parity sums.
      const int lag = causal ? 2 : 1;
      if (std::get<1>(prev) >= std::get<1>(cur) || std::get<2>(prev) != std::get<2>(cur) - lag) {
        std::printf("sum (head %d, tile %d): contributor j=%d (item %d, step %d) follows j=%d (item %d, step %d)\n",
                    std::get<0>(kv.first), std::get<1>(kv.first), std::get<3>(cur), std::get<1>(cur), std::get<2>(cur),
                    std::get<3>(prev), std::get<1>(prev), std::get<2>(prev));
        return 1;
      }
    }
  }
  return 0;
}

int main(int argc, char** argv) {
  int bad = 0, shapes = 0;
  for (int a = 1; a + 3 < argc; a += 4) {
    const int n = std::atoi(argv[a]), h = std::atoi(argv[a + 1]), c = std::atoi(argv[a + 2]);
    const int g = std::atoi(argv[a + 3]);
    const int r = check(n, h, c != 0, g);
    if (r) std::printf("FAILED ntiles %d heads %d causal %d group %d\n", n, h, c, g);
    bad |= r;
    ++shapes;
  }
  if (!bad) std::printf("OK %d shapes\n", shapes);
  return bad;
}
