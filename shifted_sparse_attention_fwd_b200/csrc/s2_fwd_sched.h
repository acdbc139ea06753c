// Host side of the forward's work distribution: which (query tile pair) units each persistent
// CTA takes. Plain C++ (no CUDA), so the library and the host tests build the same code.
//
// Each unit goes to the CTA with the least work so far, by a cost of (query tile, key tile)
// steps plus 3 for the unit's own loads, epilogue and boundary (per-role traces of the kernel
// put a unit's fixed cost at about 3.25 steps). The units are handed out in the kernel's
// L2-grouped order, which keeps the CTAs moving through the heads and groups together, except
// the last 2 x grid, which go heaviest first (longest-processing-time-first) so they even out
// what the earlier ones left: on the Llama2-7B layer the busiest CTA ends 3 % above the mean
// instead of 11 % (all units heaviest first: 2.6 %, but the lost L2 grouping costs more than that
// at B = 4). Each CTA takes its units in index order.
#pragma once

#include <algorithm>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "s2_tiles.cuh"

namespace s2 {

// start has grid + 1 entries: CTA c takes unit[start[c] .. start[c + 1]). Returns false (and
// leaves both lists empty) when there are no more units than CTAs, so that every CTA simply
// takes unit blockIdx.x, blockIdx.x + gridDim.x, ... instead.
inline bool fwd_unit_lists(int B, int Hq, int N, int G, int shb, int wrap, int grid,
                           std::vector<int>& start, std::vector<int>& unit) {
  start.clear();
  unit.clear();
  const int nqt = (N + kTileRows - 1) / kTileRows;
  const long long n_units = static_cast<long long>(B) * Hq * query_pairs_per_head(N);
  if (grid <= 0 || n_units <= grid) return false;
  std::vector<double> cost(n_units);
  for (long long u = 0; u < n_units; ++u) {
    int b, h, pair;
    query_pair_coords_chunked(static_cast<int>(u), B, Hq, N, G, kL2Chunk, b, h, pair);
    const int wrap_h = h >= shb ? wrap : kNoWrapSplit;
    double c = 3.0;
    for (int t = 0; t < 2; ++t) {
      const int qt = 2 * pair + t;
      if (qt < nqt) c += qt - group_begin(qt * kTileRows, G, wrap_h) / kTileRows + 1;
    }
    cost[u] = c;
  }
  std::vector<int> order(n_units);
  for (long long u = 0; u < n_units; ++u) order[u] = static_cast<int>(u);
  const long long tail = std::min<long long>(n_units, 2ll * grid);
  std::stable_sort(order.begin() + (n_units - tail), order.end(),
                   [&](int a, int b) { return cost[a] > cost[b]; });
  std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>,
                      std::greater<std::pair<double, int>>> load;
  for (int c = 0; c < grid; ++c) load.push({0.0, c});
  std::vector<int> owner(n_units), count(grid, 0);
  for (const int u : order) {
    const auto least = load.top();
    load.pop();
    owner[u] = least.second;
    ++count[least.second];
    load.push({least.first + cost[u], least.second});
  }
  start.assign(grid + 1, 0);
  for (int c = 0; c < grid; ++c) start[c + 1] = start[c] + count[c];
  unit.assign(n_units, 0);
  std::vector<int> fill(start.begin(), start.end() - 1);
  for (long long u = 0; u < n_units; ++u) unit[fill[owner[u]]++] = static_cast<int>(u);
  return true;
}

}  // namespace s2
