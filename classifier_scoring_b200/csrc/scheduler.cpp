// Dynamic-programming batch scheduler.
//
// "TurboTransformers: An Efficient GPU Serving System For Transformer Models"
// (abstract; proposed-method section): a serving framework whose batch
// scheduler uses dynamic programming to reach the best throughput on
// variable-length requests, grouping requests by length with minimal padding.
// The page gives no recurrence; this follows its plainest reading:
//   sort the queue by (length, arrival index); a batch of b requests whose
//   longest has length L costs T(b, L) (c0 + c1*b*L, or a table that is
//   non-decreasing in L); best[i] = min over the last batch (j, i] of
//   best[j] + T(i - j, l_i) with i - j <= Bmax, ties to the smallest j;
//   batches are numbered in execution order (ascending longest length).
// Latency-aware variants (the review's main results report the scheduler's
// mean latency at its serving rate): with objective RM_SCHED_LATENCY a batch
// that starts at sorted position j is charged T * (n - j), the delay it adds
// to every request from j on, so the DP minimises the sum of completion times
// of batches run back to back in ascending longest length; with max_cost > 0
// no batch of two or more requests may cost more than max_cost.
// Costs are summed in 128-bit integers so no queue can overflow them.
#include "host.h"

#include <algorithm>
#include <numeric>
#include <vector>

namespace rmk {

int schedule_dp(const SchedCost& cost, const int32_t* lengths, int32_t n, int32_t* out) {
  std::vector<int32_t> order(static_cast<size_t>(n));
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return lengths[a] < lengths[b]; });
  std::vector<__int128> best(static_cast<size_t>(n) + 1);
  std::vector<int32_t> from(static_cast<size_t>(n) + 1, 0);
  best[0] = 0;
  for (int32_t i = 1; i <= n; ++i) {
    const int32_t longest = lengths[order[i - 1]];
    const int32_t j0 = std::max<int32_t>(0, i - cost.bmax);
    __int128 b = -1;
    int32_t arg = j0;
    for (int32_t j = j0; j < i; ++j) {
      const int64_t t = cost.eval(i - j, longest);
      if (cost.max_cost > 0 && i - j >= 2 && t > cost.max_cost) continue;
      const __int128 w = cost.objective == RM_SCHED_LATENCY
                             ? static_cast<__int128>(t) * (n - j)
                             : static_cast<__int128>(t);
      const __int128 c = best[j] + w;
      if (b < 0 || c < b) {
        b = c;
        arg = j;
      }
    }
    best[i] = b;
    from[i] = arg;
  }
  // segments (from[i], i] walked back from n, then numbered front to back
  std::vector<int32_t> cuts;
  for (int32_t i = n; i > 0; i = from[i]) cuts.push_back(i);
  std::reverse(cuts.begin(), cuts.end());
  int32_t start = 0, id = 0;
  for (int32_t end : cuts) {
    for (int32_t k = start; k < end; ++k) out[order[k]] = id;
    start = end;
    ++id;
  }
  return id;
}

}  // namespace rmk
