// dp_partition.cu - host-side split of one global jagged batch over data-parallel ranks.
//
// The sequences of a batch are independent ("4.4 Scaling Recommendation Models", Generative
// Recommenders and HSTU, Efficiency tricks: kernels over variable-length sequences; the attention
// never crosses a sequence boundary), so a data-parallel step can hand whole sequences to ranks with
// no exchange until the gradient sum. The split balances the work of one layer step per rank:
// cost(n) = n (n + 1) + 5 D n, which is the attention's 2 D n (n + 1) flops plus the two
// projections' 10 D^2 n flops, divided by 2 D. Greedy longest-processing-time first: sequences in
// order of decreasing cost (ties by index), each to the rank with the smallest load so far (ties by
// the lowest rank). The largest load is then at most 4/3 of the best possible split's (Graham's
// bound for this greedy rule), and every rank computing the split gets the same answer.
#include <stdint.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "../../include/hstu.h"

extern "C" double hstu_dp_sequence_cost(int64_t n, int32_t D) {
  const double nn = static_cast<double>(n);
  return nn * (nn + 1.0) + 5.0 * static_cast<double>(D) * nn;
}

extern "C" hstu_status_t hstu_dp_partition(const int64_t* lengths, int32_t B, int32_t D, int32_t world,
                                           int32_t* rank_of, double* rank_cost) {
  if (B < 0 || world < 1 || D < 1 || (B > 0 && (!lengths || !rank_of))) return HSTU_ERR_INVALID_ARG;
  for (int32_t b = 0; b < B; ++b)
    if (lengths[b] < 0) return HSTU_ERR_INVALID_ARG;
  std::vector<std::pair<double, int32_t>> order(static_cast<size_t>(B));
  for (int32_t b = 0; b < B; ++b) order[b] = {hstu_dp_sequence_cost(lengths[b], D), b};
  std::stable_sort(order.begin(), order.end(),
                   [](const std::pair<double, int32_t>& x, const std::pair<double, int32_t>& y) {
                     return x.first > y.first;
                   });
  // min-heap of (load, rank): the least loaded rank, lowest index first among equal loads
  typedef std::pair<double, int32_t> Slot;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int32_t r = 0; r < world; ++r) heap.push({0.0, r});
  std::vector<double> load(static_cast<size_t>(world), 0.0);
  for (const auto& item : order) {
    const Slot s = heap.top();
    heap.pop();
    rank_of[item.second] = s.second;
    load[s.second] = s.first + item.first;
    heap.push({load[s.second], s.second});
  }
  if (rank_cost)
    for (int32_t r = 0; r < world; ++r) rank_cost[r] = load[r];
  return HSTU_OK;
}
