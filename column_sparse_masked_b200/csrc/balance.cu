// Sparsity-aware split of the query sequence into per-rank chunks (host code).
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight, names a sparsity-aware load balancer (HCC-IPO) for the context-
// parallel extension without giving its rule.  Read here in its plainest form:
// the ranks' shares of the work are made as even as possible, the work of a
// query tile being its number of unmasked (row, key) pairs.  Each rank takes a
// contiguous run of whole q-tiles, so its mask follows from the global vectors
// by the clip-shift-max localisation of the same section, with no exchange.
//
// The split minimises the largest chunk cost exactly: a binary search over the
// answer with a left-to-right greedy feasibility test (the classic linear
// partition), then one deterministic split at the optimal bound.
#include <cstdint>

#include "../../include/flashmask.h"

namespace {

// Chunks that a left-to-right greedy packing within `cap` needs (every single
// cost is <= cap).
int64_t chunks_needed(const int64_t* c, int32_t n, int64_t cap) {
  int64_t used = 1, run = 0;
  for (int32_t t = 0; t < n; ++t) {
    if (run + c[t] > cap) {
      ++used;
      run = 0;
    }
    run += c[t];
  }
  return used;
}

}  // namespace

extern "C" int flashmask_balance_chunks(const int64_t* costs, int32_t n, int32_t parts, int32_t* bounds,
                                        int64_t* max_cost) {
  if (n < 0 || parts <= 0 || !bounds || (n > 0 && !costs)) return FLASHMASK_ERR_INVALID_ARG;
  int64_t lo = 0, total = 0;
  for (int32_t t = 0; t < n; ++t) {
    if (costs[t] < 0 || costs[t] > INT64_MAX / 4 - total) return FLASHMASK_ERR_INVALID_ARG;
    total += costs[t];
    if (costs[t] > lo) lo = costs[t];
  }
  if (n <= parts) {  // one tile per chunk, the rest empty: the largest single cost is the optimum
    for (int32_t p = 0; p <= parts; ++p) bounds[p] = p < n ? p : n;
    if (max_cost) *max_cost = lo;
    return FLASHMASK_OK;
  }
  // smallest cap in [max cost, total] that `parts` greedy chunks can hold
  int64_t hi = total;
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (chunks_needed(costs, n, mid) <= parts)
      hi = mid;
    else
      lo = mid + 1;
  }
  const int64_t cap = lo;
  // Left to right, each chunk takes as many tiles as fit within the optimal
  // cap while leaving at least one tile for every later chunk.  When that
  // reserve never binds this is the greedy packing (which fits in `parts`
  // chunks); once it binds, every later chunk holds a single tile (<= cap).
  int32_t b = 0;
  bounds[0] = 0;
  for (int32_t p = 0; p + 1 < parts; ++p) {
    const int32_t last = n - (parts - 1 - p);  // exclusive end that leaves the reserve
    int64_t run = 0;
    int32_t e = b;
    while (e < last && (e == b || run + costs[e] <= cap)) run += costs[e++];
    bounds[p + 1] = e;
    b = e;
  }
  bounds[parts] = n;
  if (max_cost) *max_cost = cap;
  return FLASHMASK_OK;
}
