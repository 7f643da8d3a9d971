// Host-side partition of one jagged batch's users over several GPUs.
//
// No position reads across a user boundary (候选隔离注意力掩码, section 段 ID：掩码的表达方式: every
// query sees only keys of its own row; 'HSTU scale' tutorial, section 手算 padding 的浪费与 offset:
// user b is values[offsets[b]:offsets[b+1]]), so the users of a batch can be split over GPUs with no
// exchange at all in the forward pass: each GPU plans and runs its own users, and the outputs stay
// where they were computed. What matters is the balance: user costs span three orders of magnitude
// (a few rows against 4,100), so the split is longest-processing-time-first (LPT) list
// scheduling over each user's tile cost, the same cost the attention kernel's work queue orders by.
#include <algorithm>
#include <cstdint>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "jca.h"
#include "jca_internal.h"

extern "C" int64_t jca_user_tile_cost(int64_t row_len, int64_t n_keys) {
  if (row_len <= 0) return 0;
  const int64_t q_tiles = (row_len + jca::kTileM - 1) / jca::kTileM;
  const int64_t k_tiles = (n_keys + jca::kTileN - 1) / jca::kTileN;
  return q_tiles * (k_tiles > 1 ? k_tiles : 1);
}

extern "C" int jca_shard_users(const int64_t* row_len, const int64_t* n_keys, int64_t B,
                               int n_shards, int32_t* shard, int64_t* load) {
  if (B < 0 || n_shards < 1) return JCA_ERR_SHAPE;
  if (B > 0 && (!row_len || !n_keys || !shard)) return JCA_ERR_NULL;
  for (int64_t b = 0; b < B; ++b)
    if (row_len[b] < 0 || n_keys[b] < 0 || n_keys[b] > row_len[b]) return JCA_ERR_SHAPE;
  std::vector<int64_t> cost(static_cast<size_t>(B));
  std::vector<int64_t> order(static_cast<size_t>(B));
  for (int64_t b = 0; b < B; ++b) {
    cost[b] = jca_user_tile_cost(row_len[b], n_keys[b]);
    order[b] = b;
  }
  // Largest cost first; equal costs in user order, so that every rank computes the same split.
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t a, int64_t b) { return cost[a] > cost[b]; });
  // Least-loaded shard first; equal loads go to the lowest shard index.
  using Slot = std::pair<int64_t, int>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int s = 0; s < n_shards; ++s) heap.push({0, s});
  std::vector<int64_t> acc(static_cast<size_t>(n_shards), 0);
  for (int64_t i = 0; i < B; ++i) {
    const int64_t b = order[i];
    Slot top = heap.top();
    heap.pop();
    shard[b] = top.second;
    top.first += cost[b];
    acc[top.second] = top.first;
    heap.push(top);
  }
  if (load)
    for (int s = 0; s < n_shards; ++s) load[s] = acc[s];
  return JCA_OK;
}
