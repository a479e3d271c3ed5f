// Host side of the tensor-core attention: the batch's work list and its
// division among the CTAs.
//
// DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 4: a request's
// prefix K/V are computed once and read by all its candidate branches.  An
// item is one (request, KV head) and up to rows_per_item query rows of it:
// prefix rows (kind 0, causal over the prefix) or whole candidate branches
// (kind 1, every prefix key tile and their own branch).  The items of one
// (request, KV head) stay together in the list so that the CTAs running
// them at the same time share that head's prefix K/V through L2; groups go
// most expensive first, and inside a group branch items come first, then
// prefix items from the last rows.  A request whose first c prefix tokens
// come from the prefix KV store has query rows from c on; its key tiles
// are ceil(c / 128) store tiles, then tiles of 128 from c.
//
// Each CTA runs the items the greedy list schedule gives it: in list order,
// an item goes to the CTA with the least work so far.  The estimated cost of
// an item is its key tiles, +20% when its second query sub-tile is in use
// (the two sub-tiles run side by side), plus half a tile for starting it.
// Items stay in list order within a CTA and CTAs advance through the list at
// about the same pace, so the items of one (request, KV head) still run close
// together in time.
#include <algorithm>
#include <functional>
#include <queue>
#include <vector>

#include "duolm.h"
#include "kernels.cuh"

namespace duolm {

int64_t plan_attention(const int4* req, const int2* reqx, int64_t R, int n_kv_heads, int rows_per_item,
                       int branch_len, int n_ctas, int64_t cap_items, int4* items, int32_t* cta_off) {
  const int Rw = rows_per_item;
  const int per = (Rw / branch_len) * branch_len;  // branch rows of an item: whole candidates
  const int key_tile = 128;
  auto prefix_tiles = [&](int cached, int kend) -> int64_t {
    return (cached + key_tile - 1) / key_tile + (kend - cached + key_tile - 1) / key_tile;
  };
  std::vector<std::pair<int64_t, int64_t>> groups;  // (cost in key tiles, request * n_kv_heads + kvh)
  groups.reserve((size_t)R * n_kv_heads);
  for (int64_t r = 0; r < R; ++r) {
    const int L = req[r].y, K = req[r].z, cr = reqx[r].x;
    int64_t cost = 0;
    for (int row0 = cr; row0 < L; row0 += Rw) cost += prefix_tiles(cr, std::min(row0 + Rw, L));
    cost += (int64_t)((K * branch_len + per - 1) / per) * (prefix_tiles(cr, L) + 1);
    for (int kvh = 0; kvh < n_kv_heads; ++kvh) groups.push_back({cost, r * n_kv_heads + kvh});
  }
  std::stable_sort(groups.begin(), groups.end(), [](const auto& a, const auto& b) { return a.first > b.first; });
  int64_t n_items = 0;
  for (const auto& g : groups) {
    const int r = (int)(g.second / n_kv_heads), kvh = (int)(g.second % n_kv_heads);
    const int L = req[r].y, K = req[r].z, cr = reqx[r].x;
    const int64_t need = (K * branch_len + per - 1) / per + (L - cr + Rw - 1) / Rw;
    if (n_items + need > cap_items) return -1;
    for (int row0 = 0; row0 < K * branch_len; row0 += per) items[n_items++] = int4{r, kvh, 1, row0};
    if (L > cr)
      for (int row0 = cr + ((L - cr - 1) / Rw) * Rw; row0 >= cr; row0 -= Rw) items[n_items++] = int4{r, kvh, 0, row0};
  }
  std::vector<int> owner((size_t)n_items);
  {
    std::priority_queue<std::pair<int64_t, int>, std::vector<std::pair<int64_t, int>>, std::greater<>> load;
    for (int c = 0; c < n_ctas; ++c) load.push({0, c});
    const int half_rows = Rw / 2;  // rows of one query sub-tile
    for (int64_t i = 0; i < n_items; ++i) {
      const int4 m = items[i];
      const int L = req[m.x].y, K = req[m.x].z, cr = reqx[m.x].x;
      const int nrows = m.z ? std::min(per, K * branch_len - m.w) : std::min(Rw, L - m.w);
      const int kend = m.z ? L : std::min(m.w + Rw, L);
      const int64_t tiles = prefix_tiles(cr, kend) + (m.z ? (nrows + key_tile - 1) / key_tile : 0);
      const int64_t cost = 10 * tiles + (nrows > half_rows ? 2 * tiles : 0) + 5;
      auto top = load.top();
      load.pop();
      owner[i] = top.second;
      load.push({top.first + cost, top.second});
    }
  }
  // stable regrouping by owner: CTA c's items, in list order
  std::vector<int4> listed(items, items + n_items);
  std::fill(cta_off, cta_off + n_ctas + 1, 0);
  for (int64_t i = 0; i < n_items; ++i) ++cta_off[owner[i] + 1];
  for (int c = 0; c < n_ctas; ++c) cta_off[c + 1] += cta_off[c];
  std::vector<int32_t> fill(cta_off, cta_off + n_ctas);
  for (int64_t i = 0; i < n_items; ++i) items[fill[owner[i]]++] = listed[i];
  return n_items;
}

}  // namespace duolm

extern "C" int64_t duolm_debug_attention_plan(int n_requests, const int32_t* L, const int32_t* K,
                                              const int32_t* cached, int branch_len, int n_kv_heads,
                                              int rows_per_item, int n_ctas, int32_t* items, int64_t cap_items,
                                              int32_t* cta_off) {
  if (n_requests < 1 || !L || !K || !cached || branch_len < 1 || n_kv_heads < 1 || rows_per_item < 2 ||
      branch_len > rows_per_item || n_ctas < 1 || cap_items < 0 || (cap_items > 0 && !items) || !cta_off)
    return DUOLM_E_ARG;
  std::vector<int4> req(n_requests);
  std::vector<int2> rx(n_requests);
  for (int r = 0; r < n_requests; ++r) {
    if (cached[r] < 0 || L[r] < cached[r] || (L[r] == 0) || K[r] < 1) return DUOLM_E_ARG;
    req[r] = int4{0, L[r], K[r], 0};
    rx[r] = int2{cached[r], 0};
  }
  std::vector<int4> it((size_t)cap_items);
  const int64_t n = duolm::plan_attention(req.data(), rx.data(), n_requests, n_kv_heads, rows_per_item, branch_len,
                                          n_ctas, cap_items, it.data(), cta_off);
  if (n < 0) return DUOLM_E_CAPACITY;
  for (int64_t i = 0; i < n; ++i) {
    items[4 * i] = it[i].x;
    items[4 * i + 1] = it[i].y;
    items[4 * i + 2] = it[i].z;
    items[4 * i + 3] = it[i].w;
  }
  return n;
}
