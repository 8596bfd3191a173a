// Host pack planner: per-sample layout, cumulative offsets and the
// longest-first work list.
//
// [Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": samples of
//  different resolutions are flattened to variable-length token sequences and
//  packed with their text under a fixed token budget; attention uses
//  per-sample cumulative offsets. Video overview, 00:04:03: no padding.]
//
// The work list holds one item per (sample, head, 256-row query tile). An
// item's cost grows with the keys it attends over (its sample's length) and
// with its 128-row query sub-tiles (the last tile of a sample may hold only
// one). Items are ordered by that cost, largest first: handing the expensive
// items out first keeps the last wave of the persistent kernel short.

#include <algorithm>
#include <cstdint>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "../../include/mf_attn.h"

extern "C" int32_t mf_abi_version(void) { return 4; }

extern "C" const char* mf_status_string(mf_status status) {
  switch (status) {
    case MF_OK: return "MF_OK";
    case MF_ERR_INVALID_ARG: return "MF_ERR_INVALID_ARG";
    case MF_ERR_UNSUPPORTED: return "MF_ERR_UNSUPPORTED";
    case MF_ERR_ALIGNMENT: return "MF_ERR_ALIGNMENT";
    case MF_ERR_WORKSPACE: return "MF_ERR_WORKSPACE";
    case MF_ERR_BUDGET: return "MF_ERR_BUDGET";
    case MF_ERR_CUDA: return "MF_ERR_CUDA";
    case MF_ERR_TIMEOUT: return "MF_ERR_TIMEOUT";
    case MF_ERR_BOUNDS: return "MF_ERR_BOUNDS";
  }
  return "MF_ERR_UNKNOWN";
}

extern "C" mf_status mf_pack_plan(int32_t n_samples, const int32_t* n_text,
                                  const int32_t* grid_h, const int32_t* grid_w,
                                  const int32_t* frames, int32_t heads, int32_t head_dim,
                                  int64_t token_budget, int32_t* cu_seqlens, mf_segment* segs,
                                  mf_work_item* work, int32_t* n_work, int32_t* total_tokens) {
  if (n_samples < 1 || heads < 1 || !n_text || !grid_h || !grid_w) return MF_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return MF_ERR_UNSUPPORTED;

  std::vector<mf_segment> seg(static_cast<size_t>(n_samples));
  int64_t total = 0;
  int64_t items = 0;
  for (int32_t i = 0; i < n_samples; ++i) {
    const int64_t nt = n_text[i], gh = grid_h[i], gw = grid_w[i];
    const int64_t fr = frames ? frames[i] : 1;
    if (nt < 0 || gh < 1 || gw < 1 || fr < 1) return MF_ERR_INVALID_ARG;
    if (gh > INT32_MAX || gw > INT32_MAX || gh * gw > INT32_MAX / fr) return MF_ERR_INVALID_ARG;
    const int64_t len = nt + fr * gh * gw;
    if (len > INT32_MAX - total) return MF_ERR_INVALID_ARG;
    seg[i].start = static_cast<int32_t>(total);
    seg[i].len = static_cast<int32_t>(len);
    seg[i].n_text = static_cast<int32_t>(nt);
    seg[i].grid_h = static_cast<int32_t>(gh);
    seg[i].grid_w = static_cast<int32_t>(gw);
    seg[i].frames = static_cast<int32_t>(fr);
    total += len;
    items += ((len + MF_TILE_M - 1) / MF_TILE_M) * static_cast<int64_t>(heads);
  }
  if (token_budget > 0 && total > token_budget) return MF_ERR_BUDGET;
  if (items > INT32_MAX) return MF_ERR_INVALID_ARG;

  if (total_tokens) *total_tokens = static_cast<int32_t>(total);
  if (cu_seqlens) {
    cu_seqlens[0] = 0;
    for (int32_t i = 0; i < n_samples; ++i) cu_seqlens[i + 1] = seg[i].start + seg[i].len;
  }
  if (segs) std::copy(seg.begin(), seg.end(), segs);
  if (n_work) {
    // With work == NULL this is the size query; otherwise *n_work is the
    // capacity the caller provides, and it must be large enough.
    if (work && *n_work < items) return MF_ERR_INVALID_ARG;
    *n_work = static_cast<int32_t>(items);
  } else if (work) {
    return MF_ERR_INVALID_ARG;
  }
  if (work) {
    int64_t w = 0;
    for (int32_t si = 0; si < n_samples; ++si) {
      const int32_t tiles = (seg[si].len + MF_TILE_M - 1) / MF_TILE_M;
      for (int32_t h = 0; h < heads; ++h)
        for (int32_t qt = 0; qt < tiles; ++qt) work[w++] = mf_work_item{si, h, qt, seg[si].len};
    }
    // cost: keys x query sub-tiles (a last tile of at most half the rows has one)
    auto cost = [&](const mf_work_item& it) {
      const int64_t rows = std::min<int64_t>(MF_TILE_M, seg[it.seg].len - int64_t{it.q_tile} * MF_TILE_M);
      return int64_t{it.kv_len} * (rows > MF_TILE_M / 2 ? 2 : 1);
    };
    std::stable_sort(work, work + w, [&](const mf_work_item& a, const mf_work_item& b) {
      return cost(a) > cost(b);
    });
  }
  return MF_OK;
}

extern "C" mf_status mf_schedule_work(const mf_work_item* work, int32_t n_work, int32_t n_ctas,
                                      mf_work_item* sched, int32_t* n_sched) {
  if (!work || !n_sched || n_work < 1 || n_ctas < 1) return MF_ERR_INVALID_ARG;
  const int32_t ctas = std::min(n_ctas, n_work);
  std::vector<int64_t> cost(static_cast<size_t>(n_work));
  for (int32_t i = 0; i < n_work; ++i) {
    const mf_work_item& it = work[i];
    if (it.q_tile < 0 || it.kv_len < 1) return MF_ERR_INVALID_ARG;
    const int64_t rows = std::min<int64_t>(MF_TILE_M, int64_t{it.kv_len} - int64_t{it.q_tile} * MF_TILE_M);
    if (rows < 1) return MF_ERR_INVALID_ARG;
    const int64_t steps = (int64_t{it.kv_len} + MF_TILE_N - 1) / MF_TILE_N;
    cost[i] = steps * (rows > MF_TILE_M / 2 ? 20 : 19);
  }
  std::vector<int32_t> order(static_cast<size_t>(n_work));
  for (int32_t i = 0; i < n_work; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
  // least-loaded CTA first, lowest index on ties
  using Slot = std::pair<int64_t, int32_t>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int32_t c = 0; c < ctas; ++c) heap.push({0, c});
  std::vector<std::vector<int32_t>> lists(static_cast<size_t>(ctas));
  size_t rounds = 0;
  for (const int32_t i : order) {
    const Slot s = heap.top();
    heap.pop();
    lists[s.second].push_back(i);
    rounds = std::max(rounds, lists[s.second].size());
    heap.push({s.first + cost[i], s.second});
  }
  const int64_t total = static_cast<int64_t>(rounds) * ctas;
  if (total > INT32_MAX) return MF_ERR_INVALID_ARG;
  if (!sched) {
    *n_sched = static_cast<int32_t>(total);
    return MF_OK;
  }
  if (*n_sched < total) return MF_ERR_INVALID_ARG;
  for (size_t r = 0; r < rounds; ++r)
    for (int32_t c = 0; c < ctas; ++c)
      sched[r * ctas + c] = r < lists[c].size() ? work[lists[c][r]] : mf_work_item{0, 0, -1, 0};
  *n_sched = static_cast<int32_t>(total);
  return MF_OK;
}
