// Host-side plan object shared by the C entry points of liblags.so.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "lags.h"
#include "lags_internal.cuh"

struct lags_plan {
  int32_t L = 0, P = 0;
  uint64_t N0 = 0, N = 0, K = 0, C = 0;  // elements [N0, N) of the model; K picks per worker
  std::vector<lags::LayerDesc> layers;
  std::vector<lags::TileDesc> tiles;
  std::vector<uint32_t> sel_large, sel_small, sel_huge, sel_mid, sparse;
  std::vector<uint2> pick_chunks;  // (sparse layer, first slot) per 256 pick slots
  std::vector<uint2> agg_groups;   // (first tile, tiles) per aggregation CTA
  std::vector<int64_t> off, k, koff;
  // workspace sections (byte offsets)
  // (the sections aggregation uses come first: a workspace of agg_ws_bytes
  // serves a plan that only aggregates)
  size_t o_layers = 0, o_tiles = 0, o_large = 0, o_small = 0, o_huge = 0, o_mid = 0, o_sparse = 0,
         o_lo = 0,
         o_cnt = 0,
         o_cval = 0, o_cidx = 0, o_first = 0, o_chunks = 0, o_groups = 0, o_wrec = 0, o_wcnt = 0,
         o_status = 0,
         agg_ws_bytes = 0, ws_bytes = 0;
  void* ws = nullptr;
  bool ws_full = false;  // the bound workspace also serves lags_sparsify
  int device = -1;
  uint32_t stage_spin = lags::kSelectSpinLimit;  // polls of the select's first staging wait
  uint32_t index_spin = lags::kSelectSpinLimit;  // polls of the values-only index-copy wait
  cudaEvent_t ev_before = nullptr, ev_after = nullptr;
  uint32_t stage_small = 0, stage_large = 0, stage_huge = 0, stage_mid = 0;  // select staging per launch
  lags::DevPlan dp{};  // device view once a workspace is bound
};


// Device view of `plan` with its tables and scratch laid out at `base`
// (the workspace sections the plan computed).
inline void bind_dev_plan(const lags_plan* plan, char* base, lags::DevPlan* out) {
  using namespace lags;
  DevPlan& dp = *out;
  dp.layers = (const LayerDesc*)(base + plan->o_layers);
  dp.tiles = (const TileDesc*)(base + plan->o_tiles);
  dp.sel_large = (const uint32_t*)(base + plan->o_large);
  dp.sel_mid = (const uint32_t*)(base + plan->o_mid);
  dp.sel_small = (const uint32_t*)(base + plan->o_small);
  dp.sel_huge = (const uint32_t*)(base + plan->o_huge);
  dp.sparse = (const uint32_t*)(base + plan->o_sparse);
  dp.lo_key = (uint32_t*)(base + plan->o_lo);
  dp.tile_cnt = (uint32_t*)(base + plan->o_cnt);
  dp.cand_val = (float*)(base + plan->o_cval);
  dp.cand_idx = (uint32_t*)(base + plan->o_cidx);
  dp.pick_first = (uint32_t*)(base + plan->o_first);
  dp.pick_chunks = (const uint2*)(base + plan->o_chunks);
  dp.agg_groups = (const uint2*)(base + plan->o_groups);
  dp.wrec = (uint2*)(base + plan->o_wrec);
  dp.wcnt = (uint32_t*)(base + plan->o_wcnt);
  dp.status = (uint32_t*)(base + plan->o_status);
  dp.L = (uint32_t)plan->L;
  dp.T = (uint32_t)plan->tiles.size();
  dp.P = (uint32_t)plan->P;
  dp.n_large = (uint32_t)plan->sel_large.size();
  dp.n_mid = (uint32_t)plan->sel_mid.size();
  dp.n_small = (uint32_t)plan->sel_small.size();
  dp.n_huge = (uint32_t)plan->sel_huge.size();
  dp.n_sparse = (uint32_t)plan->sparse.size();
  dp.n_chunks = (uint32_t)plan->pick_chunks.size();
  dp.n_groups = (uint32_t)plan->agg_groups.size();
  dp.N = (uint32_t)plan->N;
  dp.K = plan->K;
  dp.C = plan->C;
  dp.stage_small = plan->stage_small;
  dp.stage_large = plan->stage_large;
  dp.stage_mid = plan->stage_mid;
  dp.stage_huge = plan->stage_huge;
  dp.stage_spin = plan->stage_spin;
  dp.index_spin = plan->index_spin;
}

// The status a poll returns for the flags it read: a timeout first (its picks
// may be incomplete), then a failed self-check, then malformed pick lists.
inline lags_status lags_status_of_flags(uint32_t flags) {
  if (flags & LAGS_FLAG_TIMEOUT) return LAGS_ERR_TIMEOUT;
  if (flags & LAGS_FLAG_INTERNAL) return LAGS_ERR_INTERNAL;
  if (flags & LAGS_FLAG_BAD_PICKS) return LAGS_ERR_BAD_PICKS;
  return LAGS_OK;
}
