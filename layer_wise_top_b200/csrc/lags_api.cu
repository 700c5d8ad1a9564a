// C ABI of liblags.so: plan construction (host), workspace binding, argument
// validation and the launches.  See include/lags.h for the contract.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "lags.h"
#include "lags_internal.cuh"
#include "lags_plan.cuh"

namespace lags {
cudaError_t configure_estimate();
cudaError_t configure_select();
cudaError_t configure_aggregate();
}  // namespace lags

using namespace lags;

namespace {

constexpr size_t kAlign = 256;

size_t section(size_t& cursor, size_t bytes) {
  size_t at = (cursor + kAlign - 1) / kAlign * kAlign;
  cursor = at + bytes;
  return at;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Candidate slots per tile for a layer of d entries split in `ntiles` tiles,
// expecting `cand` candidates: six times a tile's share (candidates spread
// evenly), or up to 24 times it (and at most 1.5x the layer's expected total)
// when the large values crowd into a few tiles, e.g. a segment spanning
// tensors of different gradient scales; plus 64, in warp multiples.
uint32_t slot_capacity(uint64_t d, uint64_t ntiles, double cand) {
  const double share = cand * std::min<double>(kTile, (double)d) / (double)d;
  const double spread = 6.0 * share;
  const double crowded = std::min(1.5 * cand, 24.0 * cand / (double)ntiles);
  const double cap = std::ceil(std::max(spread, crowded)) + 64.0;
  uint64_t c = ((uint64_t)cap + 31) / 32 * 32;
  return (uint32_t)(c < kTile ? c : kTile);
}

// Sample rank r* for a sample of m entries out of d, k picks: the expected
// number mu of sampled entries above the k-th largest, plus four standard
// deviations and a floor of 6, so the threshold it sets keeps the k largest
// entries with overwhelming probability.  A whole-layer sample uses r* = k.
uint32_t sample_rank(uint64_t m, uint64_t d, uint64_t k) {
  if (m == d) return (uint32_t)k;
  double mu = (double)m * (double)k / (double)d;
  double r = std::ceil(mu + 4.0 * std::sqrt(mu) + 6.0);
  if (r > (double)m) r = (double)m;
  if (r < 1.0) r = 1.0;
  return (uint32_t)r;
}

// Candidates the fused pass is expected to keep for a layer: its sample rank
// scaled from the sample to the layer (exactly k when the sample is the layer).
double expected_candidates(const LayerDesc& ld) {
  if (ld.sample == ld.d) return (double)ld.k;
  return std::ceil((double)ld.rank * ld.d / ld.sample);
}

lags_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LAGS_OK : LAGS_ERR_CUDA; }

// Calls that enqueue work on a plan's workspace run on the device it was bound on.
lags_status check_device(const lags_plan* plan) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LAGS_ERR_CUDA;
  return dev == plan->device ? LAGS_OK : LAGS_ERR_WRONG_DEVICE;
}

bool fill_workers(const lags_plan* plan, const float* const* grads, float* const* residuals,
                  WorkerPtrs* wp, lags_status* err) {
  std::memset(wp, 0, sizeof(*wp));
  for (int p = 0; p < plan->P; ++p) {
    if (!grads[p] || !residuals[p]) {
      *err = LAGS_ERR_INVALID_ARG;
      return false;
    }
    if (!aligned(grads[p], 16) || !aligned(residuals[p], 16)) {
      *err = LAGS_ERR_ALIGNMENT;
      return false;
    }
    wp->g[p] = grads[p];
    wp->r[p] = residuals[p];
  }
  return true;
}

}  // namespace

extern "C" {

lags_status lags_plan_create(const int64_t* layer_sizes, const double* densities,
                             int32_t num_layers, int32_t num_workers, lags_plan** out_plan) {
  return lags_plan_create_range(layer_sizes, densities, num_layers, num_workers, 0, num_layers,
                                out_plan);
}

lags_status lags_plan_create_range(const int64_t* layer_sizes, const double* densities,
                                   int32_t num_layers, int32_t num_workers, int32_t layer_begin,
                                   int32_t layer_end, lags_plan** out_plan) {
  if (!out_plan) return LAGS_ERR_INVALID_ARG;
  *out_plan = nullptr;
  if (!layer_sizes || !densities || num_layers < 1 || num_layers > (1 << 24) ||
      num_workers < 1 || num_workers > LAGS_MAX_WORKERS || layer_begin < 0 ||
      layer_end <= layer_begin || layer_end > num_layers)
    return LAGS_ERR_INVALID_ARG;
  // element offsets are those of the whole model: skip the layers before the range
  uint64_t off = 0;
  for (int32_t l = 0; l < layer_begin; ++l) {
    if (layer_sizes[l] <= 0) return LAGS_ERR_INVALID_ARG;
    off += (uint64_t)layer_sizes[l];
    if (off > LAGS_MAX_ELEMENTS) return LAGS_ERR_INVALID_ARG;
  }
  lags_plan* plan = new (std::nothrow) lags_plan();
  if (!plan) return LAGS_ERR_INVALID_ARG;
  plan->L = layer_end - layer_begin;
  plan->P = num_workers;
  plan->N0 = off;
  uint64_t koff = 0, slots = 0;
  for (int32_t l = 0; l < plan->L; ++l) {
    const int64_t d = layer_sizes[layer_begin + l];
    const double rho = densities[layer_begin + l];
    if (d <= 0 || !(rho > 0.0) || !(rho <= 1.0)) {
      delete plan;
      return LAGS_ERR_INVALID_ARG;
    }
    double kd = std::ceil(rho * (double)d);
    uint64_t k = kd < 1.0 ? 1 : (kd >= (double)d ? (uint64_t)d : (uint64_t)kd);
    if (off + (uint64_t)d > LAGS_MAX_ELEMENTS) {  // indices are uint32, with headroom
      delete plan;
      return LAGS_ERR_INVALID_ARG;
    }
    LayerDesc ld{};
    ld.off = (uint32_t)off;
    ld.d = (uint32_t)d;
    ld.k = (uint32_t)k;
    ld.koff = (uint32_t)koff;
    ld.tile_begin = (uint32_t)plan->tiles.size();
    const uint64_t j0 = off / kTile, j1 = (off + d - 1) / kTile;
    for (uint64_t j = j0; j <= j1; ++j) {
      uint64_t s = j * kTile > off ? j * kTile : off;
      uint64_t e = (j + 1) * kTile < off + d ? (j + 1) * kTile : off + d;
      TileDesc td{(uint32_t)s, (uint32_t)(e - s), (uint32_t)l, 0};
      plan->tiles.push_back(td);
    }
    ld.tile_end = (uint32_t)plan->tiles.size();
    const bool dense = k == (uint64_t)d;
    if (!dense) {
      ld.sample = (uint32_t)((uint64_t)d < kSampleMax ? d : kSampleMax);
      ld.rank = sample_rank(ld.sample, d, k);
      ld.slot_cap = slot_capacity(d, ld.tile_end - ld.tile_begin, expected_candidates(ld));
      ld.slot_base = (uint32_t)slots;
      slots += (uint64_t)(ld.tile_end - ld.tile_begin) * ld.slot_cap;
      plan->sparse.push_back((uint32_t)l);
      for (uint64_t j0 = 0; j0 < k; j0 += 256) plan->pick_chunks.push_back(make_uint2(l, j0));
      // one CTA when its shared memory can stage the expected candidates with
      // a third to spare, else a 4-CTA cluster staging values only, else an
      // 8-CTA cluster, else a 16-CTA cluster
      const double expect = expected_candidates(ld);
      auto fits = [&](int ctas) { return 1.33 * expect / ctas + 512.0 <= (double)kSelectStageMax; };
      const bool fits_values =
          1.33 * expect / kSelectClusterMid + 512.0 <= (double)kSelectStageMaxValues &&
          (ld.tile_end - ld.tile_begin + kSelectClusterMid - 1) / kSelectClusterMid <= kSelectWindow;
      (fits(1)         ? plan->sel_small
       : fits_values   ? plan->sel_mid
       : fits(kSelectCluster) ? plan->sel_large
                              : plan->sel_huge)
          .push_back((uint32_t)l);
    }
    if (slots >= (1ull << 32) || koff + k >= (1ull << 32)) {
      delete plan;
      return LAGS_ERR_INVALID_ARG;
    }
    plan->layers.push_back(ld);
    plan->off.push_back((int64_t)off);
    plan->k.push_back((int64_t)k);
    plan->koff.push_back((int64_t)koff);
    off += (uint64_t)d;
    koff += k;
  }
  // 4-CTA clusters only pay when their launch fills the GPU (one CTA per SM
  // at least); fewer clusters keep more CTAs per layer with 8-CTA clusters
  // (VGG-16's whole-model segments: 0.742 vs 0.631 ms per step)
  if (!plan->sel_mid.empty() &&
      plan->sel_mid.size() * (uint64_t)num_workers * kSelectClusterMid < 148) {
    plan->sel_large.insert(plan->sel_large.end(), plan->sel_mid.begin(), plan->sel_mid.end());
    plan->sel_mid.clear();
  }
  // staging capacity of each select launch: 1.5x the largest expected
  // candidate count of one CTA (the sample rank scaled to the layer) plus 512
  auto stage_for = [plan, num_workers](const std::vector<uint32_t>& list, uint32_t ctas,
                                       uint32_t most_entries) {
    double most = 0.0;
    for (uint32_t l : list) {
      const LayerDesc& ld = plan->layers[l];
      const double tiles = std::ceil((double)(ld.tile_end - ld.tile_begin) / ctas);
      // staged runs are padded to multiples of 4 entries: up to 3 per tile
      most = std::max(most, 1.5 * expected_candidates(ld) / ctas + 3.0 * tiles);
    }
    uint64_t cap = ((uint64_t)std::ceil(most + 512.0) + 255) / 256 * 256;
    // a launch whose CTAs all run at once with one per SM (148 SMs) gives each
    // the largest stage at no cost: crowded segments (a global top-k over
    // tensors of different scales) then stay on the candidate lists
    if ((uint64_t)list.size() * ctas * (uint64_t)num_workers <= 148) cap = most_entries;
    return (uint32_t)std::min<uint64_t>(std::max<uint64_t>(cap, kSelectStageMin), most_entries);
  };
  plan->stage_small = stage_for(plan->sel_small, 1, kSelectStageMax);
  plan->stage_mid = stage_for(plan->sel_mid, kSelectClusterMid, kSelectStageMaxValues);
  plan->stage_large = stage_for(plan->sel_large, kSelectCluster, kSelectStageMax);
  plan->stage_huge = stage_for(plan->sel_huge, kSelectClusterHuge, kSelectStageMax);
  // aggregation groups: consecutive tiles of one layer, about a thousand
  // expected picks (P k / d per element) per group and at most 16 tiles, but
  // never so few groups that the GPU has fewer than 8 per SM (grouping only
  // pays when tiles far outnumber the CTAs that run at once); tiles expected
  // to need the shared tile accumulator stay alone
  {
    const double cap_by_count =
        std::max(1.0, std::floor((double)plan->tiles.size() / (8.0 * 148.0)));
    for (const LayerDesc& ld : plan->layers) {
      const bool dense_l = ld.k == ld.d;
      const double per_tile =
          dense_l ? 0.0 : (double)num_workers * ld.k * std::min<double>(kTile, ld.d) / ld.d;
      double g = dense_l ? 4.0 : per_tile > 256.0 ? 1.0 : 1024.0 / std::max(per_tile, 1.0);
      g = std::max(1.0, std::min({g, 16.0, cap_by_count}));
      const uint32_t gi = (uint32_t)g;
      for (uint32_t t0 = ld.tile_begin; t0 < ld.tile_end; t0 += gi)
        plan->agg_groups.push_back(make_uint2(t0, std::min(gi, ld.tile_end - t0)));
    }
  }
  // select the layers with the most picks first, so the longest CTAs start early
  auto by_k_desc = [plan](uint32_t a, uint32_t b) {
    return plan->layers[a].k != plan->layers[b].k ? plan->layers[a].k > plan->layers[b].k : a < b;
  };
  std::sort(plan->sel_large.begin(), plan->sel_large.end(), by_k_desc);
  std::sort(plan->sel_mid.begin(), plan->sel_mid.end(), by_k_desc);
  std::sort(plan->sel_huge.begin(), plan->sel_huge.end(), by_k_desc);
  std::sort(plan->sel_small.begin(), plan->sel_small.end(), by_k_desc);
  std::sort(plan->sparse.begin(), plan->sparse.end(), by_k_desc);
  plan->N = off;
  plan->K = koff;
  plan->C = slots;
  const uint64_t P = (uint64_t)num_workers, T = plan->tiles.size();
  size_t cur = 0;
  // what aggregation reads: tables, per-tile first picks, status words
  plan->o_layers = section(cur, plan->layers.size() * sizeof(LayerDesc));
  plan->o_tiles = section(cur, T * sizeof(TileDesc));
  plan->o_chunks = section(cur, (plan->pick_chunks.size() + 1) * sizeof(uint2));
  plan->o_groups = section(cur, (plan->agg_groups.size() + 1) * sizeof(uint2));
  plan->o_first = section(cur, P * T * 4);
  plan->o_wrec = section(cur, plan->agg_groups.size() * (size_t)kAggPickCap * sizeof(uint2));
  plan->o_wcnt = section(cur, (plan->agg_groups.size() + 1) * 4);
  plan->o_status = section(cur, kStatusWords * 4);
  plan->agg_ws_bytes = (cur + kAlign - 1) / kAlign * kAlign;
  // what only the selection reads
  plan->o_large = section(cur, (plan->sel_large.size() + 1) * 4);
  plan->o_mid = section(cur, (plan->sel_mid.size() + 1) * 4);
  plan->o_small = section(cur, (plan->sel_small.size() + 1) * 4);
  plan->o_huge = section(cur, (plan->sel_huge.size() + 1) * 4);
  plan->o_sparse = section(cur, (plan->sparse.size() + 1) * 4);
  plan->o_lo = section(cur, P * (uint64_t)plan->L * 4);
  plan->o_cnt = section(cur, P * T * 4);
  plan->o_cval = section(cur, P * (plan->C + 1) * 4);
  plan->o_cidx = section(cur, P * (plan->C + 1) * 4);
  plan->ws_bytes = (cur + kAlign - 1) / kAlign * kAlign;
  *out_plan = plan;
  return LAGS_OK;
}

lags_status lags_plan_destroy(lags_plan* plan) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  delete plan;
  return LAGS_OK;
}

lags_status lags_plan_info(const lags_plan* plan, int64_t* N, int64_t* K,
                           size_t* workspace_bytes) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  if (N) *N = (int64_t)plan->N;
  if (K) *K = (int64_t)plan->K;
  if (workspace_bytes) *workspace_bytes = plan->ws_bytes;
  return LAGS_OK;
}

lags_status lags_plan_aggregate_workspace_bytes(const lags_plan* plan, size_t* bytes) {
  if (!plan || !bytes) return LAGS_ERR_INVALID_ARG;
  *bytes = plan->agg_ws_bytes;
  return LAGS_OK;
}

lags_status lags_plan_layer(const lags_plan* plan, int32_t l, int64_t* offset, int64_t* k,
                            int64_t* pick_offset) {
  if (!plan || l < 0 || l >= plan->L) return LAGS_ERR_INVALID_ARG;
  if (offset) *offset = plan->off[l];
  if (k) *k = plan->k[l];
  if (pick_offset) *pick_offset = plan->koff[l];
  return LAGS_OK;
}

lags_status lags_plan_set_workspace(lags_plan* plan, void* workspace, size_t bytes,
                                    void* stream) {
  if (!plan || !workspace) return LAGS_ERR_INVALID_ARG;
  if (!aligned(workspace, kAlign)) return LAGS_ERR_ALIGNMENT;
  if (bytes < plan->agg_ws_bytes) return LAGS_ERR_WORKSPACE;
  const bool full = bytes >= plan->ws_bytes;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LAGS_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return LAGS_ERR_CUDA;
  if (major != 10 || minor != 0) return LAGS_ERR_UNSUPPORTED_DEVICE;
  if (configure_estimate() != cudaSuccess || configure_select() != cudaSuccess ||
      configure_aggregate() != cudaSuccess)
    return LAGS_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  char* base = (char*)workspace;
  auto up = [&](size_t o, const void* src, size_t n) {
    return n ? cudaMemcpyAsync(base + o, src, n, cudaMemcpyHostToDevice, s) : cudaSuccess;
  };
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = up(plan->o_layers, plan->layers.data(), plan->layers.size() * sizeof(LayerDesc));
  if (e == cudaSuccess) e = up(plan->o_tiles, plan->tiles.data(), plan->tiles.size() * sizeof(TileDesc));
  if (full) {
    if (e == cudaSuccess) e = up(plan->o_large, plan->sel_large.data(), plan->sel_large.size() * 4);
    if (e == cudaSuccess) e = up(plan->o_mid, plan->sel_mid.data(), plan->sel_mid.size() * 4);
    if (e == cudaSuccess) e = up(plan->o_small, plan->sel_small.data(), plan->sel_small.size() * 4);
    if (e == cudaSuccess) e = up(plan->o_huge, plan->sel_huge.data(), plan->sel_huge.size() * 4);
    if (e == cudaSuccess) e = up(plan->o_sparse, plan->sparse.data(), plan->sparse.size() * 4);
  }
  if (e == cudaSuccess)
    e = up(plan->o_chunks, plan->pick_chunks.data(), plan->pick_chunks.size() * sizeof(uint2));
  if (e == cudaSuccess)
    e = up(plan->o_groups, plan->agg_groups.data(), plan->agg_groups.size() * sizeof(uint2));
  if (e == cudaSuccess) e = cudaMemsetAsync(base + plan->o_status, 0, kStatusWords * 4, s);
  // pageable sources: make sure the copies are done before returning
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LAGS_ERR_CUDA;
  bind_dev_plan(plan, base, &plan->dp);
  plan->ws = workspace;
  plan->ws_full = full;
  plan->device = dev;
  return LAGS_OK;
}

lags_status lags_sparsify(lags_plan* plan, const float* const* grads, float* const* residuals,
                          float lr, uint32_t* out_idx, float* out_val, void* stream) {
  if (!plan || !grads || !residuals || !out_idx || !out_val) return LAGS_ERR_INVALID_ARG;
  if (!plan->ws || !plan->ws_full) return LAGS_ERR_WORKSPACE;
  if (!aligned(out_idx, 4) || !aligned(out_val, 4)) return LAGS_ERR_ALIGNMENT;
  WorkerPtrs wp;
  lags_status err = LAGS_OK;
  if (!fill_workers(plan, grads, residuals, &wp, &err)) return err;
  if ((err = check_device(plan)) != LAGS_OK) return err;
  cudaStream_t s = (cudaStream_t)stream;
  const bool timed = plan->ev_before && plan->ev_after;
  // under stream capture the timing events become event-record nodes of the
  // graph (recorded at every replay) instead of capture-internal markers
  unsigned rec_flags = cudaEventRecordDefault;
  if (timed) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return LAGS_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusActive) rec_flags = cudaEventRecordExternal;
  }
  cudaError_t e = launch_estimate(plan->dp, wp, lr, s);
  if (e == cudaSuccess && timed) e = cudaEventRecordWithFlags(plan->ev_before, s, rec_flags);
  if (e == cudaSuccess) e = launch_ef_capture(plan->dp, wp, lr, out_idx, out_val, s);
  if (e == cudaSuccess && timed) e = cudaEventRecordWithFlags(plan->ev_after, s, rec_flags);
  if (e == cudaSuccess) e = launch_select(plan->dp, wp, out_idx, out_val, s);
  return cuda_status(e);
}

lags_status lags_aggregate(lags_plan* plan, const uint32_t* idx, const float* val,
                           float* dense_out, void* stream) {
  if (!plan || !idx || !val || !dense_out) return LAGS_ERR_INVALID_ARG;
  if (!plan->ws) return LAGS_ERR_WORKSPACE;
  if (!aligned(idx, 4) || !aligned(val, 4) || !aligned(dense_out, 16)) return LAGS_ERR_ALIGNMENT;
  const lags_status dev_ok = check_device(plan);
  if (dev_ok != LAGS_OK) return dev_ok;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_pick_bounds(plan->dp, idx, s);
  if (e == cudaSuccess) e = launch_aggregate(plan->dp, idx, val, dense_out, nullptr, s);
  return cuda_status(e);
}

lags_status lags_aggregate_apply(lags_plan* plan, const uint32_t* idx, const float* val,
                                 float* dense_out, float* weights, void* stream) {
  if (!plan || !idx || !val || !dense_out || !weights) return LAGS_ERR_INVALID_ARG;
  if (!plan->ws) return LAGS_ERR_WORKSPACE;
  if (!aligned(idx, 4) || !aligned(val, 4) || !aligned(dense_out, 16) || !aligned(weights, 16))
    return LAGS_ERR_ALIGNMENT;
  const lags_status dev_ok = check_device(plan);
  if (dev_ok != LAGS_OK) return dev_ok;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_pick_bounds(plan->dp, idx, s);
  if (e == cudaSuccess) e = launch_aggregate(plan->dp, idx, val, dense_out, weights, s);
  if (e == cudaSuccess) e = launch_weight_updates(plan->dp, weights, s);
  return cuda_status(e);
}

lags_status lags_adaptive_densities(const int64_t* layer_sizes, const double* backward_seconds,
                                    int32_t num_layers, double alpha, double beta,
                                    double rho_min, double* out_densities) {
  if (!layer_sizes || !backward_seconds || !out_densities || num_layers < 1) return LAGS_ERR_INVALID_ARG;
  if (!(alpha >= 0.0) || !(beta >= 0.0) || !(rho_min > 0.0) || !(rho_min <= 1.0))
    return LAGS_ERR_INVALID_ARG;
  double end = 0.0;  // R_0: the backward pass ends after every layer
  for (int32_t l = 0; l < num_layers; ++l) {
    if (layer_sizes[l] <= 0 || !(backward_seconds[l] >= 0.0)) return LAGS_ERR_INVALID_ARG;
    end += backward_seconds[l];
  }
  double produced = 0.0, link_free = 0.0;
  for (int32_t l = num_layers - 1; l >= 0; --l) {
    produced += backward_seconds[l];  // R_l = sum_{j >= l} t_j
    const double start = std::max(produced, link_free);
    const double d = (double)layer_sizes[l];
    const double budget = end - start - alpha;  // seconds left for 8 k beta
    double rho = rho_min;
    if (budget >= 0.0) {
      const double kmax = beta > 0.0 ? std::floor(budget / (8.0 * beta)) : d;
      rho = std::min(1.0, std::max(rho_min, kmax / d));
    }
    // the k this density yields (the rule of lags_plan_create), for the link
    const double kd = std::ceil(rho * d);
    const double k = kd < 1.0 ? 1.0 : std::min(kd, d);
    out_densities[l] = rho;
    link_free = start + alpha + beta * 8.0 * k;
  }
  return LAGS_OK;
}

lags_status lags_merge_layers(const int64_t* message_bytes, const double* backward_seconds,
                              int32_t num_layers, double alpha, double beta,
                              int32_t* out_bucket_first, int32_t* out_num_buckets,
                              double* out_end_seconds) {
  if (!message_bytes || !backward_seconds || !out_bucket_first || !out_num_buckets ||
      num_layers < 1 || num_layers > (1 << 20) || !(alpha >= 0.0) || !(beta >= 0.0))
    return LAGS_ERR_INVALID_ARG;
  const int32_t L = num_layers;
  // ready[l]: the backward pass has produced layers L-1 .. l (it runs downwards)
  std::vector<double> ready(L + 1, 0.0);
  for (int32_t l = L - 1; l >= 0; --l) {
    if (message_bytes[l] < 0 || !(backward_seconds[l] >= 0.0)) return LAGS_ERR_INVALID_ARG;
    ready[l] = ready[l + 1] + backward_seconds[l];
  }
  // best[i]: earliest time at which messages covering layers [i, L) can have
  // been sent, over all ways of cutting them into buckets of consecutive
  // layers; a bucket [i, j) is one message of alpha + beta * bytes that starts
  // once layer i is produced and the previous message (layers [j, L)) is done.
  // Since that start time only grows with the previous end time, the best cut
  // of [i, L) extends a best cut of some [j, L): best[i] = min over j, O(L^2)
  // in all.  Equal end times go to the longer bucket.
  std::vector<double> best(L + 1, 0.0);
  std::vector<int32_t> next(L + 1, L);
  for (int32_t i = L - 1; i >= 0; --i) {
    double bytes = 0.0;
    for (int32_t j = i + 1; j <= L; ++j) {
      bytes += (double)message_bytes[j - 1];
      const double end = std::max(ready[i], best[j]) + alpha + beta * bytes;
      if (j == i + 1 || end <= best[i]) {
        best[i] = end;
        next[i] = j;
      }
    }
  }
  int32_t nb = 0;
  for (int32_t i = 0; i < L; i = next[i]) out_bucket_first[nb++] = i;
  *out_num_buckets = nb;
  if (out_end_seconds) *out_end_seconds = best[0];
  return LAGS_OK;
}

lags_status lags_dense_sum(const float* const* grads, int32_t num_workers, int64_t N, float lr,
                           float* sum_out, void* stream) {
  if (!grads || !sum_out || num_workers < 1 || num_workers > LAGS_MAX_WORKERS || N < 1)
    return LAGS_ERR_INVALID_ARG;
  if (!aligned(sum_out, 16)) return LAGS_ERR_ALIGNMENT;
  DenseGrads gp;
  std::memset(&gp, 0, sizeof(gp));
  for (int32_t p = 0; p < num_workers; ++p) {
    if (!grads[p]) return LAGS_ERR_INVALID_ARG;
    if (!aligned(grads[p], 16)) return LAGS_ERR_ALIGNMENT;
    gp.g[p] = grads[p];
  }
  return cuda_status(launch_dense_sum(gp, (uint32_t)num_workers, (uint64_t)N, lr, sum_out,
                                      (cudaStream_t)stream));
}

lags_status lags_dense_finish(const float* sum, int64_t N, int32_t num_workers_total,
                              float* dense_out, float* weights, void* stream) {
  if (!sum || !dense_out || N < 1 || num_workers_total < 1) return LAGS_ERR_INVALID_ARG;
  if (!aligned(sum, 16) || !aligned(dense_out, 16) || (weights && !aligned(weights, 16)))
    return LAGS_ERR_ALIGNMENT;
  return cuda_status(launch_dense_finish(sum, (uint64_t)N, (uint32_t)num_workers_total,
                                         dense_out, weights, (cudaStream_t)stream));
}

lags_status lags_plan_kernel_launches(const lags_plan* plan, int32_t* sparsify,
                                      int32_t* aggregate, int32_t* apply) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  const bool any_sparse = !plan->sparse.empty();
  if (sparsify)
    *sparsify = (any_sparse ? 1 : 0) + 1 + (plan->sel_small.empty() ? 0 : 1) +
                (plan->sel_large.empty() ? 0 : 1) + (plan->sel_huge.empty() ? 0 : 1) +
                (plan->sel_mid.empty() ? 0 : 1);
  if (aggregate) *aggregate = 3;  // (lags_aggregate_apply; lags_aggregate enqueues 2)
  if (apply) *apply = 1;
  return LAGS_OK;
}

lags_status lags_apply(const lags_plan* plan, float* weights, const float* dense_out,
                       void* stream) {
  if (!plan || !weights || !dense_out) return LAGS_ERR_INVALID_ARG;
  if (!aligned(weights, 16) || !aligned(dense_out, 16)) return LAGS_ERR_ALIGNMENT;
  if (plan->device >= 0) {  // (apply reads no workspace; a bound plan keeps its device)
    const lags_status dev_ok = check_device(plan);
    if (dev_ok != LAGS_OK) return dev_ok;
  }
  return cuda_status(launch_apply((uint32_t)plan->N0, (uint32_t)plan->N, weights, dense_out,
                                  (cudaStream_t)stream));
}

lags_status lags_plan_set_events(lags_plan* plan, void* before, void* after) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  const bool on = before && after;
  plan->ev_before = on ? (cudaEvent_t)before : nullptr;
  plan->ev_after = on ? (cudaEvent_t)after : nullptr;
  return LAGS_OK;
}

lags_status lags_plan_set_stage_wait_limit(lags_plan* plan, uint32_t polls) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  plan->stage_spin = polls;
  plan->dp.stage_spin = polls;
  return LAGS_OK;
}

lags_status lags_plan_set_index_wait_limit(lags_plan* plan, uint32_t polls) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  plan->index_spin = polls;
  plan->dp.index_spin = polls;
  return LAGS_OK;
}

lags_status lags_status_poll(lags_plan* plan, uint32_t* flags, uint32_t* exact_fallbacks,
                             void* stream) {
  if (!plan) return LAGS_ERR_INVALID_ARG;
  if (!plan->ws) return LAGS_ERR_WORKSPACE;
  const lags_status dev_ok = check_device(plan);
  if (dev_ok != LAGS_OK) return dev_ok;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t words[2] = {0, 0};
  uint32_t* dev = plan->dp.status;
  cudaError_t e = cudaMemcpyAsync(words, dev, sizeof(words), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dev, 0, sizeof(words), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LAGS_ERR_CUDA;
  if (flags) *flags = words[kStatusFlags];
  if (exact_fallbacks) *exact_fallbacks = words[kStatusFallbacks];
  return lags_status_of_flags(words[kStatusFlags]);
}

const char* lags_error_string(lags_status status) {
  switch (status) {
    case LAGS_OK: return "ok";
    case LAGS_ERR_INVALID_ARG: return "invalid argument";
    case LAGS_ERR_ALIGNMENT: return "device pointer not aligned as required";
    case LAGS_ERR_CUDA: return "CUDA runtime error";
    case LAGS_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
    case LAGS_ERR_WORKSPACE: return "workspace missing or too small";
    case LAGS_ERR_BAD_PICKS: return "pick list not ascending or outside its layer";
    case LAGS_ERR_TIMEOUT:
      return "a kernel's bounded wait on its own copies gave up; picks may be incomplete";
    case LAGS_ERR_INTERNAL: return "a kernel failed a self-check (library bug)";
    case LAGS_ERR_WRONG_DEVICE: return "the current device is not the plan's device";
  }
  return "unknown status";
}

}  // extern "C"
