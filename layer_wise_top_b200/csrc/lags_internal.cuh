// Internal declarations shared by the kernels and the C ABI of liblags.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "lags.h"

namespace lags {

// Elements per tile: the unit of the fused error-feedback pass, of candidate
// storage and of aggregation.  Tiles never cross a layer boundary; interior
// tile boundaries sit on multiples of kTile in the flattened buffer, so every
// tile but a layer's first and last is 16-byte aligned at both ends.
constexpr uint32_t kTile = 8192;
constexpr uint32_t kEfThreads = 256;                        // fused pass block
constexpr uint32_t kEfVecPerThread = kTile / 4 / kEfThreads;  // float4 per thread = 8

// Largest sample the threshold estimate draws per (worker, layer).
constexpr uint32_t kSampleMax = 16384;
// contiguous elements per sample run: short runs for segments longer than
// kSampleShortAbove (whole-model segments span tensors of different scales),
// long runs (fewer, larger reads) for the rest
constexpr uint32_t kSampleRunShort = 16;
constexpr uint32_t kSampleRunLong = 64;
constexpr uint32_t kSampleShortAbove = 1u << 23;
constexpr uint32_t kEstThreads = 512;

// Cluster size used to select layers whose expected candidates exceed what one
// CTA stages in shared memory; the other layers use one CTA.
constexpr int kSelectCluster = 8;
// Layers whose expected candidates 4 CTAs stage as values only (4 bytes each;
// the indices are read back from the candidate slots for the picks) use a
// 4-CTA cluster instead: twice the clusters resident of the 8-CTA launch.
constexpr int kSelectClusterMid = 4;
// Layers whose expected candidates exceed what 8 CTAs stage use a 16-CTA
// cluster (a non-portable size; checked on the device before use).
constexpr int kSelectClusterHuge = 16;
constexpr uint32_t kSelectThreads = 512;       // clustered select
constexpr uint32_t kSelectThreadsSmall = 512;  // single-CTA select (256 measured slower)
constexpr uint32_t kSelectWindow = 2048;  // tiles whose prefix sits in smem at once
// Candidates one selection CTA copies to shared memory (sized per launch from
// the expected candidate counts, at most kSelectStageMax); a CTA with more
// reads them from global memory on every pass instead.
constexpr uint32_t kSelectStageMin = 1024;
constexpr uint32_t kSelectStageMax = 20480;  // multiple of 4 (16-byte staged runs)
// Values-only stage of the 4-CTA launch: two CTAs per SM with the kernel's
// static shared memory (multiple of 256).
constexpr uint32_t kSelectStageMaxValues = 17408;
constexpr uint32_t kSelectSpinLimit = LAGS_STAGE_WAIT_POLLS;  // polls of the staging mbarrier


// Picks of one aggregation group staged in shared memory (more: the group
// takes the worker-ordered accumulation path, reading them from global memory).
constexpr uint32_t kAggPickCap = 2048;

// Radix digits of the magnitude key (bits 30..0 of the fp32 pattern).
constexpr int kDigitShift0 = 20;  // level 0: bits 30..20, 2048 bins
constexpr int kDigitShift1 = 9;   // level 1: bits 19..9,  2048 bins
constexpr int kDigitShift2 = 0;   // level 2: bits 8..0,    512 bins
constexpr uint32_t kBins = 2048;

struct LayerDesc {
  uint32_t off;         // first element in a worker buffer
  uint32_t d;           // elements
  uint32_t k;           // picks
  uint32_t koff;        // first slot of this layer's picks in a worker pick list
  uint32_t tile_begin;  // first tile id
  uint32_t tile_end;    // one past the last tile id
  uint32_t slot_cap;    // candidate slots per tile (0: dense layer)
  uint32_t slot_base;   // first candidate slot of the layer in a worker region
  uint32_t sample;      // threshold-estimate sample size m_l
  uint32_t rank;        // sample rank r*_l that sets the candidate threshold
  uint32_t pad0, pad1;
};
static_assert(sizeof(LayerDesc) == 48, "LayerDesc layout");

struct TileDesc {
  uint32_t start;  // first element (flattened index)
  uint32_t len;    // elements, 1..kTile
  uint32_t layer;
  uint32_t pad;
};
static_assert(sizeof(TileDesc) == 16, "TileDesc layout");

// Worker buffers, passed by value in the launch arguments.
struct WorkerPtrs {
  const float* g[LAGS_MAX_WORKERS];
  float* r[LAGS_MAX_WORKERS];
};

// Gradient buffers of the dense S-SGD baseline, one per worker.
struct DenseGrads {
  const float* g[LAGS_MAX_WORKERS];
};

// Device status words (in the workspace).
enum StatusWord : uint32_t { kStatusFlags = 0, kStatusFallbacks = 1, kStatusWords = 64 };

// Device-side view of a plan with its workspace bound.
struct DevPlan {
  const LayerDesc* layers;
  const TileDesc* tiles;
  const uint32_t* sel_large;  // sparse layers selected by an 8-CTA cluster
  const uint32_t* sel_mid;    // sparse layers selected by a 4-CTA cluster (values staged)
  const uint32_t* sel_huge;   // sparse layers selected by a 16-CTA cluster
  const uint32_t* sel_small;  // sparse layers selected by one CTA
  const uint32_t* sparse;     // all sparse layers (estimate pass)
  uint32_t* lo_key;           // [P][L] candidate threshold key
  uint32_t* tile_cnt;         // [P][T] candidates found per tile
  float* cand_val;            // [P][C]
  uint32_t* cand_idx;         // [P][C]
  uint32_t* pick_first;       // [P][T] first pick slot of each tile (aggregate)
  const uint2* pick_chunks;   // (sparse layer, first slot) per 256 pick slots
  const uint2* agg_groups;    // (first tile, tiles) per aggregation CTA
  uint2* wrec;                // [groups][kAggPickCap] (position, quotient) weight updates
  uint32_t* wcnt;             // [groups] records of each group (0: none)
  uint32_t* status;           // kStatusWords
  uint32_t L, T, P;
  uint32_t n_large, n_small, n_huge, n_mid, n_sparse, n_chunks, n_groups;
  uint32_t N;
  uint64_t K;
  uint64_t C;  // candidate slots per worker
  uint32_t stage_small, stage_large, stage_huge, stage_mid;  // select staging per launch
  uint32_t stage_spin;    // polls of the select's first staging wait before it gives up
  uint32_t index_spin;    // polls of the values-only select's index-copy wait
};

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_estimate(const DevPlan& dp, const WorkerPtrs& wp, float lr, cudaStream_t s);
cudaError_t launch_ef_capture(const DevPlan& dp, const WorkerPtrs& wp, float lr,
                              uint32_t* out_idx, float* out_val, cudaStream_t s);
cudaError_t launch_select(const DevPlan& dp, const WorkerPtrs& wp, uint32_t* out_idx,
                          float* out_val, cudaStream_t s);
cudaError_t launch_pick_bounds(const DevPlan& dp, const uint32_t* idx, cudaStream_t s);
cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, float* weights, cudaStream_t s);
cudaError_t launch_apply(uint32_t first, uint32_t end, float* w, const float* dense, cudaStream_t s);
cudaError_t launch_weight_updates(const DevPlan& dp, float* weights, cudaStream_t s);
cudaError_t launch_dense_sum(const DenseGrads& gp, uint32_t P, uint64_t N, float lr, float* sum,
                             cudaStream_t s);
cudaError_t launch_dense_finish(const float* sum, uint64_t N, uint32_t P, float* dense,
                                float* weights, cudaStream_t s);


// ------------------------------------------------------------------ launches
// Programmatic dependent launch: each kernel of a step is launched so that it
// may be scheduled while its predecessor's last CTAs still run.  Every kernel
// lets its dependents launch as soon as it starts (pdl_trigger) and waits for
// its predecessor to complete, with memory visible, before touching anything
// the predecessor may have written (pdl_wait).  Plan tables are written only
// by lags_plan_set_workspace and may be read before the wait.  Launched
// without the attribute, both are no-ops.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Data the step's earlier kernels wrote must be read after pdl_wait().  Loads
// through the read-only path (__ldg) are invariant to the compiler, and the
// cache-hinted loads are asm without a memory clobber, so either may be moved
// above the wait; a plain "memory" clobber does not hold them.  Every kernel
// therefore reads such data through pointers passed through after_wait()
// behind its pdl_wait(): the compiler learns their value only there, so no
// load through them can be issued before the wait.
template <typename T>
__device__ __forceinline__ T* after_wait(T* p) {
  uint64_t v = reinterpret_cast<uint64_t>(p);
  asm volatile("" : "+l"(v));
  return reinterpret_cast<T*>(v);
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t mag_key(float x) {
  return __float_as_uint(x) & 0x7FFFFFFFu;
}

}  // namespace lags
