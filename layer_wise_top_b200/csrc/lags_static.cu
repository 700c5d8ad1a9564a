// lags_sparsify_static: lags_sparsify without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they call the
// library: code running inside a custom allocator or memory-pool callback,
// runtimes that own every device allocation and forbid side allocations, and
// hosts that reserve the device up front and forbid cudaMalloc afterwards.
// For them this entry point keeps its scratch (the plan tables, the sampled
// thresholds, the per-tile candidate counts and the candidate slots) in one
// array with static storage that is part of the library image on each device.
//
//  - Limit: a plan whose workspace exceeds kStaticPlanBytes (16 MiB less the
//    status block at the end of the array) is rejected with
//    LAGS_ERR_WORKSPACE before anything is enqueued.
//  - Every GPU on which the array is loaded holds its 16 MiB until the
//    process exits.
//  - All calls share the one array and it keeps the last call's contents:
//    each call re-uploads its plan's tables, and everything the kernels need
//    zeroed is written by them before it is read.  Calls whose work overlaps
//    on the GPU (different streams without ordering, or several host threads)
//    race on the array.
//  - The status words sit at a fixed place at the end of the array, are
//    cleared once when the device is set up, collect the flags of every call
//    and are read and cleared by lags_static_status_poll.
//  - The first call on a device (either entry point) resolves the array's
//    device address there (cudaGetSymbolAddress, with that device current),
//    configures the kernels and clears the status words.  With CUDA's lazy
//    module loading that is also when the driver loads this file's device
//    code and reserves the array on the device, so the first call belongs at
//    start-up, outside code that must not allocate and before any capture.
//  - Neither entry point calls cudaMalloc, cudaFree or another allocating
//    routine.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "lags.h"
#include "lags_internal.cuh"
#include "lags_plan.cuh"

namespace lags {
cudaError_t configure_estimate();
cudaError_t configure_select();
}  // namespace lags

using namespace lags;

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;
constexpr size_t kStaticStatusBytes = 256;  // >= kStatusWords * 4
constexpr size_t kStaticPlanBytes = kStaticScratchBytes - kStaticStatusBytes;
static_assert(kStatusWords * 4 <= kStaticStatusBytes, "status block");
constexpr int kMaxDevices = 64;

// Host code must not use g_static_scratch as an address: on the host it names
// a shadow object, not device memory.  Kernels get g_scratch_dev[device].
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
char* g_scratch_dev[kMaxDevices] = {};

// Once per device, with that device current: the scratch array's device
// address, the sm_100 check, the kernel attributes and cleared status words
// (enqueued on `s`).
lags_status scratch_for_current_device(cudaStream_t s, char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LAGS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LAGS_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_dev[dev]) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return LAGS_ERR_CUDA;
    if (major != 10 || minor != 0) return LAGS_ERR_UNSUPPORTED_DEVICE;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr)
      return LAGS_ERR_CUDA;
    if (configure_estimate() != cudaSuccess || configure_select() != cudaSuccess)
      return LAGS_ERR_CUDA;
    if (cudaMemsetAsync((char*)ptr + kStaticPlanBytes, 0, kStaticStatusBytes, s) != cudaSuccess)
      return LAGS_ERR_CUDA;
    g_scratch_dev[dev] = (char*)ptr;
  }
  *out = g_scratch_dev[dev];
  return LAGS_OK;
}

bool aligned_to(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" lags_status lags_sparsify_static(lags_plan* plan, const float* const* grads,
                                            float* const* residuals, float lr,
                                            uint32_t* out_idx, float* out_val, void* stream) {
  if (!plan || !grads || !residuals || !out_idx || !out_val) return LAGS_ERR_INVALID_ARG;
  if (plan->ws_bytes > kStaticPlanBytes) return LAGS_ERR_WORKSPACE;
  if (!aligned_to(out_idx, 4) || !aligned_to(out_val, 4)) return LAGS_ERR_ALIGNMENT;
  WorkerPtrs wp;
  std::memset(&wp, 0, sizeof(wp));
  for (int p = 0; p < plan->P; ++p) {
    if (!grads[p] || !residuals[p]) return LAGS_ERR_INVALID_ARG;
    if (!aligned_to(grads[p], 16) || !aligned_to(residuals[p], 16)) return LAGS_ERR_ALIGNMENT;
    wp.g[p] = grads[p];
    wp.r[p] = residuals[p];
  }
  cudaStream_t s = (cudaStream_t)stream;
  char* base = nullptr;
  lags_status st = scratch_for_current_device(s, &base);
  if (st != LAGS_OK) return st;

  auto up = [&](size_t o, const void* src, size_t n) {
    return n ? cudaMemcpyAsync(base + o, src, n, cudaMemcpyHostToDevice, s) : cudaSuccess;
  };
  cudaError_t e = up(plan->o_layers, plan->layers.data(), plan->layers.size() * sizeof(LayerDesc));
  if (e == cudaSuccess) e = up(plan->o_tiles, plan->tiles.data(), plan->tiles.size() * sizeof(TileDesc));
  if (e == cudaSuccess) e = up(plan->o_large, plan->sel_large.data(), plan->sel_large.size() * 4);
  if (e == cudaSuccess) e = up(plan->o_mid, plan->sel_mid.data(), plan->sel_mid.size() * 4);
  if (e == cudaSuccess) e = up(plan->o_small, plan->sel_small.data(), plan->sel_small.size() * 4);
  if (e == cudaSuccess) e = up(plan->o_huge, plan->sel_huge.data(), plan->sel_huge.size() * 4);
  if (e == cudaSuccess) e = up(plan->o_sparse, plan->sparse.data(), plan->sparse.size() * 4);
  if (e != cudaSuccess) return LAGS_ERR_CUDA;

  DevPlan dp;
  bind_dev_plan(plan, base, &dp);
  dp.status = reinterpret_cast<uint32_t*>(base + kStaticPlanBytes);  // the fixed status block
  e = launch_estimate(dp, wp, lr, s);
  if (e == cudaSuccess) e = launch_ef_capture(dp, wp, lr, out_idx, out_val, s);
  if (e == cudaSuccess) e = launch_select(dp, wp, out_idx, out_val, s);
  return e == cudaSuccess ? LAGS_OK : LAGS_ERR_CUDA;
}

extern "C" lags_status lags_static_status_poll(uint32_t* flags, uint32_t* exact_fallbacks,
                                               void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  char* base = nullptr;
  lags_status st = scratch_for_current_device(s, &base);
  if (st != LAGS_OK) return st;
  uint32_t words[2] = {0, 0};
  uint32_t* dev = reinterpret_cast<uint32_t*>(base + kStaticPlanBytes);
  cudaError_t e = cudaMemcpyAsync(words, dev, sizeof(words), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dev, 0, sizeof(words), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LAGS_ERR_CUDA;
  if (flags) *flags = words[kStatusFlags];
  if (exact_fallbacks) *exact_fallbacks = words[kStatusFallbacks];
  return lags_status_of_flags(words[kStatusFlags]);
}
