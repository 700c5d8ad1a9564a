// Deterministic sparse aggregation and the weight update.
//
// Sparsified S-SGD ("Layer-wise Adaptive Gradient Sparsification ..." review,
// abstract) sums the workers' sparse sets into one averaged dense update.
// Here every CTA owns one tile of the flattened buffer and builds that tile of
// the update in shared memory: it starts from +0, adds worker 0's picks, then
// worker 1's, ... worker P-1's (one rounding per add, a barrier between
// workers, no atomics), and finally divides by P with a correctly rounded
// division.  The result is bit-identical however the grid is scheduled.
//
// k_pick_bounds first turns each worker's ascending pick list into the slot of
// the first pick of every tile, so each aggregation CTA reads only its own
// picks.  It also checks that the lists are ascending and inside their layer.
#include "lags_internal.cuh"

namespace lags {

constexpr uint32_t kAggThreads = 256;

__device__ __forceinline__ uint32_t tile_of(const LayerDesc& ld, uint32_t x) {
  return ld.tile_begin + (x / kTile - ld.off / kTile);
}

__global__ void __launch_bounds__(256) k_pick_bounds(DevPlan dp, const uint32_t* __restrict__ idx) {
  const uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint32_t p = blockIdx.y;
  if (i >= dp.K) return;
  // layer holding pick slot i: the last layer with koff <= i
  uint32_t lo = 0, hi = dp.L - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (dp.layers[mid].koff <= i) lo = mid; else hi = mid - 1;
  }
  const LayerDesc ld = dp.layers[lo];
  if (ld.k == ld.d) return;  // dense layer: slot of element e is koff + e - off
  const uint32_t* pi = idx + (uint64_t)p * dp.K;
  const uint32_t x = pi[i];
  const uint32_t lend = ld.off + ld.d;
  if (x < ld.off || x >= lend) {
    atomicOr(dp.status + kStatusFlags, LAGS_FLAG_BAD_PICKS);
    return;
  }
  const uint32_t ti = tile_of(ld, x);
  uint32_t tprev;
  if (i == ld.koff) {
    tprev = ld.tile_begin - 1;  // wraps for tile_begin == 0; only used as tprev + 1
  } else {
    const uint32_t xp = pi[i - 1];
    if (xp < ld.off || xp >= x) {
      atomicOr(dp.status + kStatusFlags, LAGS_FLAG_BAD_PICKS);
      return;
    }
    tprev = tile_of(ld, xp);
  }
  uint32_t* first = dp.pick_first + (size_t)p * dp.T;
  for (uint32_t t = tprev + 1; t <= ti; ++t) first[t] = (uint32_t)i;
  if (i == (uint64_t)ld.koff + ld.k - 1)
    for (uint32_t t = ti + 1; t < ld.tile_end; ++t) first[t] = ld.koff + ld.k;
}

__global__ void __launch_bounds__(kAggThreads)
    k_aggregate(DevPlan dp, const uint32_t* __restrict__ idx, const float* __restrict__ val,
                float* __restrict__ dense) {
  __shared__ float s_acc[kTile];
  __shared__ uint32_t s_rng[2 * LAGS_MAX_WORKERS];
  const uint32_t t = blockIdx.x;
  const TileDesc td = dp.tiles[t];
  const LayerDesc ld = dp.layers[td.layer];
  const uint32_t P = dp.P;
  const float fP = (float)P;
  const uint64_t K = dp.K;

  if (ld.k == ld.d) {
    // dense layer: every worker sent every entry; slot = koff + (e - off)
    const uint64_t s0 = ld.koff + (td.start - ld.off);
    for (uint32_t i = threadIdx.x; i < td.len; i += kAggThreads) {
      float s = 0.0f;
      for (uint32_t p = 0; p < P; ++p) s = __fadd_rn(s, val[p * K + s0 + i]);
      dense[td.start + i] = __fdiv_rn(s, fP);
    }
    return;
  }

  for (uint32_t i = threadIdx.x; i < td.len; i += kAggThreads) s_acc[i] = 0.0f;
  const uint32_t kend = ld.koff + ld.k;
  for (uint32_t p = threadIdx.x; p < P; p += kAggThreads) {
    const uint32_t* first = dp.pick_first + (size_t)p * dp.T;
    uint32_t a = first[t];
    uint32_t b = (t + 1 < ld.tile_end) ? first[t + 1] : kend;
    a = min(max(a, ld.koff), kend);  // keeps a bad pick list inside the layer
    b = min(max(b, a), kend);
    s_rng[2 * p] = a;
    s_rng[2 * p + 1] = b;
  }
  __syncthreads();
  for (uint32_t p = 0; p < P; ++p) {
    const uint32_t a = s_rng[2 * p], b = s_rng[2 * p + 1];
    for (uint32_t j = a + threadIdx.x; j < b; j += kAggThreads) {
      const uint32_t loc = idx[p * K + j] - td.start;
      if (loc < td.len) s_acc[loc] = __fadd_rn(s_acc[loc], val[p * K + j]);
    }
    __syncthreads();
  }
  for (uint32_t i = threadIdx.x; i < td.len; i += kAggThreads)
    dense[td.start + i] = __fdiv_rn(s_acc[i], fP);
}

__global__ void __launch_bounds__(256) k_apply(uint32_t N, float* __restrict__ w,
                                               const float* __restrict__ dense) {
  const uint32_t n4 = N / 4;
  const uint32_t stride = gridDim.x * blockDim.x;
  float4* w4 = reinterpret_cast<float4*>(w);
  const float4* d4 = reinterpret_cast<const float4*>(dense);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = w4[i];
    const float4 b = __ldcs(d4 + i);
    a.x = __fsub_rn(a.x, b.x);
    a.y = __fsub_rn(a.y, b.y);
    a.z = __fsub_rn(a.z, b.z);
    a.w = __fsub_rn(a.w, b.w);
    w4[i] = a;
  }
  const uint32_t tail = n4 * 4 + blockIdx.x * blockDim.x + threadIdx.x;
  if (tail < N) w[tail] = __fsub_rn(w[tail], dense[tail]);
}

cudaError_t launch_pick_bounds(const DevPlan& dp, const uint32_t* idx, cudaStream_t s) {
  dim3 grid((unsigned)((dp.K + 255) / 256), dp.P);
  k_pick_bounds<<<grid, 256, 0, s>>>(dp, idx);
  return cudaGetLastError();
}

cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, cudaStream_t s) {
  k_aggregate<<<dp.T, kAggThreads, 0, s>>>(dp, idx, val, dense);
  return cudaGetLastError();
}

cudaError_t launch_apply(uint32_t N, float* w, const float* dense, cudaStream_t s) {
  uint32_t blocks = (N / 4 + 255) / 256;
  if (blocks > 148u * 16u) blocks = 148u * 16u;
  if (blocks == 0) blocks = 1;
  k_apply<<<blocks, 256, 0, s>>>(N, w, dense);
  return cudaGetLastError();
}

}  // namespace lags
