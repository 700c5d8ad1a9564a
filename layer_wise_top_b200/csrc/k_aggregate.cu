// Deterministic sparse aggregation and the weight update.
//
// Sparsified S-SGD ("Layer-wise Adaptive Gradient Sparsification ..." review,
// abstract) sums the workers' sparse sets into one averaged dense update:
// dense_j = ((+0 + v_0j) + v_1j + ... + v_(P-1)j) / P, workers in order, one
// rounding per add, a correctly rounded division.  Every CTA owns one tile of
// the flattened buffer and builds that tile of the update in shared memory.
// It stages all workers' picks of the tile (each worker's list ascending);
// for every position, the thread holding the lowest worker's pick of it finds
// the other workers' picks by binary search and adds them in worker order.
// Positions nobody picked stay +0.  Tiles with more picks than fit in shared
// memory (layers sent at high density) accumulate worker by worker with a
// barrier in between.  No atomics: the result is bit-identical however the
// grid is scheduled.
//
// k_pick_bounds first turns each worker's ascending pick list into the slot of
// the first pick of every tile, so each aggregation CTA reads only its own
// picks.  It also checks that the lists are ascending and inside their layer.
#include "block_ops.cuh"
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

// Picks of one tile that fit in shared memory at once; a tile with more picks
// (layers sent at high density) is summed worker by worker instead.
constexpr uint32_t kAggPickCap = 4096;

struct AggShared {
  uint16_t loc[kAggPickCap];      // pick position inside the tile, per worker ascending
  float val[kAggPickCap];
  uint32_t base[LAGS_MAX_WORKERS + 1];  // first staged pick of each worker
  uint32_t rng[2 * LAGS_MAX_WORKERS];
  uint32_t warp[kAggThreads / 32];
};

// Lower bound of x in the ascending loc[a, b).
__device__ __forceinline__ uint32_t lower_bound_loc(const uint16_t* loc, uint32_t a, uint32_t b,
                                                    uint32_t x) {
  while (a < b) {
    const uint32_t m = (a + b) >> 1;
    if (loc[m] < x) a = m + 1; else b = m;
  }
  return a;
}

__global__ void __launch_bounds__(kAggThreads)
    k_aggregate(DevPlan dp, const uint32_t* __restrict__ idx, const float* __restrict__ val,
                float* __restrict__ dense) {
  extern __shared__ __align__(16) unsigned char agg_smem[];
  AggShared& sh = *reinterpret_cast<AggShared*>(agg_smem);
  const uint32_t t = blockIdx.x;
  const TileDesc td = dp.tiles[t];
  const LayerDesc ld = dp.layers[td.layer];
  const uint32_t P = dp.P;
  const float fP = (float)P;
  const uint64_t K = dp.K;
  const int tid = threadIdx.x;

  if (ld.k == ld.d) {
    // dense layer: every worker sent every entry; slot = koff + (e - off)
    const uint64_t s0 = ld.koff + (td.start - ld.off);
    for (uint32_t i = tid; i < td.len; i += kAggThreads) {
      float s = 0.0f;
      for (uint32_t p = 0; p < P; ++p) s = __fadd_rn(s, val[p * K + s0 + i]);
      dense[td.start + i] = __fdiv_rn(s, fP);
    }
    return;
  }

  // positions nobody picked are +0: write the whole tile as zeros first
  // (16-byte stores where aligned); picked positions are overwritten below
  // after a barrier, which orders the two writes
  {
    const uint32_t head = min(td.len, (4u - (td.start & 3u)) & 3u);
    const uint32_t nvec = (td.len - head) / 4;
    for (uint32_t i = tid; i < head; i += kAggThreads) dense[td.start + i] = 0.0f;
    float4* d4 = reinterpret_cast<float4*>(dense + td.start + head);
    for (uint32_t v = tid; v < nvec; v += kAggThreads) d4[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (uint32_t i = head + 4 * nvec + tid; i < td.len; i += kAggThreads)
      dense[td.start + i] = 0.0f;
  }
  const uint32_t kend = ld.koff + ld.k;
  uint32_t cnt = 0;
  if (tid < (int)P) {
    const uint32_t* first = dp.pick_first + (size_t)tid * dp.T;
    uint32_t a = first[t];
    uint32_t b = (t + 1 < ld.tile_end) ? first[t + 1] : kend;
    a = min(max(a, ld.koff), kend);  // keeps a bad pick list inside the layer
    b = min(max(b, a), kend);
    sh.rng[2 * tid] = a;
    sh.rng[2 * tid + 1] = b;
    cnt = b - a;
  }
  uint32_t total;
  const uint32_t before = block_excl_scan<kAggThreads>(cnt, sh.warp, &total);
  if (tid < (int)P) sh.base[tid] = before;
  if (tid == 0) sh.base[P] = total;
  __syncthreads();

  if (total <= kAggPickCap) {
    // stage every worker's picks of this tile (each list ascending); staged
    // pick i belongs to the last worker p with base[p] <= i
    for (uint32_t i = tid; i < total; i += kAggThreads) {
      uint32_t p = 0, hi = P - 1;
      while (p < hi) {
        const uint32_t m = (p + hi + 1) >> 1;
        if (sh.base[m] <= i) p = m; else hi = m - 1;
      }
      const uint64_t slot = p * K + sh.rng[2 * p] + (i - sh.base[p]);
      const uint32_t x = idx[slot] - td.start;
      sh.loc[i] = (uint16_t)(x < td.len ? x : 0xFFFFu);
      sh.val[i] = val[slot];
    }
    __syncthreads();
    // the first worker that picked a position sums all workers' values for it
    // in worker order, then divides by P
    for (uint32_t i = tid; i < total; i += kAggThreads) {
      const uint32_t x = sh.loc[i];
      if (x >= td.len) continue;
      uint32_t p = 0, hi = P - 1;  // worker of staged pick i
      while (p < hi) {
        const uint32_t m = (p + hi + 1) >> 1;
        if (sh.base[m] <= i) p = m; else hi = m - 1;
      }
      bool first_owner = true;
      float s = 0.0f;
      for (uint32_t q = 0; q < P && first_owner; ++q) {
        if (q == p) {
          s = __fadd_rn(s, sh.val[i]);
          continue;
        }
        const uint32_t at = lower_bound_loc(sh.loc, sh.base[q], sh.base[q + 1], x);
        if (at < sh.base[q + 1] && sh.loc[at] == x) {
          if (q < p) first_owner = false;
          else s = __fadd_rn(s, sh.val[at]);
        }
      }
      if (first_owner) dense[td.start + x] = __fdiv_rn(s, fP);
    }
  } else {
    // many picks in this tile: accumulate worker by worker in the output
    // itself (the zeros above), one barrier between workers
    for (uint32_t p = 0; p < P; ++p) {
      const uint32_t a = sh.rng[2 * p], b = sh.rng[2 * p + 1];
      for (uint32_t j = a + tid; j < b; j += kAggThreads) {
        const uint32_t x = idx[p * K + j] - td.start;
        if (x < td.len) dense[td.start + x] = __fadd_rn(dense[td.start + x], val[p * K + j]);
      }
      __syncthreads();
    }
    for (uint32_t i = tid; i < td.len; i += kAggThreads)
      dense[td.start + i] = __fdiv_rn(dense[td.start + i], fP);
  }
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

cudaError_t configure_aggregate() {
  return cudaFuncSetAttribute(k_aggregate, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(AggShared));
}

cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, cudaStream_t s) {
  k_aggregate<<<dp.T, kAggThreads, sizeof(AggShared), s>>>(dp, idx, val, dense);
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
