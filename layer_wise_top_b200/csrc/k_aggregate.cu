// Deterministic sparse aggregation and the weight update.
//
// Sparsified S-SGD ("Layer-wise Adaptive Gradient Sparsification ..." review,
// abstract) sums the workers' sparse sets into one averaged dense update:
// dense_j = ((+0 + v_0j) + v_1j + ... + v_(P-1)j) / P, workers in order, one
// rounding per add, a correctly rounded division; positions no worker picked
// are +0.  One CTA per tile of the flattened buffer: it stages all workers'
// picks of the tile in shared memory, then each thread sums its own span of
// positions worker by worker.  No atomics and no cross-thread reduction, so the
// result is bit-identical however the grid is scheduled.  With a weights
// pointer the same kernel also applies the SGD update (weights -= dense).
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
  __shared__ uint32_t s_layer0;
  const uint64_t i0 = (uint64_t)blockIdx.x * blockDim.x;
  const uint64_t i = i0 + threadIdx.x;
  const uint32_t p = blockIdx.y;
  if (threadIdx.x == 0) {  // layer holding the block's first slot: last layer with koff <= i0
    uint32_t lo = 0, hi = dp.L - 1;
    while (lo < hi) {
      const uint32_t mid = (lo + hi + 1) >> 1;
      if (dp.layers[mid].koff <= i0) lo = mid; else hi = mid - 1;
    }
    s_layer0 = lo;
  }
  __syncthreads();
  if (i >= dp.K) return;
  uint32_t lo = s_layer0;  // slots are consecutive: step forward to this slot's layer
  while (lo + 1 < dp.L && dp.layers[lo + 1].koff <= i) ++lo;
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

// Picks of one tile staged in shared memory; a tile with more picks (layers
// sent at high density by many workers) reads them from global memory.
constexpr uint32_t kAggPickCap = 4096;
// Up to this many picks in a tile, the thread holding a position's first pick
// looks the position up in the other workers' lists (binary search); above it,
// and when the launch has room for a tile accumulator, the CTA adds the
// workers' picks into shared memory one worker at a time instead.
constexpr uint32_t kAggOwnerMax = 512;

struct AggShared {
  uint16_t loc[kAggPickCap];             // pick position inside the tile, per worker ascending
  float val[kAggPickCap];
  uint32_t base[LAGS_MAX_WORKERS + 1];   // first staged pick of each worker
  uint32_t rng[2 * LAGS_MAX_WORKERS];
  uint32_t warp[kAggThreads / 32];
};
struct AggTileAcc {                      // only in launches that may need it
  float acc[kTile];
  uint32_t hit[kTile / 32];              // bit i of word w: position 32 w + i was picked
};

__global__ void __launch_bounds__(kAggThreads)
    k_aggregate(DevPlan dp, const uint32_t* __restrict__ idx, const float* __restrict__ val,
                float* __restrict__ dense, float* __restrict__ weights, bool have_acc) {
  extern __shared__ __align__(16) unsigned char agg_smem[];
  AggShared& sh = *reinterpret_cast<AggShared*>(agg_smem);
  AggTileAcc& ta = *reinterpret_cast<AggTileAcc*>(agg_smem + sizeof(AggShared));
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
      const float dv = __fdiv_rn(s, fP);
      dense[td.start + i] = dv;
      if (weights) weights[td.start + i] = __fsub_rn(weights[td.start + i], dv);
    }
    return;
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
  auto worker_of = [&](uint32_t i) {  // staged pick i: last worker p with base[p] <= i
    uint32_t p = 0, hi = P - 1;
    while (p < hi) {
      const uint32_t m = (p + hi + 1) >> 1;
      if (sh.base[m] <= i) p = m; else hi = m - 1;
    }
    return p;
  };
  const bool staged = total <= kAggPickCap;
  if (staged) {
    for (uint32_t i = tid; i < total; i += kAggThreads) {
      const uint32_t p = worker_of(i);
      const uint64_t slot = p * K + sh.rng[2 * p] + (i - sh.base[p]);
      const uint32_t x = idx[slot] - td.start;
      sh.loc[i] = (uint16_t)(x < td.len ? x : 0xFFFFu);
      sh.val[i] = val[slot];
    }
  }
  const uint32_t head = min(td.len, (4u - (td.start & 3u)) & 3u);
  const uint32_t nvec = (td.len - head) / 4;

  if (staged && (total <= kAggOwnerMax || !have_acc)) {
    // ---- few picks: zeros everywhere, then each position's first owner ----
    for (uint32_t i = tid; i < head; i += kAggThreads) dense[td.start + i] = 0.0f;
    float4* d4 = reinterpret_cast<float4*>(dense + td.start + head);
    for (uint32_t v = tid; v < nvec; v += kAggThreads) __stcs(d4 + v, make_float4(0.f, 0.f, 0.f, 0.f));
    for (uint32_t i = head + 4 * nvec + tid; i < td.len; i += kAggThreads) dense[td.start + i] = 0.0f;
    __syncthreads();  // orders the zeros before the sums written below
    for (uint32_t i = tid; i < total; i += kAggThreads) {
      const uint32_t x = sh.loc[i];
      if (x >= td.len) continue;
      const uint32_t p = worker_of(i);
      bool first_owner = true;
      float s = 0.0f;
      for (uint32_t q = 0; q < P && first_owner; ++q) {
        if (q == p) {
          s = __fadd_rn(s, sh.val[i]);
          continue;
        }
        uint32_t a = sh.base[q], b = sh.base[q + 1];
        while (a < b) {  // lower bound of x in worker q's staged picks
          const uint32_t m = (a + b) >> 1;
          if (sh.loc[m] < x) a = m + 1; else b = m;
        }
        if (a < sh.base[q + 1] && sh.loc[a] == x) {
          if (q < p) first_owner = false;
          else s = __fadd_rn(s, sh.val[a]);
        }
      }
      if (first_owner) {
        const float dv = __fdiv_rn(s, fP);
        dense[td.start + x] = dv;
        if (weights) weights[td.start + x] = __fsub_rn(weights[td.start + x], dv);
      }
    }
    return;
  }

  if (have_acc) {
    // ---- many picks: worker-ordered accumulation in a shared tile ----
    for (uint32_t i = tid; i < kTile; i += kAggThreads) ta.acc[i] = 0.0f;
    for (uint32_t i = tid; i < kTile / 32; i += kAggThreads) ta.hit[i] = 0;
    __syncthreads();
    for (uint32_t p = 0; p < P; ++p) {
      if (staged) {
        for (uint32_t j = sh.base[p] + tid; j < sh.base[p + 1]; j += kAggThreads) {
          const uint32_t x = sh.loc[j];
          if (x >= td.len) continue;
          ta.acc[x] = __fadd_rn(ta.acc[x], sh.val[j]);
          atomicOr(&ta.hit[x / 32], 1u << (x % 32));
        }
      } else {
        const uint64_t row = p * K;
        for (uint32_t j = sh.rng[2 * p] + tid; j < sh.rng[2 * p + 1]; j += kAggThreads) {
          const uint32_t x = idx[row + j] - td.start;
          if (x >= td.len) continue;
          ta.acc[x] = __fadd_rn(ta.acc[x], val[row + j]);
          atomicOr(&ta.hit[x / 32], 1u << (x % 32));
        }
      }
      __syncthreads();
    }
    auto picked = [&](uint32_t i) -> bool { return (ta.hit[i / 32] >> (i % 32)) & 1u; };
    auto value_at = [&](uint32_t i) -> float {
      return picked(i) ? __fdiv_rn(ta.acc[i], fP) : 0.0f;
    };
    for (uint32_t i = tid; i < head; i += kAggThreads) {
      const float q = value_at(i);
      dense[td.start + i] = q;
      if (weights && picked(i)) weights[td.start + i] = __fsub_rn(weights[td.start + i], q);
    }
    float4* d4 = reinterpret_cast<float4*>(dense + td.start + head);
    float4* w4 = weights ? reinterpret_cast<float4*>(weights + td.start + head) : nullptr;
    for (uint32_t v = tid; v < nvec; v += kAggThreads) {
      const uint32_t i = head + 4 * v;
      const float4 q = make_float4(value_at(i), value_at(i + 1), value_at(i + 2), value_at(i + 3));
      __stcs(d4 + v, q);
      if (w4 && (picked(i) || picked(i + 1) || picked(i + 2) || picked(i + 3))) {
        float4 wv = w4[v];  // 16-byte aligned: weights and dense share the layout
        if (picked(i)) wv.x = __fsub_rn(wv.x, q.x);
        if (picked(i + 1)) wv.y = __fsub_rn(wv.y, q.y);
        if (picked(i + 2)) wv.z = __fsub_rn(wv.z, q.z);
        if (picked(i + 3)) wv.w = __fsub_rn(wv.w, q.w);
        w4[v] = wv;
      }
    }
    for (uint32_t i = head + 4 * nvec + tid; i < td.len; i += kAggThreads) {
      const float q = value_at(i);
      dense[td.start + i] = q;
      if (weights && picked(i)) weights[td.start + i] = __fsub_rn(weights[td.start + i], q);
    }
    return;
  }

  // ---- more picks than the stage holds and no tile accumulator: accumulate
  // worker by worker in the output itself, a barrier between workers ----
  for (uint32_t i = tid; i < td.len; i += kAggThreads) dense[td.start + i] = 0.0f;
  __syncthreads();
  for (uint32_t p = 0; p < P; ++p) {
    const uint64_t row = p * K;
    for (uint32_t j = sh.rng[2 * p] + tid; j < sh.rng[2 * p + 1]; j += kAggThreads) {
      const uint32_t x = idx[row + j] - td.start;
      if (x < td.len) dense[td.start + x] = __fadd_rn(dense[td.start + x], val[row + j]);
    }
    __syncthreads();
  }
  for (uint32_t i = tid; i < td.len; i += kAggThreads) {
    const float s = dense[td.start + i];
    if (s != 0.0f) {  // +0 stays +0 (0 / P), and w - (+0) == w
      const float dv = __fdiv_rn(s, fP);
      dense[td.start + i] = dv;
      if (weights) weights[td.start + i] = __fsub_rn(weights[td.start + i], dv);
    }
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
                              (int)(sizeof(AggShared) + sizeof(AggTileAcc)));
}

cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, float* weights, cudaStream_t s) {
  const size_t smem = sizeof(AggShared) + (dp.agg_tile_acc ? sizeof(AggTileAcc) : 0);
  k_aggregate<<<dp.T, kAggThreads, smem, s>>>(dp, idx, val, dense, weights, dp.agg_tile_acc != 0);
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
