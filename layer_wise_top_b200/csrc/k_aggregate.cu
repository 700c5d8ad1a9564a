// Deterministic sparse aggregation and the weight update.
//
// Sparsified S-SGD ("Layer-wise Adaptive Gradient Sparsification ..." review,
// abstract) sums the workers' sparse sets into one averaged dense update:
// dense_j = ((+0 + v_0j) + v_1j + ... + v_(P-1)j) / P, workers in order, one
// rounding per add, a correctly rounded division; positions no worker picked
// are +0.  One CTA per group of consecutive tiles of one layer (the plan sizes
// groups to about a thousand expected picks): it stages all workers' picks of
// the group in shared memory; the thread holding the lowest worker's pick of a
// position finds the other workers' picks of it by binary search and adds them
// in worker order.  Tiles expected to hold many picks form groups of one and
// accumulate worker by worker in a shared tile instead.  No atomics, so the
// result is bit-identical however the grid is scheduled.  With a weights
// pointer the same kernel also applies the SGD update (weights -= dense).
//
// Pick lists are read through the read-only path (they are inputs; plain
// loads would be ordered behind the kernels' own scattered stores).
//
// k_pick_bounds first turns each worker's ascending pick list into the slot of
// the first pick of every tile, so each aggregation CTA reads only its own
// picks.  It also checks that the lists are ascending and inside their layer.
#include "block_ops.cuh"
#include "lags_internal.cuh"
#include "tma.cuh"

namespace lags {

constexpr uint32_t kAggThreads = 256;

__device__ __forceinline__ uint32_t tile_of(const LayerDesc& ld, uint32_t x) {
  return ld.tile_begin + (x / kTile - ld.off / kTile);
}

__global__ void __launch_bounds__(256) k_pick_bounds(DevPlan dp, const uint32_t* __restrict__ idx) {
  // one block per (chunk of 256 pick slots of a sparse layer, worker)
  pdl_trigger();
  const uint2 ch = dp.pick_chunks[blockIdx.x];  // (layer, first slot within the layer)
  const uint32_t p = blockIdx.y;
  const LayerDesc ld = dp.layers[ch.x];
  const uint32_t j = ch.y + threadIdx.x;
  pdl_wait();
  if (j >= ld.k) return;
  const uint64_t i = (uint64_t)ld.koff + j;
  const uint32_t* pi = idx + (uint64_t)p * dp.K;
  const uint32_t x = __ldg(pi + i);
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
    const uint32_t xp = __ldg(pi + i - 1);
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
constexpr uint32_t kAggPickCap = 2048;
// Up to this many picks in a tile, the thread holding a position's first pick
// looks the position up in the other workers' lists (binary search); above it,
// and when the launch has room for a tile accumulator, the CTA adds the
// workers' picks into shared memory one worker at a time instead.
constexpr uint32_t kAggOwnerMax = 512;

// Zeros the owner path sends to the dense output with bulk stores.
constexpr uint32_t kAggZeroBytes = 4096;  // keeps 4 tile-accumulator CTAs per SM

struct AggShared {
  float4 zero[kAggZeroBytes / 16];       // first: 16-byte aligned source of the bulk stores
  uint32_t loc[kAggPickCap];             // pick position inside the group, per worker ascending
  float val[kAggPickCap];
  uint32_t base[LAGS_MAX_WORKERS + 1];   // first staged pick of each worker
  uint32_t rng[2 * LAGS_MAX_WORKERS];
  uint32_t warp[kAggThreads / 32];
};
// Tile accumulator, only in launches that may need it.  A sum that started at
// +0 is never -0, so acc != 0 tells exactly which positions need the division
// and the weight update (0 / P == +0 and w - (+0) == w).
struct AggTileAcc {
  float acc[kTile];
};
// The accumulator follows AggShared in dynamic shared memory and is cleared
// with 16-byte stores, so it starts on a 128-byte boundary.
constexpr size_t kAggAccOffset = (sizeof(AggShared) + 127) / 128 * 128;
static_assert(kAggAccOffset % 16 == 0, "tile accumulator alignment");

__global__ void __launch_bounds__(kAggThreads, 4)
    k_aggregate(DevPlan dp, const uint32_t* __restrict__ idx, const float* __restrict__ val,
                float* __restrict__ dense, float* __restrict__ weights, bool have_acc) {
  extern __shared__ __align__(16) unsigned char agg_smem[];
  AggShared& sh = *reinterpret_cast<AggShared*>(agg_smem);
  AggTileAcc& ta = *reinterpret_cast<AggTileAcc*>(agg_smem + kAggAccOffset);
  pdl_trigger();
  // a group of consecutive tiles of one layer: elements [gs, gs + glen)
  const uint2 grp = dp.agg_groups[blockIdx.x];
  const uint32_t t = grp.x, nt = grp.y;
  const TileDesc td0 = dp.tiles[t];
  const TileDesc tdl = dp.tiles[t + nt - 1];
  const LayerDesc ld = dp.layers[td0.layer];
  const TileDesc td{td0.start, tdl.start + tdl.len - td0.start, td0.layer, 0};
  const uint32_t P = dp.P;
  const float fP = (float)P;
  const uint64_t K = dp.K;
  const int tid = threadIdx.x;
  // source of the bulk zero stores (this CTA's own shared memory)
  for (uint32_t i = tid; i < kAggZeroBytes / 16; i += kAggThreads)
    sh.zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  fence_proxy_async_shared();  // visible to the bulk copies after the next barrier
  pdl_wait();

  if (ld.k == ld.d) {
    // dense layer: every worker sent every entry; slot = koff + (e - off)
    const uint64_t s0 = ld.koff + (td.start - ld.off);
    for (uint32_t i = tid; i < td.len; i += kAggThreads) {
      float s = 0.0f;
      for (uint32_t p = 0; p < P; ++p) s = __fadd_rn(s, __ldg(val + p * K + s0 + i));
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
    uint32_t a = __ldg(first + t);
    uint32_t b = (t + nt < ld.tile_end) ? __ldg(first + t + nt) : kend;
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
  const bool staged = total <= kAggPickCap;
  // the tile accumulator covers one tile: groups of several tiles use the
  // owner search (the plan groups only tiles expected to hold few picks)
  const bool owner_path = staged && (total <= kAggOwnerMax || !have_acc || nt > 1);
  const uint32_t head = min(td.len, (4u - (td.start & 3u)) & 3u);
  const uint32_t nvec = (td.len - head) / 4;
  if (owner_path && tid == 0 && nvec > 0) {
    // the group's 16-byte-aligned middle is cleared by the bulk-copy engine
    // while the CTA stages and sums its picks; waited for before the sums
    char* dst = reinterpret_cast<char*>(dense + td.start + head);
    const uint64_t bytes = (uint64_t)nvec * 16;
    for (uint64_t o = 0; o < bytes; o += kAggZeroBytes) {
      const uint64_t n = bytes - o < kAggZeroBytes ? bytes - o : kAggZeroBytes;
      bulk_store(dst + o, sh.zero, (uint32_t)n);
    }
    bulk_commit();
  }
  auto worker_of = [&](uint32_t i) {  // staged pick i: last worker p with base[p] <= i
    uint32_t p = 0, hi = P - 1;
    while (p < hi) {
      const uint32_t m = (p + hi + 1) >> 1;
      if (sh.base[m] <= i) p = m; else hi = m - 1;
    }
    return p;
  };
  if (staged) {
    for (uint32_t i = tid; i < total; i += kAggThreads) {
      const uint32_t p = worker_of(i);
      const uint64_t slot = p * K + sh.rng[2 * p] + (i - sh.base[p]);
      const uint32_t x = __ldg(idx + slot) - td.start;
      sh.loc[i] = x < td.len ? x : 0xFFFFFFFFu;
      sh.val[i] = __ldg(val + slot);
    }
  }
  if (owner_path) {
    // ---- few picks: zeros everywhere, then each position's first owner ----
    // Owned positions, their sums and their old weights are all gathered
    // before this thread's first store: a load issued after stores waits for
    // them to drain.
    __syncthreads();  // staged picks visible to all threads
    constexpr uint32_t OI = kAggPickCap / kAggThreads;  // staged picks per thread
    uint32_t own_x[OI];
    float own_v[OI], own_w[OI];
#pragma unroll
    for (uint32_t j = 0; j < OI; ++j) {
      own_x[j] = 0xFFFFFFFFu;
      own_v[j] = 0.0f;
      own_w[j] = 0.0f;
      const uint32_t i = tid + j * kAggThreads;
      if (i >= total) continue;
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
        own_x[j] = x;
        own_v[j] = __fdiv_rn(s, fP);
      }
    }
    if (weights) {
#pragma unroll
      for (uint32_t j = 0; j < OI; ++j)
        if (own_x[j] != 0xFFFFFFFFu) own_w[j] = weights[td.start + own_x[j]];
    }
    // the unaligned ends of the group (the middle went to the bulk copies)
    for (uint32_t i = tid; i < head; i += kAggThreads) dense[td.start + i] = 0.0f;
    for (uint32_t i = head + 4 * nvec + tid; i < td.len; i += kAggThreads) dense[td.start + i] = 0.0f;
    if (tid == 0 && nvec > 0) {
      bulk_wait_all();             // the bulk zeros have landed ...
      fence_proxy_async_global();  // ... and are ordered before generic stores
    }
    __syncthreads();  // orders the zeros before the sums written below
#pragma unroll
    for (uint32_t j = 0; j < OI; ++j) {
      if (own_x[j] == 0xFFFFFFFFu) continue;
      dense[td.start + own_x[j]] = own_v[j];
      if (weights) weights[td.start + own_x[j]] = __fsub_rn(own_w[j], own_v[j]);
    }
    return;
  }

  if (have_acc && nt == 1) {
    // ---- many picks: worker-ordered accumulation in a shared tile ----
    float4* acc4 = reinterpret_cast<float4*>(ta.acc);
    for (uint32_t i = tid; i < kTile / 4; i += kAggThreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    for (uint32_t p = 0; p < P; ++p) {
      if (staged) {
        for (uint32_t j = sh.base[p] + tid; j < sh.base[p + 1]; j += kAggThreads) {
          const uint32_t x = sh.loc[j];
          if (x < td.len) ta.acc[x] = __fadd_rn(ta.acc[x], sh.val[j]);
        }
      } else {
        const uint64_t row = p * K;
        for (uint32_t j = sh.rng[2 * p] + tid; j < sh.rng[2 * p + 1]; j += kAggThreads) {
          const uint32_t x = __ldg(idx + row + j) - td.start;
          if (x < td.len) ta.acc[x] = __fadd_rn(ta.acc[x], __ldg(val + row + j));
        }
      }
      __syncthreads();
    }
    auto value_at = [&](uint32_t i) -> float {
      const float a = ta.acc[i];
      return a != 0.0f ? __fdiv_rn(a, fP) : 0.0f;
    };
    for (uint32_t i = tid; i < head; i += kAggThreads) {
      const float q = value_at(i);
      dense[td.start + i] = q;
      if (weights && __float_as_uint(q) != 0u)  // skip only +0: w - (-0) may differ from w
        weights[td.start + i] = __fsub_rn(weights[td.start + i], q);
    }
    float4* d4 = reinterpret_cast<float4*>(dense + td.start + head);
    float4* w4 = weights ? reinterpret_cast<float4*>(weights + td.start + head) : nullptr;
    // a thread's weight loads all go out before its first store (a load
    // issued after stores waits for them)
    constexpr uint32_t GV = (kTile / 4 + kAggThreads - 1) / kAggThreads;
    float4 wv[GV];
    bool upd[GV];
#pragma unroll
    for (uint32_t j = 0; j < GV; ++j) {
      const uint32_t v = tid + j * kAggThreads, i = head + 4 * v;
      upd[j] = w4 && v < nvec &&
               (ta.acc[i] != 0.f || ta.acc[i + 1] != 0.f || ta.acc[i + 2] != 0.f ||
                ta.acc[i + 3] != 0.f);
      if (upd[j]) wv[j] = w4[v];  // 16-byte aligned: weights and dense share the layout
    }
#pragma unroll
    for (uint32_t j = 0; j < GV; ++j) {
      const uint32_t v = tid + j * kAggThreads, i = head + 4 * v;
      if (v >= nvec) continue;
      const float4 q = make_float4(value_at(i), value_at(i + 1), value_at(i + 2), value_at(i + 3));
      __stcs(d4 + v, q);
      if (upd[j]) {
        wv[j].x = __fsub_rn(wv[j].x, q.x);
        wv[j].y = __fsub_rn(wv[j].y, q.y);
        wv[j].z = __fsub_rn(wv[j].z, q.z);
        wv[j].w = __fsub_rn(wv[j].w, q.w);
        w4[v] = wv[j];
      }
    }
    for (uint32_t i = head + 4 * nvec + tid; i < td.len; i += kAggThreads) {
      const float q = value_at(i);
      dense[td.start + i] = q;
      if (weights && __float_as_uint(q) != 0u)  // skip only +0: w - (-0) may differ from w
        weights[td.start + i] = __fsub_rn(weights[td.start + i], q);
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
      const uint32_t x = __ldg(idx + row + j) - td.start;
      if (x < td.len) dense[td.start + x] = __fadd_rn(dense[td.start + x], __ldg(val + row + j));
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

__global__ void __launch_bounds__(256) k_apply(uint32_t first, uint32_t end,
                                               float* __restrict__ w,
                                               const float* __restrict__ dense) {
  // elements [first, end): a scalar head up to the first 16-byte boundary,
  // float4 over the aligned middle, a scalar tail
  pdl_trigger();
  pdl_wait();
  const uint32_t a0 = min(end, (first + 3u) & ~3u);
  const uint32_t n4 = (end - a0) / 4;
  const uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x;
  const uint32_t stride = gridDim.x * blockDim.x;
  float4* w4 = reinterpret_cast<float4*>(w + a0);
  const float4* d4 = reinterpret_cast<const float4*>(dense + a0);
  for (uint32_t i = gid; i < n4; i += stride) {
    float4 a = w4[i];
    const float4 b = __ldcs(d4 + i);
    a.x = __fsub_rn(a.x, b.x);
    a.y = __fsub_rn(a.y, b.y);
    a.z = __fsub_rn(a.z, b.z);
    a.w = __fsub_rn(a.w, b.w);
    w4[i] = a;
  }
  if (gid < a0 - first) w[first + gid] = __fsub_rn(w[first + gid], dense[first + gid]);
  const uint32_t tail0 = a0 + n4 * 4;  // (compared as a count: tail0 + gid may pass 2^32)
  if (gid < end - tail0) w[tail0 + gid] = __fsub_rn(w[tail0 + gid], dense[tail0 + gid]);
}

cudaError_t launch_pick_bounds(const DevPlan& dp, const uint32_t* idx, cudaStream_t s) {
  if (dp.n_chunks == 0) return cudaSuccess;
  dim3 grid(dp.n_chunks, dp.P);
  return launch_pdl(k_pick_bounds, grid, dim3(256), 0, s, 1, dp, idx);
}

cudaError_t configure_aggregate() {
  return cudaFuncSetAttribute(k_aggregate, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(kAggAccOffset + sizeof(AggTileAcc)));
}

cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, float* weights, cudaStream_t s) {
  const size_t smem = dp.agg_tile_acc ? kAggAccOffset + sizeof(AggTileAcc) : sizeof(AggShared);
  return launch_pdl(k_aggregate, dim3(dp.n_groups), dim3(kAggThreads), smem, s, 1, dp, idx, val,
                    dense, weights, dp.agg_tile_acc != 0);
}

cudaError_t launch_apply(uint32_t first, uint32_t end, float* w, const float* dense,
                         cudaStream_t s) {
  uint32_t blocks = ((end - first) / 4 + 255) / 256;
  if (blocks > 148u * 16u) blocks = 148u * 16u;
  if (blocks == 0) blocks = 1;
  return launch_pdl(k_apply, dim3(blocks), dim3(256), 0, s, 1, first, end, w, dense);
}

}  // namespace lags
