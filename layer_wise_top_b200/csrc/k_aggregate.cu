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
// accumulate worker by worker in a shared tile instead.  Either way each tile
// of the update is composed in shared memory and written once, with aligned
// 16-byte stores: the kernel streams the dense output at the HBM rate and
// never writes a position twice.  No atomics, so the result is bit-identical
// however the grid is scheduled.  With a weights pointer the SGD update
// (weights -= dense) follows at the picked positions: the kernel leaves one
// (position, quotient) record per pick for k_weight_updates, and groups of
// one high-density tile apply it themselves.
//
// Pick lists are read through the read-only path (they are inputs; plain
// loads would be ordered behind the kernels' own scattered stores).
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
  // one block per (chunk of 256 pick slots of a sparse layer, worker)
  pdl_trigger();
  const uint2 ch = dp.pick_chunks[blockIdx.x];  // (layer, first slot within the layer)
  const uint32_t p = blockIdx.y;
  const LayerDesc ld = dp.layers[ch.x];
  const uint32_t j = ch.y + threadIdx.x;
  pdl_wait();
  if (j >= ld.k) return;
  const uint64_t i = (uint64_t)ld.koff + j;
  const uint32_t* pi = after_wait(idx) + (uint64_t)p * dp.K;
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

// Up to this many picks in a one-tile group, the thread holding a position's
// first pick looks the position up in the other workers' lists (binary
// search); above it the CTA adds the workers' picks into the shared tile one
// worker at a time instead.
constexpr uint32_t kAggOwnerMax = 512;
// The shared tile holds one tile of the dense update, placed so that shared
// index j is element (tile start rounded down to 4) + j: float4 slot v of the
// tile is then one aligned 16-byte store.  A tile spans at most kTile + 3
// such positions.
constexpr uint32_t kAggTileSlots = kTile / 4 + 1;  // float4 slots
constexpr uint32_t kAggSlotsPerThread = (kAggTileSlots + kAggThreads - 1) / kAggThreads;

struct AggShared {
  float4 tile[kAggTileSlots];            // first: 16-byte aligned
  uint32_t loc[kAggPickCap];             // pick position inside the group, per worker ascending
  float val[kAggPickCap];
  uint32_t seen[2][kTile / 32];          // positions of a tile picked by some worker
  uint32_t multi[2][kTile / 32];         // ... by more than one worker (two sets: tiles alternate)
  uint32_t base[LAGS_MAX_WORKERS + 1];   // first staged pick of each worker
  uint32_t rng[2 * LAGS_MAX_WORKERS];    // each worker's pick slots [a, b) of the group / tile
  uint32_t warp[kAggThreads / 32];
};

__device__ __forceinline__ float f4_get(const float4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Writes tile [start, start + len) of the dense update from the shared tile
// (positions relative to start & ~3) with aligned 16-byte streaming stores
// (scalar stores at a tile's unaligned ends) and clears the shared tile behind
// it.  With `divide`, the tile holds sums: each nonzero sum is divided by P
// (a sum that started at +0 is never -0, so zero means "no pick": +0 / P = +0
// and w - (+0) = w) and, with weights, applied to them.  Without `divide` the
// tile holds finished values and the weights were updated by their owners.
__device__ __forceinline__ void agg_write_tile(AggShared& sh, uint32_t start, uint32_t len,
                                               float* __restrict__ dense,
                                               float* __restrict__ weights, bool divide,
                                               float fP) {
  const uint32_t base = start & ~3u, end = start + len;
  const uint32_t nv = (end - base + 3) / 4;
  float4 wv[kAggSlotsPerThread];
  bool upd[kAggSlotsPerThread];
  // first the quotients (back into the shared tile) and every weight load of
  // this thread, then the stores (a load issued after stores waits for them)
#pragma unroll
  for (uint32_t j = 0; j < kAggSlotsPerThread; ++j) {
    const uint32_t v = threadIdx.x + j * kAggThreads;
    upd[j] = false;
    if (!divide || v >= nv) continue;
    float4 a = sh.tile[v];
    // (most slots hold no pick: divide only where a sum is)
    if ((__float_as_uint(a.x) | __float_as_uint(a.y) | __float_as_uint(a.z) |
         __float_as_uint(a.w)) == 0u)
      continue;
    a.x = a.x != 0.0f ? __fdiv_rn(a.x, fP) : 0.0f;
    a.y = a.y != 0.0f ? __fdiv_rn(a.y, fP) : 0.0f;
    a.z = a.z != 0.0f ? __fdiv_rn(a.z, fP) : 0.0f;
    a.w = a.w != 0.0f ? __fdiv_rn(a.w, fP) : 0.0f;
    sh.tile[v] = a;
    // skip only +0: w - (-0) may differ from w
    upd[j] = weights && (__float_as_uint(a.x) | __float_as_uint(a.y) | __float_as_uint(a.z) |
                         __float_as_uint(a.w)) != 0u;
    const uint32_t e0 = base + 4 * v;
    if (upd[j]) {
      if (e0 >= start && e0 + 4 <= end) {
        wv[j] = *reinterpret_cast<const float4*>(weights + e0);
      } else {
        float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (e0 + c >= start && e0 + c < end) t[c] = weights[e0 + c];
        wv[j] = make_float4(t[0], t[1], t[2], t[3]);
      }
    }
  }
#pragma unroll
  for (uint32_t j = 0; j < kAggSlotsPerThread; ++j) {
    const uint32_t v = threadIdx.x + j * kAggThreads;
    if (v >= nv) continue;
    const uint32_t e0 = base + 4 * v;
    const float4 a = sh.tile[v];
    sh.tile[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 nw = wv[j];
    if (upd[j]) {
      nw.x = __fsub_rn(nw.x, a.x);
      nw.y = __fsub_rn(nw.y, a.y);
      nw.z = __fsub_rn(nw.z, a.z);
      nw.w = __fsub_rn(nw.w, a.w);
    }
    if (e0 >= start && e0 + 4 <= end) {
      __stcs(reinterpret_cast<float4*>(dense + e0), a);
      if (upd[j]) *reinterpret_cast<float4*>(weights + e0) = nw;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (e0 + c < start || e0 + c >= end) continue;
        dense[e0 + c] = f4_get(a, c);
        if (upd[j] && __float_as_uint(f4_get(a, c)) != 0u) weights[e0 + c] = f4_get(nw, c);
      }
    }
  }
}

// One CTA per group of consecutive tiles of one layer (the plan sizes groups
// to about a thousand expected picks).  The CTA loads the group's pick bounds
// and stages every worker's picks of the group in shared memory.  Then, tile
// by tile:
//   1. every pick marks its position in a bitmap; a second bitmap marks the
//      positions that several workers picked;
//   2. a position picked by one worker gets fl(+0 + v) in the shared tile
//      from that pick; a position picked by several gets its worker-ordered
//      sum from the pick of the lowest worker, which looks the position up in
//      the other workers' staged lists (binary search);
//   3. the CTA divides the tile by P and writes all of it once, coalesced.
// The pick that wrote a position (its "owner") writes the quotient itself, so
// the tile write divides nothing.  With weights, every staged pick leaves a
// record for k_weight_updates: (position, quotient) for owners, a skip mark
// for the others; the weights' scattered read-modify-writes then run in a
// pass of their own instead of slowing the dense stream.  Groups of one
// high-density tile instead add the workers' picks into the shared tile
// worker by worker (a barrier between workers), then divide, apply the
// weights and write.
__global__ void __launch_bounds__(kAggThreads, 4)
    k_aggregate(DevPlan dp, const uint32_t* __restrict__ idx0, const float* __restrict__ val0,
                float* __restrict__ dense, float* __restrict__ weights) {
  extern __shared__ __align__(16) unsigned char agg_smem[];
  AggShared& sh = *reinterpret_cast<AggShared*>(agg_smem);
  pdl_trigger();
  const uint2 grp = dp.agg_groups[blockIdx.x];
  const uint32_t t = grp.x, nt = grp.y;
  const uint32_t P = dp.P;
  const float fP = (float)P;
  const uint64_t K = dp.K;
  const int tid = threadIdx.x;
  for (uint32_t v = tid; v < kAggTileSlots; v += kAggThreads)
    sh.tile[v] = make_float4(0.f, 0.f, 0.f, 0.f);
  pdl_wait();
  const uint32_t* __restrict__ idx = after_wait(idx0);
  const float* __restrict__ val = after_wait(val0);
  const uint32_t* __restrict__ pick_first = after_wait(dp.pick_first);
  // each worker's first picks of the group and of the next tile (addresses
  // from the group alone) first, the tile and layer descriptors behind them:
  // loads issued before the dependency wait measured to delay the loads after it
  uint32_t first_a = 0, first_b = 0;
  if (tid < (int)P) {
    const uint32_t* f = pick_first + (size_t)tid * dp.T;
    first_a = __ldg(f + t);
    if (t + nt < dp.T) first_b = __ldg(f + t + nt);
  }
  const TileDesc td0 = after_wait(dp.tiles)[t];
  const TileDesc tdl = after_wait(dp.tiles)[t + nt - 1];
  const LayerDesc ld = after_wait(dp.layers)[td0.layer];
  const uint32_t gs = td0.start, glen = tdl.start + tdl.len - td0.start;

  if (weights && tid == 0) dp.wcnt[blockIdx.x] = 0;  // (the owner path below sets it)
  if (ld.k == ld.d) {
    // dense layer: every worker sent every entry; slot = koff + (e - off)
    const uint64_t s0 = ld.koff + (gs - ld.off);
    for (uint32_t i = tid; i < glen; i += kAggThreads) {
      float s = 0.0f;
      for (uint32_t p = 0; p < P; ++p) s = __fadd_rn(s, __ldg(val + p * K + s0 + i));
      const float dv = __fdiv_rn(s, fP);
      dense[gs + i] = dv;
      if (weights) weights[gs + i] = __fsub_rn(weights[gs + i], dv);
    }
    return;
  }

  const uint32_t kend = ld.koff + ld.k;
  // each worker's picks of [first, first + n) tiles (a bad pick list is kept
  // inside its layer)
  auto load_bounds = [&](uint32_t first, uint32_t n) -> uint32_t {
    uint32_t c = 0;
    if (tid < (int)P) {
      const uint32_t* f = pick_first + (size_t)tid * dp.T;
      uint32_t a = __ldg(f + first);
      uint32_t b = (first + n < ld.tile_end) ? __ldg(f + first + n) : kend;
      a = min(max(a, ld.koff), kend);
      b = min(max(b, a), kend);
      sh.rng[2 * tid] = a;
      sh.rng[2 * tid + 1] = b;
      c = b - a;
    }
    return c;
  };
  uint32_t c0 = 0;  // this worker's picks of the group (as load_bounds(t, nt))
  if (tid < (int)P) {
    uint32_t a = first_a, b = (t + nt < ld.tile_end) ? first_b : kend;
    a = min(max(a, ld.koff), kend);
    b = min(max(b, a), kend);
    sh.rng[2 * tid] = a;
    sh.rng[2 * tid + 1] = b;
    c0 = b - a;
  }
  uint32_t total;
  const uint32_t before = block_excl_scan<kAggThreads>(c0, sh.warp, &total);
  if (tid < (int)P) sh.base[tid] = before;
  if (tid == 0) sh.base[P] = total;
  __syncthreads();
  const bool staged = total <= kAggPickCap;
  auto worker_of = [&](uint32_t i) {  // staged pick i: last worker p with base[p] <= i
    uint32_t p = 0, hi = P - 1;
    while (p < hi) {
      const uint32_t m = (p + hi + 1) >> 1;
      if (sh.base[m] <= i) p = m; else hi = m - 1;
    }
    return p;
  };
  constexpr uint32_t OI = kAggPickCap / kAggThreads;  // staged picks per thread
  // staged pick i = tid + 256 j belongs to this thread: its position in the
  // group and its worker stay in registers for the owner path below
  static_assert(OI == 8 && LAGS_MAX_WORKERS <= 256, "eight 8-bit worker ids per thread");
  uint32_t px[OI];
  uint64_t pw = 0;  // byte j: worker of pick j
  if (staged) {
    // all of a thread's loads in flight before the shared stores
    float sv[OI];
#pragma unroll
    for (uint32_t j = 0; j < OI; ++j) {
      const uint32_t i = tid + j * kAggThreads;
      px[j] = 0xFFFFFFFFu;
      sv[j] = 0.0f;
      if (i < total) {
        const uint32_t p = worker_of(i);
        pw |= (uint64_t)p << (8 * j);
        const uint64_t slot = p * K + sh.rng[2 * p] + (i - sh.base[p]);
        px[j] = __ldg(idx + slot) - gs;
        sv[j] = __ldg(val + slot);
      }
    }
#pragma unroll
    for (uint32_t j = 0; j < OI; ++j) {
      const uint32_t i = tid + j * kAggThreads;
      if (px[j] >= glen) px[j] = 0xFFFFFFFFu;  // (a bad pick list stays inside the group)
      if (i < total) {
        sh.loc[i] = px[j];
        sh.val[i] = sv[j];
      }
    }
  }
  __syncthreads();  // staged picks visible to all threads

  float* tile = reinterpret_cast<float*>(sh.tile);
  if (staged && (nt > 1 || total <= kAggOwnerMax)) {
    uint32_t own = 0;  // bit j: this thread writes pick j's position
    // Two barriers per tile: the bitmaps alternate between tiles (a set is
    // cleared while the other is in use), and the write of tile q is
    // separated from the owners' writes of tile q + 1 by that tile's first
    // barrier.
    for (uint32_t w = tid; w < kTile / 32; w += kAggThreads) {
      sh.seen[0][w] = 0;
      sh.multi[0][w] = 0;
    }
    __syncthreads();
    for (uint32_t q = 0; q < nt; ++q) {
      const TileDesc tq = nt == 1 ? td0 : dp.tiles[t + q];
      const uint32_t lo = tq.start - gs;
      const uint32_t shift = tq.start & 3u;  // shared index of the tile's first element
      uint32_t* seen = sh.seen[q & 1];
      uint32_t* multi = sh.multi[q & 1];
      // 1. which positions of the tile do several workers pick?
#pragma unroll
      for (uint32_t j = 0; j < OI; ++j) {
        const uint32_t x = px[j] - lo;
        if (x < tq.len) {
          const uint32_t bit = 1u << (x & 31);
          if (atomicOr(&seen[x >> 5], bit) & bit) atomicOr(&multi[x >> 5], bit);
        }
      }
      __syncthreads();
      // the other set was last read before this tile's barrier: clear it
      for (uint32_t w = tid; w < kTile / 32; w += kAggThreads) {
        sh.seen[(q + 1) & 1][w] = 0;
        sh.multi[(q + 1) & 1][w] = 0;
      }
      // 2. one pick per position writes its worker-ordered sum
#pragma unroll
      for (uint32_t j = 0; j < OI; ++j) {
        const uint32_t x = px[j] - lo;
        if (x >= tq.len) continue;
        const uint32_t i = tid + j * kAggThreads;
        float s;
        if (!(multi[x >> 5] & (1u << (x & 31)))) {
          s = __fadd_rn(0.0f, sh.val[i]);
        } else {
          // several workers: the lowest one sums them in worker order
          const uint32_t p = (uint32_t)(pw >> (8 * j)) & 0xFFu, gx = px[j];
          bool first_owner = true;
          s = 0.0f;
          for (uint32_t r = 0; r < P && first_owner; ++r) {
            if (r == p) {
              s = __fadd_rn(s, sh.val[i]);
              continue;
            }
            uint32_t u = sh.base[r], e = sh.base[r + 1];
            while (u < e) {  // lower bound of gx in worker r's staged picks
              const uint32_t m = (u + e) >> 1;
              if (sh.loc[m] < gx) u = m + 1; else e = m;
            }
            if (u < sh.base[r + 1] && sh.loc[u] == gx) {
              if (r < p) first_owner = false;
              else s = __fadd_rn(s, sh.val[u]);
            }
          }
          if (!first_owner) continue;
        }
        const float qv = __fdiv_rn(s, fP);  // (+0 / P = +0)
        tile[shift + x] = qv;
        own |= 1u << j;
        // kept for the weight record in the pick's own value slot (only the
        // owner ever reads an owner's value)
        sh.val[i] = qv;
      }
      __syncthreads();
      // 3. the whole tile, once (clearing it behind; the next tile's owners
      // write after its first barrier)
      agg_write_tile(sh, tq.start, tq.len, dense, nullptr, false, fP);
    }
    if (weights) {
      // one record per staged pick: owners whose quotient is not +0 (w - (+0)
      // == w; w - (-0) may differ from w) update their weight
      uint2* rec = dp.wrec + (size_t)blockIdx.x * kAggPickCap;
#pragma unroll
      for (uint32_t j = 0; j < OI; ++j) {
        const uint32_t i = tid + j * kAggThreads;
        if (i >= total) break;
        const float qj = sh.val[i];
        const bool upd = ((own >> j) & 1u) && __float_as_uint(qj) != 0u;
        rec[i] = upd ? make_uint2(gs + px[j], __float_as_uint(qj)) : make_uint2(0xFFFFFFFFu, 0u);
      }
      if (tid == 0) dp.wcnt[blockIdx.x] = total;
    }
    return;
  }

  // ---- many picks: worker-ordered accumulation in the shared tile, one tile
  // at a time (a group of one tile with staged picks reads them from shared
  // memory, otherwise from global memory) ----
  for (uint32_t q = 0; q < nt; ++q) {
    const TileDesc tq = nt == 1 ? td0 : dp.tiles[t + q];
    const uint32_t shift = tq.start & 3u;
    const bool from_stage = staged && nt == 1;
    if (!from_stage) {
      load_bounds(t + q, 1);
      __syncthreads();
    }
    for (uint32_t p = 0; p < P; ++p) {
      if (from_stage) {
        for (uint32_t j = sh.base[p] + tid; j < sh.base[p + 1]; j += kAggThreads) {
          const uint32_t x = sh.loc[j];
          if (x < tq.len) tile[shift + x] = __fadd_rn(tile[shift + x], sh.val[j]);
        }
      } else {
        const uint64_t row = p * K;
        for (uint32_t j = sh.rng[2 * p] + tid; j < sh.rng[2 * p + 1]; j += kAggThreads) {
          const uint32_t x = __ldg(idx + row + j) - tq.start;
          if (x < tq.len) tile[shift + x] = __fadd_rn(tile[shift + x], __ldg(val + row + j));
        }
      }
      __syncthreads();
    }
    agg_write_tile(sh, tq.start, tq.len, dense, weights, true, fP);
    __syncthreads();
  }
}

// The weight updates the aggregation recorded: w = fl32(w - q) at every
// owner's position, one CTA per aggregation group, every weight load of a
// thread issued before its stores.
__global__ void __launch_bounds__(kAggThreads) k_weight_updates(DevPlan dp,
                                                                 float* __restrict__ weights) {
  pdl_trigger();
  pdl_wait();
  const uint32_t n = after_wait(dp.wcnt)[blockIdx.x];
  if (n == 0) return;
  const uint2* rec = after_wait(dp.wrec) + (size_t)blockIdx.x * kAggPickCap;
  constexpr uint32_t OI = kAggPickCap / kAggThreads;
  uint2 r[OI];
  float w[OI];
#pragma unroll
  for (uint32_t j = 0; j < OI; ++j) {
    const uint32_t i = threadIdx.x + j * kAggThreads;
    r[j] = i < n ? __ldg(rec + i) : make_uint2(0xFFFFFFFFu, 0u);
  }
#pragma unroll
  for (uint32_t j = 0; j < OI; ++j)
    if (r[j].x != 0xFFFFFFFFu) w[j] = weights[r[j].x];
#pragma unroll
  for (uint32_t j = 0; j < OI; ++j)
    if (r[j].x != 0xFFFFFFFFu) weights[r[j].x] = __fsub_rn(w[j], __uint_as_float(r[j].y));
}

__global__ void __launch_bounds__(256) k_apply(uint32_t first, uint32_t end,
                                               float* __restrict__ w,
                                               const float* __restrict__ dense) {
  // elements [first, end): a scalar head up to the first 16-byte boundary,
  // float4 over the aligned middle, a scalar tail
  pdl_trigger();
  pdl_wait();
  w = after_wait(w);
  dense = after_wait(dense);
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
                              (int)sizeof(AggShared));
}

cudaError_t launch_aggregate(const DevPlan& dp, const uint32_t* idx, const float* val,
                             float* dense, float* weights, cudaStream_t s) {
  return launch_pdl(k_aggregate, dim3(dp.n_groups), dim3(kAggThreads), sizeof(AggShared), s, 1,
                    dp, idx, val, dense, weights);
}

cudaError_t launch_weight_updates(const DevPlan& dp, float* weights, cudaStream_t s) {
  return launch_pdl(k_weight_updates, dim3(dp.n_groups), dim3(kAggThreads), 0, s, 1, dp, weights);
}

cudaError_t launch_apply(uint32_t first, uint32_t end, float* w, const float* dense,
                         cudaStream_t s) {
  uint32_t blocks = ((end - first) / 4 + 255) / 256;
  if (blocks > 148u * 16u) blocks = 148u * 16u;
  if (blocks == 0) blocks = 1;
  return launch_pdl(k_apply, dim3(blocks), dim3(256), 0, s, 1, first, end, w, dense);
}

}  // namespace lags
