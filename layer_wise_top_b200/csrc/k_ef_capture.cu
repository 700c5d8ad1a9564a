// Fused error-feedback and candidate-capture pass (the streaming hot loop).
//
// One CTA per (tile, worker).  Each thread loads 8 float4 of the gradient and
// 8 float4 of the residual with 128-bit coalesced loads, forms
// acc = fl32(residual + fl32(lr * grad)) (error compensation, "Layer-wise
// Adaptive Gradient Sparsification ..." review, "proposed method") and writes
// acc back over the residual.  This is the only full pass over the data:
// 12 bytes per element (read g, read r, write r).
//
//  - sparse layers: every entry whose magnitude key reaches the layer's
//    sampled threshold lo_key is appended, in index order, to the tile's
//    candidate slots (value, global index), and the tile's candidate count is
//    recorded (counts above the slot capacity mark an overflow);
//  - dense layers (k_l = d_l): every entry is a pick; it goes straight to the
//    pick list and its residual becomes +0.
#include "block_ops.cuh"
#include "lags_internal.cuh"

namespace lags {

// Streaming (evict-first) loads and stores: each byte is touched once.  Plain
// loads/stores measured 13% slower and L2 256-byte prefetch hints no faster.
__device__ __forceinline__ float4 ld_grad(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 ld_resid(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}
__device__ __forceinline__ float comp(const float4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Three CTAs per SM: the 16 float4 loads of a thread stay in flight together
// (about 80 registers), which measured 1.2x faster than four CTAs with loads
// interleaved with arithmetic and than two CTAs with all loads in flight.
//
// Warp w owns the contiguous 1024 entries [w * 1024, (w + 1) * 1024) of the
// tile (lane l takes float4 v * 32 + l of them, so every load and store of a
// warp covers 512 contiguous bytes).  A warp's candidates are then contiguous
// in index order, and a candidate's slot is the candidates of the warps before
// it plus its rank inside its warp: one block barrier per tile, to publish the
// warps' totals.
__global__ void __launch_bounds__(kEfThreads, 3) k_ef_capture(DevPlan dp, WorkerPtrs wp, float lr,
                                                           uint32_t* __restrict__ out_idx,
                                                           float* __restrict__ out_val) {
  constexpr int V = kEfVecPerThread;
  constexpr int NWARP = kEfThreads / 32;
  static_assert(NWARP <= 32, "warp totals fit one warp");
  __shared__ uint32_t s_wtot[NWARP];  // candidates of each warp

  pdl_trigger();
  const uint32_t t = blockIdx.x, p = blockIdx.y;
  const TileDesc td = dp.tiles[t];
  const float* g0 = wp.g[p];
  float* r0 = wp.r[p];
  const uint32_t start = td.start, end = td.start + td.len;
  const uint32_t N = dp.N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // first element of this thread's float4 v: the warp's run, then lane order
  const uint32_t wbase = (start & ~3u) + 4u * (uint32_t)(warp * V * 32 + lane);
  pdl_wait();
  const float* __restrict__ g = after_wait(g0);
  float* __restrict__ r = after_wait(r0);

  float4 a[V];
  float4 gv[V];
  // every load of the tile is issued before any arithmetic
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const uint32_t e0 = wbase + 128u * v;
    gv[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    a[v] = gv[v];
    if (e0 < end) {
      if (e0 + 4 <= N) {
        gv[v] = ld_grad(g + e0);
        a[v] = ld_resid(r + e0);
      } else {
        gv[v].x = g[e0];
        a[v].x = r[e0];
        if (e0 + 1 < N) { gv[v].y = g[e0 + 1]; a[v].y = r[e0 + 1]; }
        if (e0 + 2 < N) { gv[v].z = g[e0 + 2]; a[v].z = r[e0 + 2]; }
      }
    }
  }
  // the layer's descriptor and candidate threshold (the threshold written by
  // k_estimate; unused in dense layers, which have none), behind the loads:
  // loads issued before the dependency wait measured to delay the loads after it
  const LayerDesc ld = after_wait(dp.layers)[td.layer];
  const uint32_t lo = after_wait(dp.lo_key)[(size_t)p * dp.L + td.layer];
#pragma unroll
  for (int v = 0; v < V; ++v) {
    a[v].x = __fadd_rn(a[v].x, __fmul_rn(lr, gv[v].x));
    a[v].y = __fadd_rn(a[v].y, __fmul_rn(lr, gv[v].y));
    a[v].z = __fadd_rn(a[v].z, __fmul_rn(lr, gv[v].z));
    a[v].w = __fadd_rn(a[v].w, __fmul_rn(lr, gv[v].w));
  }

  if (ld.k == ld.d) {
    // dense layer: all entries are picks, residual becomes +0
    const uint64_t ob = (uint64_t)p * dp.K + ld.koff;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint32_t e0 = wbase + 128u * v;
      if (e0 >= end) continue;
      if (e0 >= start && e0 + 4 <= end) {
        st_stream(r + e0, make_float4(0.f, 0.f, 0.f, 0.f));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t e = e0 + j;
        if (e < start || e >= end) continue;
        out_idx[ob + (e - ld.off)] = e;
        out_val[ob + (e - ld.off)] = comp(a[v], j);
        if (!(e0 >= start && e0 + 4 <= end)) r[e] = 0.0f;
      }
    }
    return;
  }

  // sparse layer: write acc back and capture candidates in index order
  uint32_t masks = 0;
  uint32_t excl[V];   // candidates of this warp before this thread's float4 v
  uint32_t run = 0;   // candidates of this warp in float4s v' < v (warp-uniform)
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const uint32_t e0 = wbase + 128u * v;
    uint32_t m4 = 0;
    if (e0 < end) {
      const bool full = e0 >= start && e0 + 4 <= end;
      if (full) st_stream(r + e0, a[v]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t e = e0 + j;
        if (e < start || e >= end) continue;
        const float x = comp(a[v], j);
        if (!full) r[e] = x;
        if (mag_key(x) >= lo) m4 |= 1u << j;
      }
    }
    masks |= m4 << (4 * v);
    const uint32_t c = __popc(m4);
    excl[v] = run;
    if (__ballot_sync(kFull, c != 0u)) {
      const uint32_t incl = warp_incl_scan(c);
      excl[v] = run + incl - c;
      run += __shfl_sync(kFull, incl, 31);
    }
  }
  if (lane == 0) s_wtot[warp] = run;
  __syncthreads();
  // this warp's first slot: the candidates of the warps before it
  const uint32_t wt = lane < NWARP ? s_wtot[lane] : 0u;
  const uint32_t wincl = warp_incl_scan(wt);
  const uint32_t before = __shfl_sync(kFull, wincl - wt, warp);
  const uint32_t total = __shfl_sync(kFull, wincl, NWARP - 1);

  const uint32_t cap = ld.slot_cap;
  const uint64_t slot0 =
      (uint64_t)p * dp.C + ld.slot_base + (uint64_t)(t - ld.tile_begin) * cap;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const uint32_t m4 = (masks >> (4 * v)) & 0xFu;
    if (!m4) continue;
    const uint32_t e0 = wbase + 128u * v;
    uint32_t pos = before + excl[v];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!((m4 >> j) & 1u)) continue;
      if (pos < cap) {
        dp.cand_val[slot0 + pos] = comp(a[v], j);
        dp.cand_idx[slot0 + pos] = e0 + j;
      }
      ++pos;
    }
  }
  if (threadIdx.x == 0) dp.tile_cnt[(size_t)p * dp.T + t] = total;
}

cudaError_t launch_ef_capture(const DevPlan& dp, const WorkerPtrs& wp, float lr,
                              uint32_t* out_idx, float* out_val, cudaStream_t s) {
  dim3 grid(dp.T, dp.P);
  return launch_pdl(k_ef_capture, grid, dim3(kEfThreads), 0, s, 1, dp, wp, lr, out_idx, out_val);
}

}  // namespace lags
