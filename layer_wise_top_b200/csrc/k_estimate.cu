// Candidate threshold estimate.
//
// Before the fused pass streams a layer, one CTA per sparse (worker, layer)
// draws a sample of m_l entries of acc = residual + lr*grad (the whole layer
// when it is at most kSampleMax long, otherwise runs of contiguous entries,
// one at a hashed offset inside each of m_l / run equal strata) and finds the
// magnitude key of the sample's r*-th largest entry, rounded down to a
// level-1 radix bin edge.  Segments longer than kSampleShortAbove use runs of
// 16 (1024 strata): such a segment may span tensors of different scales, and
// a run must not stand for a whole stratum of differently scaled values.
// With 64-entry runs, one run inside the 1,728-entry first layer of VGG-16 set
// the threshold of a global top-k over the model above its 14,720th value.
// Shorter segments keep runs of 64, which measured faster there.  The fused pass
// then keeps every entry at or above that key as a candidate.  r* is chosen on
// the host so that, for a sample drawn from the layer, the candidates hold the
// layer's k largest entries with overwhelming probability; when they do not
// (or a tile overflows its candidate slots) the selection kernel falls back to
// an exhaustive radix select, so the estimate only affects speed, never the
// result.  For layers sampled whole r* = k, which makes the bound certain.
#include "block_ops.cuh"
#include "lags_internal.cuh"

namespace lags {

// Integer finaliser (xor-shift-multiply) to place the sample runs.
__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

__global__ void __launch_bounds__(kEstThreads) k_estimate(DevPlan dp, WorkerPtrs wp, float lr) {
  extern __shared__ uint32_t s_keys[];  // kSampleMax
  __shared__ uint32_t s_hist[kBins];
  __shared__ uint32_t s_chunk[kSampleMax / kSampleRunShort];  // first element of each run
  __shared__ uint32_t s_tmp[kEstThreads + kEstThreads / 32 + 4];

  pdl_trigger();
  const uint32_t layer = dp.sparse[blockIdx.x];
  const uint32_t p = blockIdx.y;
  const LayerDesc ld = dp.layers[layer];
  const float* g0 = wp.g[p];
  const float* r0 = wp.r[p];
  const uint32_t m = ld.sample;
  const uint32_t run = ld.d > kSampleShortAbove ? kSampleRunShort : kSampleRunLong;
  const uint32_t run_shift = run == kSampleRunShort ? 4 : 6;  // log2(run)
  static_assert(kSampleRunShort == 16 && kSampleRunLong == 64, "run_shift");
  const uint32_t nchunk = m >> run_shift;
  pdl_wait();
  const float* __restrict__ g = after_wait(g0);
  const float* __restrict__ r = after_wait(r0);

  for (uint32_t i = threadIdx.x; i < kBins; i += kEstThreads) s_hist[i] = 0;
  // sample positions: the whole layer, or nchunk runs of `run` entries spread
  // evenly over it
  if (m != ld.d)
    for (uint32_t c = threadIdx.x; c < nchunk; c += kEstThreads) {
      // stratified: run c lies at a hashed offset inside the c-th of nchunk
      // equal strata, so every region of the layer is sampled in proportion
      const uint32_t a = (uint32_t)((uint64_t)c * ld.d / nchunk);
      const uint32_t b = (uint32_t)((uint64_t)(c + 1) * ld.d / nchunk);
      s_chunk[c] = ld.off + a + mix32(c * 0x9E3779B9u + layer) % (b - a - run + 1);
    }
  __syncthreads();
  constexpr uint32_t U = 8;  // loads per array in flight per thread
  for (uint32_t i0 = 0; i0 < m; i0 += kEstThreads * U) {
    float gv[U], rv[U];
#pragma unroll
    for (uint32_t u = 0; u < U; ++u) {
      const uint32_t i = i0 + u * kEstThreads + threadIdx.x;
      gv[u] = 0.f;
      rv[u] = 0.f;
      if (i < m) {
        const uint32_t e = m == ld.d ? ld.off + i : s_chunk[i >> run_shift] + (i & (run - 1));
        gv[u] = __ldg(g + e);
        rv[u] = __ldg(r + e);
      }
    }
#pragma unroll
    for (uint32_t u = 0; u < U; ++u) {
      const uint32_t i = i0 + u * kEstThreads + threadIdx.x;
      if (i < m) s_keys[i] = mag_key(__fadd_rn(rv[u], __fmul_rn(lr, gv[u])));
    }
  }
  __syncthreads();

  // level 0: bits 30..20
  for (uint32_t i = threadIdx.x; i < m; i += kEstThreads) atomicAdd(&s_hist[s_keys[i] >> 20], 1u);
  __syncthreads();
  BinPick b0 = block_find_bin<kEstThreads, kBins>(s_hist, ld.rank, s_tmp);
  const uint32_t rem = ld.rank - b0.above;
  for (uint32_t i = threadIdx.x; i < kBins; i += kEstThreads) s_hist[i] = 0;
  __syncthreads();
  // level 1: bits 19..9 among keys of bin b0
  for (uint32_t i = threadIdx.x; i < m; i += kEstThreads) {
    const uint32_t k = s_keys[i];
    if ((k >> 20) == b0.bin) atomicAdd(&s_hist[(k >> 9) & 0x7FFu], 1u);
  }
  __syncthreads();
  BinPick b1 = block_find_bin<kEstThreads, kBins>(s_hist, rem, s_tmp);
  if (threadIdx.x == 0) dp.lo_key[(size_t)p * dp.L + layer] = (b0.bin << 20) | (b1.bin << 9);
}

cudaError_t configure_estimate() {
  return cudaFuncSetAttribute(k_estimate, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(kSampleMax * sizeof(uint32_t)));
}

cudaError_t launch_estimate(const DevPlan& dp, const WorkerPtrs& wp, float lr, cudaStream_t s) {
  if (dp.n_sparse == 0) return cudaSuccess;
  dim3 grid(dp.n_sparse, dp.P);
  return launch_pdl(k_estimate, grid, dim3(kEstThreads), kSampleMax * sizeof(uint32_t), s, 1, dp,
                    wp, lr);
}

}  // namespace lags
