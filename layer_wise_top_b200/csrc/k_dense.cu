// Dense S-SGD, the baseline LAGS-SGD is measured against ("Layer-wise
// Adaptive Gradient Sparsification ..." review, main findings: LAGS-SGD
// against dense S-SGD, where every worker sends its whole gradient and the
// averaged gradient updates the model).
//
// k_dense_sum:    sum_j = (((+0 + fl(lr g_0j)) + fl(lr g_1j)) + ...), workers
//                 in order: the dense sum of every worker's error-feedback
//                 value with a zero residual, i.e. exactly the sum a LAGS step
//                 with density 1 forms.  Across ranks the caller all-reduces
//                 these partial sums.
// k_dense_finish: dense_j = fl(sum_j / P), and optionally w_j = fl(w_j - dense_j).
//
// Both are streams over HBM: each thread owns 4 consecutive elements and keeps
// kDenseBatch workers' 16-byte loads in flight before adding them in order.
#include "lags_internal.cuh"

namespace lags {

constexpr int kDenseBatch = 8;
constexpr uint32_t kDenseThreads = 256;

__global__ void __launch_bounds__(kDenseThreads) k_dense_sum(DenseGrads gp, uint32_t P,
                                                             uint64_t N, float lr,
                                                             float* __restrict__ sum) {
  pdl_trigger();
  pdl_wait();  // (the gradients come from the caller's work, which does not
               // trigger dependents early: no read below can precede it)
  const uint64_t n4 = N / 4;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  const uint64_t gid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (uint64_t i = gid; i < n4; i += stride) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (uint32_t p0 = 0; p0 < P; p0 += kDenseBatch) {
      float4 v[kDenseBatch];
#pragma unroll
      for (int u = 0; u < kDenseBatch; ++u)
        if (p0 + u < P) v[u] = __ldcs(reinterpret_cast<const float4*>(gp.g[p0 + u]) + i);
#pragma unroll
      for (int u = 0; u < kDenseBatch; ++u) {
        if (p0 + u >= P) break;
        acc.x = __fadd_rn(acc.x, __fmul_rn(lr, v[u].x));
        acc.y = __fadd_rn(acc.y, __fmul_rn(lr, v[u].y));
        acc.z = __fadd_rn(acc.z, __fmul_rn(lr, v[u].z));
        acc.w = __fadd_rn(acc.w, __fmul_rn(lr, v[u].w));
      }
    }
    reinterpret_cast<float4*>(sum)[i] = acc;
  }
  const uint64_t t = n4 * 4 + gid;  // the last N % 4 elements
  if (t < N) {
    float a = 0.0f;
    for (uint32_t p = 0; p < P; ++p) a = __fadd_rn(a, __fmul_rn(lr, gp.g[p][t]));
    sum[t] = a;
  }
}

__global__ void __launch_bounds__(kDenseThreads) k_dense_finish(const float* __restrict__ sum,
                                                                uint64_t N, float fP,
                                                                float* __restrict__ dense,
                                                                float* __restrict__ weights) {
  pdl_trigger();
  pdl_wait();
  sum = after_wait(sum);
  const uint64_t n4 = N / 4;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  const uint64_t gid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (uint64_t i = gid; i < n4; i += stride) {
    const float4 s = __ldcs(reinterpret_cast<const float4*>(sum) + i);
    const float4 d = make_float4(__fdiv_rn(s.x, fP), __fdiv_rn(s.y, fP), __fdiv_rn(s.z, fP),
                                 __fdiv_rn(s.w, fP));
    reinterpret_cast<float4*>(dense)[i] = d;
    if (weights) {
      float4 w = reinterpret_cast<const float4*>(weights)[i];
      w.x = __fsub_rn(w.x, d.x);
      w.y = __fsub_rn(w.y, d.y);
      w.z = __fsub_rn(w.z, d.z);
      w.w = __fsub_rn(w.w, d.w);
      reinterpret_cast<float4*>(weights)[i] = w;
    }
  }
  const uint64_t t = n4 * 4 + gid;
  if (t < N) {
    const float d = __fdiv_rn(sum[t], fP);
    dense[t] = d;
    if (weights) weights[t] = __fsub_rn(weights[t], d);
  }
}

namespace {
uint32_t dense_blocks(uint64_t N) {
  uint64_t b = (N / 4 + kDenseThreads - 1) / kDenseThreads;
  if (b > 148u * 16u) b = 148u * 16u;
  return b ? (uint32_t)b : 1u;
}
}  // namespace

cudaError_t launch_dense_sum(const DenseGrads& gp, uint32_t P, uint64_t N, float lr, float* sum,
                             cudaStream_t s) {
  return launch_pdl(k_dense_sum, dim3(dense_blocks(N)), dim3(kDenseThreads), 0, s, 1, gp, P, N,
                    lr, sum);
}

cudaError_t launch_dense_finish(const float* sum, uint64_t N, uint32_t P, float* dense,
                                float* weights, cudaStream_t s) {
  return launch_pdl(k_dense_finish, dim3(dense_blocks(N)), dim3(kDenseThreads), 0, s, 1, sum, N,
                    (float)P, dense, weights);
}

}  // namespace lags
