// Device side of the seeded input generator (see philox.h).  A test and bench
// fixture: it fills gradient buffers on the GPU with the same bits the host
// generator produces, so large workloads need not cross PCIe.
#include <cuda_runtime.h>
#include <stdint.h>
#include "philox.h"

__global__ void synth_fill_kernel(float* __restrict__ out, uint64_t first, uint64_t count,
                                  uint32_t seed, uint32_t worker, uint32_t step, int dist,
                                  float scale) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
    out[i] = synth_value(seed, worker, step, (uint32_t)(first + i), dist, scale);
}

extern "C" int synth_fill_device(float* out, uint64_t first, uint64_t count, uint32_t seed,
                                 uint32_t worker, uint32_t step, int dist, float scale,
                                 cudaStream_t stream) {
  if (count == 0) return 0;
  uint64_t blocks = (count + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  synth_fill_kernel<<<(unsigned)blocks, 256, 0, stream>>>(out, first, count, seed, worker, step,
                                                          dist, scale);
  return (int)cudaGetLastError();
}
