/* Host side of the seeded input generator (see philox.h).  Built with
 * -ffp-contract=off so every float step rounds once, like the device side. */
#include <stdint.h>
#include "philox.h"

void synth_philox_block(const uint32_t ctr[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
  synth_u32x4 c;
  for (int i = 0; i < 4; ++i) c.v[i] = ctr[i];
  synth_u32x4 o = synth_philox4x32_10(c, k0, k1);
  for (int i = 0; i < 4; ++i) out[i] = o.v[i];
}

/* out[i] = value of element first + i, i < count. */
void synth_fill_host(float* out, uint64_t first, uint64_t count, uint32_t seed, uint32_t worker,
                     uint32_t step, int dist, float scale) {
  int64_t n = (int64_t)count;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = synth_value(seed, worker, step, (uint32_t)(first + (uint64_t)i), dist, scale);
}
