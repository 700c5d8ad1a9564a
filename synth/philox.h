/*
 * Seeded synthetic-input generator: Philox4x32-10 counter-based RNG and the
 * gradient distributions built on it.  This header holds no step of the
 * sparsification method; it only manufactures the gradients that are fed to
 * both the CUDA path and the CPU oracle, which is why both sides may use it.
 *
 * Philox4x32-10 follows its published definition: Salmon, Moraes, Dror and
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 4
 * (Philox S-box: two 32x32->64 multiplies, xor with the round key, Weyl key
 * schedule, 10 rounds).
 *
 * Value recipe (identical bits on host and device, since every float step is a
 * single correctly rounded IEEE operation and no libm transcendental is used):
 *   counter = (element, call, worker, step), key = (seed, 0x4C414753)
 *   each call yields 4 words = 8 unsigned 16-bit halves h (low half first)
 *   standard normal  Z = (sum_{i<12} (2 h_i + 1) - 12*65536) * 2^-17
 *                    (Irwin-Hall sum of 12 uniforms, exact integer numerator)
 *   dist 0: value = Z0 * scale                              (calls 0..1)
 *   dist 1: Student-t, nu = 3: q = (Z1^2 + Z2^2 + Z3^2) / 3,
 *           value = (Z0 / sqrt(q)) * scale, with q == 0 read as q == 1
 *                                                           (calls 0..5)
 */
#ifndef SYNTH_PHILOX_H
#define SYNTH_PHILOX_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN __host__ __device__ static inline
#else
#define SYNTH_FN static inline
#include <math.h>
#endif

#if defined(__CUDA_ARCH__)
#define SYNTH_FMUL(a, b) __fmul_rn((a), (b))
#define SYNTH_FADD(a, b) __fadd_rn((a), (b))
#define SYNTH_FDIV(a, b) __fdiv_rn((a), (b))
#define SYNTH_FSQRT(a) __fsqrt_rn(a)
#define SYNTH_I2F(a) __int2float_rn(a)
#else
#define SYNTH_FMUL(a, b) ((float)((a) * (b)))
#define SYNTH_FADD(a, b) ((float)((a) + (b)))
#define SYNTH_FDIV(a, b) ((float)((a) / (b)))
#define SYNTH_FSQRT(a) sqrtf(a)
#define SYNTH_I2F(a) ((float)(a))
#endif

#define SYNTH_KEY_HI 0x4C414753u /* "LAGS" */

typedef struct {
  uint32_t v[4];
} synth_u32x4;

SYNTH_FN void synth_mulhilo(uint32_t a, uint32_t b, uint32_t* hi, uint32_t* lo) {
  uint64_t p = (uint64_t)a * (uint64_t)b;
  *hi = (uint32_t)(p >> 32);
  *lo = (uint32_t)p;
}

/* One Philox4x32-10 block: 10 rounds of the S-box with the key bumped by the
 * Weyl constants between rounds. */
SYNTH_FN synth_u32x4 synth_philox4x32_10(synth_u32x4 c, uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint32_t hi0, lo0, hi1, lo1;
    synth_mulhilo(0xD2511F53u, c.v[0], &hi0, &lo0);
    synth_mulhilo(0xCD9E8D57u, c.v[2], &hi1, &lo1);
    synth_u32x4 n;
    n.v[0] = hi1 ^ c.v[1] ^ k0;
    n.v[1] = lo1;
    n.v[2] = hi0 ^ c.v[3] ^ k1;
    n.v[3] = lo0;
    c = n;
  }
  return c;
}

/* Irwin-Hall standard normal from 12 consecutive 16-bit halves of the word
 * stream w[] starting at half index h0. */
SYNTH_FN float synth_normal_from_words(const uint32_t* w, int h0) {
  int32_t num = 0;
  for (int i = 0; i < 12; ++i) {
    int h = h0 + i;
    uint32_t word = w[h >> 1];
    uint32_t half = (h & 1) ? (word >> 16) : (word & 0xFFFFu);
    num += (int32_t)(2u * half + 1u);
  }
  num -= 12 * 65536;
  return SYNTH_FMUL(SYNTH_I2F(num), 7.62939453125e-06f /* 2^-17 */);
}

/* Value of element `elem` of worker `worker` at step `step`. */
SYNTH_FN float synth_value(uint32_t seed, uint32_t worker, uint32_t step, uint32_t elem,
                           int dist, float scale) {
  uint32_t w[24];
  int ncalls = dist == 0 ? 2 : 6;
  for (int call = 0; call < ncalls; ++call) {
    synth_u32x4 c;
    c.v[0] = elem;
    c.v[1] = (uint32_t)call;
    c.v[2] = worker;
    c.v[3] = step;
    synth_u32x4 o = synth_philox4x32_10(c, seed, SYNTH_KEY_HI);
    w[4 * call + 0] = o.v[0];
    w[4 * call + 1] = o.v[1];
    w[4 * call + 2] = o.v[2];
    w[4 * call + 3] = o.v[3];
  }
  float z0 = synth_normal_from_words(w, 0);
  if (dist == 0) return SYNTH_FMUL(z0, scale);
  float z1 = synth_normal_from_words(w, 12);
  float z2 = synth_normal_from_words(w, 24);
  float z3 = synth_normal_from_words(w, 36);
  float q = SYNTH_FMUL(z1, z1);
  q = SYNTH_FADD(q, SYNTH_FMUL(z2, z2));
  q = SYNTH_FADD(q, SYNTH_FMUL(z3, z3));
  q = SYNTH_FDIV(q, 3.0f);
  if (q == 0.0f) q = 1.0f;
  float t = SYNTH_FDIV(z0, SYNTH_FSQRT(q));
  return SYNTH_FMUL(t, scale);
}

#endif /* SYNTH_PHILOX_H */
