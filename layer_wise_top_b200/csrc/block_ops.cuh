// Block-wide primitives used by the selection kernels: exclusive scan and the
// "which histogram bin holds the r-th largest key" search.
#pragma once

#include <stdint.h>

namespace lags {

constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive scan of v over the block in thread order; *total gets the sum.
// s_warp: shared scratch of NT/32 words.  Contains the barriers it needs and
// leaves s_warp free for reuse on return.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp,
                                                    uint32_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = warp_incl_scan(v);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NW ? s_warp[lane] : 0u;
    w = warp_incl_scan(w);
    if (lane < NW) s_warp[lane] = w;
  }
  __syncthreads();
  uint32_t before = warp > 0 ? s_warp[warp - 1] : 0u;
  *total = s_warp[NW - 1];
  __syncthreads();
  return before + incl - v;
}

template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* s_warp) {
  uint32_t total;
  block_excl_scan<NT>(v, s_warp, &total);
  return total;
}

struct BinPick {
  uint32_t bin;    // bin holding the r-th largest key
  uint32_t above;  // keys in bins above it
  uint32_t count;  // keys in that bin
};

// Over a histogram of bins held in registers (thread t holds bins
// [t * PER, (t + 1) * PER), bin order = key order, zeros past the last bin),
// find the largest bin b with sum(hist[b..)) >= r, for 1 <= r <= sum(hist).
// All threads get the same result (zeros when r exceeds the total).  s_tmp:
// shared scratch of NT/32 + 3 words.
template <int NT, int PER>
__device__ __forceinline__ BinPick block_find_bin_regs(const uint32_t (&h)[PER], uint32_t r,
                                                       uint32_t* s_tmp) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 32, "warp totals fit one warp");
  uint32_t* s_warp = s_tmp;      // NW
  uint32_t* s_res = s_tmp + NW;  // 3
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += h[i];
  // keys in the bins of this thread and the warp's later threads (suffix sum)
  uint32_t suf = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += n;
  }
  if (lane == 0) s_warp[warp] = suf;
  if (t == 0) {
    s_res[0] = 0;
    s_res[1] = 0;
    s_res[2] = 0;
  }
  __syncthreads();
  if (warp == 0) {
    // keys of the warps after each warp (exclusive suffix sum over warps)
    const uint32_t w = lane < NW ? s_warp[lane] : 0u;
    uint32_t ws = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_down_sync(kFull, ws, o);
      if (lane + o < 32) ws += n;
    }
    if (lane < NW) s_warp[lane] = ws - w;
  }
  __syncthreads();
  const uint32_t above = s_warp[warp] + (suf - mine);
  if (above < r && r <= above + mine) {
    uint32_t acc = above;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (acc + h[i] >= r) {
        s_res[0] = (uint32_t)(t * PER + i);
        s_res[1] = acc;
        s_res[2] = h[i];
        break;
      }
      acc += h[i];
    }
  }
  __syncthreads();
  BinPick out{s_res[0], s_res[1], s_res[2]};
  __syncthreads();
  return out;
}

// The same search over a shared histogram of NB bins.
template <int NT, int NB>
__device__ __forceinline__ BinPick block_find_bin(const uint32_t* hist, uint32_t r,
                                                  uint32_t* s_tmp) {
  static_assert(NB % NT == 0 || NT % NB == 0, "bins per thread");
  constexpr int PER = NB >= NT ? NB / NT : 1;
  const int b0 = threadIdx.x * PER;
  uint32_t h[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) h[i] = b0 < NB ? hist[b0 + i] : 0u;
  return block_find_bin_regs<NT, PER>(h, r, s_tmp);
}

}  // namespace lags
