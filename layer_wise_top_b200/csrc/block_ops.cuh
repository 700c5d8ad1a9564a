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

// Over a shared histogram of NB bins (bin order = key order), find the largest
// bin b with sum(hist[b..NB)) >= r, for 1 <= r <= sum(hist).  All threads get
// the same result.  s_tmp: shared scratch of NT + NT/32 + 3 words.
template <int NT, int NB>
__device__ __forceinline__ BinPick block_find_bin(const uint32_t* hist, uint32_t r,
                                                  uint32_t* s_tmp) {
  static_assert(NB % NT == 0 || NT % NB == 0, "bins per thread");
  constexpr int PER = NB >= NT ? NB / NT : 1;
  uint32_t* s_sum = s_tmp;             // NT
  uint32_t* s_warp = s_tmp + NT;       // NT/32
  uint32_t* s_res = s_warp + NT / 32;  // 3
  const int t = threadIdx.x;
  const int b0 = t * PER;
  uint32_t mine = 0;
  if (b0 < NB) {
#pragma unroll
    for (int i = 0; i < PER; ++i) mine += hist[b0 + i];
  }
  s_sum[t] = mine;
  if (t == 0) {  // defined result even if r exceeded the histogram total
    s_res[0] = 0;
    s_res[1] = 0;
    s_res[2] = 0;
  }
  __syncthreads();
  // exclusive scan in descending thread order: thread t scans position NT-1-t
  uint32_t rv = s_sum[NT - 1 - t];
  uint32_t tot;
  uint32_t ex = block_excl_scan<NT>(rv, s_warp, &tot);
  s_sum[NT - 1 - t] = ex;  // = keys in the bins of threads above NT-1-t
  __syncthreads();
  uint32_t above = s_sum[t];
  if (b0 < NB && above < r && r <= above + mine) {
    uint32_t acc = above;
    for (int i = PER - 1; i >= 0; --i) {
      uint32_t h = hist[b0 + i];
      if (acc + h >= r) {
        s_res[0] = (uint32_t)(b0 + i);
        s_res[1] = acc;
        s_res[2] = h;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
  BinPick out{s_res[0], s_res[1], s_res[2]};
  __syncthreads();
  return out;
}

}  // namespace lags
