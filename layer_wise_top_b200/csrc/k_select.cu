// Exact per-layer top-k (radix select) and ordered emission.
//
// One thread-block cluster of CL CTAs per sparse (worker, layer); each CTA owns
// a contiguous, index-ordered share of the layer.  The CTAs count the layer's
// candidates; if the sampled threshold held (at least k_l candidates, and
// every tile that overflowed its slots lies in a share that can be staged)
// they work on the candidate lists, otherwise on the full acc of the layer
// (held in the residual buffer after the fused pass).  Either way the result
// is the exact top-k of the layer.
//
// CL is 1, 4, 8, or 16.  4-CTA clusters stage candidate values only (4 bytes
// instead of 8), which keeps two CTAs per SM for layers whose candidates
// would otherwise need 8-CTA clusters; after the emission they copy the
// candidates' indices over the stage for the index write-back.  16 is used
// for layers whose candidates need more shared memory than 8 CTAs hold, and
// it is a non-portable cluster size used only where the occupancy query says
// it fits.  Shares are equal tile ranges; a crowded clustered segment
// (overflow that equal shares cannot stage) is split again into shares of
// equal candidate counts.
//
// A CTA whose candidates fit in shared memory stages them there, with plain
// bulk copies (cp.async.bulk, one per tile and array, completing on one
// mbarrier).  An overflowed tile is instead recompacted from its acc by the
// whole CTA.  Every pass below then reads shared memory only.  The exhaustive
// path walks the acc in rounds of 4 consecutive entries per thread.
//
//  1. radix select on the magnitude key (bits 30..20, 19..9, 8..0): every CTA
//     builds a shared-memory histogram of its share (warp-aggregated with
//     __match_any_sync on the exhaustive path), the CTAs add their nonzero
//     bins into CTA 0's histogram through distributed shared memory, and every
//     CTA reads the merged histogram into registers to pick the bin holding
//     the k-th largest key.  It stops early once a whole bin is taken.  The
//     result is a key prefix (shift s, value T): entries with key>>s > T are
//     picks, entries with key>>s == T are ties of which the `need` lowest
//     indices are picks ("lower index wins").
//  2. each CTA counts its strict picks and ties, the counts are exchanged, and
//     each CTA emits its picks in index order at
//         pos = strict_before + min(need, ties_before)
//     (staged shares: warp ballots; otherwise block-wide scans), writing
//     (index, acc) to the pick list and +0 over the picked residuals.
// No CTA ever waits on another outside the hardware cluster barrier.
#include <cooperative_groups.h>

#include <mutex>
#include <type_traits>
#include <vector>

#include "block_ops.cuh"
#include "lags_internal.cuh"
#include "tma.cuh"

namespace cg = cooperative_groups;

namespace lags {

namespace {

template <int CL>
struct Cluster {
  __device__ __forceinline__ static void sync() {
    if constexpr (CL > 1) {
      cg::this_cluster().sync();
    } else {
      __syncthreads();
    }
  }
  __device__ __forceinline__ static uint32_t rank() {
    if constexpr (CL > 1) {
      return cg::this_cluster().block_rank();
    } else {
      return 0;
    }
  }
  // split cluster barrier: arrive once this CTA no longer reads its peers'
  // shared memory, wait before leaving (so no peer's memory goes away while
  // it is read); no-ops for a single CTA
  __device__ __forceinline__ static void arrive() {
    if constexpr (CL > 1) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  }
  __device__ __forceinline__ static void wait() {
    if constexpr (CL > 1) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  }
  template <typename T>
  __device__ __forceinline__ static T* remote(T* p, uint32_t r) {
    if constexpr (CL > 1) {
      return cg::this_cluster().map_shared_rank(p, r);
    } else {
      return p;
    }
  }
};

template <int NT>
struct SelectShared {
  uint32_t tpre[kSelectWindow + 1];
  uint32_t tmp[NT + NT / 32 + 4];
  uint32_t xch[4];               // read by the other CTAs of the cluster
  uint32_t split[2];             // first tiles of this CTA's and the next CTA's share
};

}  // namespace

template <int CL, int NT, bool VO>
__global__ void __launch_bounds__(NT, CL == 1 ? 4 : 2) k_select(DevPlan dp, WorkerPtrs wp, const uint32_t* list,
                                               uint32_t stage_cap,
                                               uint32_t* __restrict__ out_idx,
                                               float* __restrict__ out_val) {
  using C = Cluster<CL>;
  __shared__ SelectShared<NT> sh;
  // this CTA's histogram of the current radix level
  __shared__ __align__(16) uint32_t hist[kBins];
  // CTA 0 of a cluster: the cluster-wide histogram of each level
  __shared__ __align__(16) uint32_t merged[CL > 1 ? 3 : 1][CL > 1 ? kBins : 4];
  // staged candidates: stage_cap values, then (unless VO: values only) their
  // stage_cap global indices
  extern __shared__ __align__(16) float stage_val[];
  uint32_t* stage_idx = reinterpret_cast<uint32_t*>(stage_val + stage_cap);
  __shared__ __align__(8) uint64_t stage_bar;  // completion of the bulk copies
  pdl_trigger();
  const uint32_t rank = C::rank();
  const uint32_t layer = list[blockIdx.x / CL];
  const uint32_t p = blockIdx.y;
  const LayerDesc ld = dp.layers[layer];
  const int tid = threadIdx.x, lane = tid & 31;
  float* r0 = wp.r[p];
  pdl_wait();
  float* __restrict__ r = after_wait(r0);
  const float* __restrict__ cand_val = after_wait(dp.cand_val);
  const uint32_t* __restrict__ cand_idx = after_wait(dp.cand_idx);

  for (int i = tid; i < (int)kBins; i += NT) {
    hist[i] = 0;
    if constexpr (CL > 1) {
#pragma unroll
      for (int q = 0; q < 3; ++q) merged[q][i] = 0;
    }
  }

  // ---- mode: candidate lists or exhaustive ----
  const uint32_t nt = ld.tile_end - ld.tile_begin;
  // this CTA's share of the segment: equal tile ranges (see below for the
  // candidate-balanced split a crowded segment gets)
  uint32_t ta = ld.tile_begin + (uint32_t)((uint64_t)nt * rank / CL);
  uint32_t tb = ld.tile_begin + (uint32_t)((uint64_t)nt * (rank + 1) / CL);
  const uint32_t cap = ld.slot_cap;
  const uint32_t* cnt = after_wait(dp.tile_cnt) + (size_t)p * dp.T;
  uint32_t my = 0, ovf = 0, pad = 0;
  for (uint32_t t = ta + tid; t < tb; t += NT) {
    const uint32_t c = __ldg(cnt + t);
    my += c;
    ovf |= c > cap;
    pad += (c + 3u) & ~3u;
  }
  my = block_sum<NT>(my, sh.tmp);
  ovf = block_sum<NT>(ovf, sh.tmp);
  if (ovf) pad = block_sum<NT>(pad, sh.tmp);  // (block-uniform; only needed then)
  // A tile whose candidates overflowed its slots is still usable when this
  // CTA stages its share: the CTA then recompacts that tile's candidates from
  // its acc (held in the residual buffer) instead of copying the slots.  Only
  // an overflow in a share that cannot be staged forces the exhaustive path.
  const uint32_t lo_key = after_wait(dp.lo_key)[(size_t)p * dp.L + layer];
  const bool stageable =
      ovf && tb - ta <= kSelectWindow && lo_key >= (1u << 20) && pad <= stage_cap;
  if (tid == 0) {
    sh.xch[0] = my;
    sh.xch[1] = ovf && !stageable;
  }
  C::sync();  // also publishes the zeroed histograms cluster-wide
  uint64_t total = 0;
  uint32_t any_bad = 0;
#pragma unroll
  for (int q = 0; q < CL; ++q) {
    const uint32_t* x = C::remote(sh.xch, q);
    total += x[0];
    any_bad |= x[1];
  }
  bool fast = !any_bad && total >= ld.k;
  if constexpr (CL > 1) {
    if (any_bad && total >= ld.k) {  // cluster-uniform: every CTA read the same words
      // A crowded segment (its large values gather in a few tiles, as in a
      // global top-k over tensors of different scales) overflows one CTA's
      // stage under equal tile shares.  Split it again so that every CTA
      // holds about the same number of (padded) candidates: CTA r takes the
      // tiles whose candidate prefix lies in [total r / CL, total (r+1) / CL).
      // The shares stay contiguous and in index order.
      uint32_t ptot = 0;
      for (uint32_t t = ld.tile_begin + tid; t < ld.tile_end; t += NT)
        ptot += (__ldg(cnt + t) + 3u) & ~3u;
      ptot = block_sum<NT>(ptot, sh.tmp);
      const uint64_t lo_t = (uint64_t)ptot * rank / CL, hi_t = (uint64_t)ptot * (rank + 1) / CL;
      if (tid < 2) sh.split[tid] = ld.tile_end;
      uint64_t run = 0;  // candidates before the window
      for (uint32_t w0 = ld.tile_begin; w0 < ld.tile_end; w0 += NT) {
        const uint32_t t = w0 + tid;
        const uint32_t c = t < ld.tile_end ? (__ldg(cnt + t) + 3u) & ~3u : 0u;
        uint32_t wtot;
        const uint64_t pre = run + block_excl_scan<NT>(c, sh.tmp, &wtot);
        if (t < ld.tile_end && pre >= lo_t) atomicMin(&sh.split[0], t);
        if (t < ld.tile_end && pre >= hi_t) atomicMin(&sh.split[1], t);
        run += wtot;
      }
      __syncthreads();
      ta = rank == 0 ? ld.tile_begin : sh.split[0];
      tb = rank == CL - 1 ? ld.tile_end : sh.split[1];
      ovf = 0;
      pad = 0;
      for (uint32_t t = ta + tid; t < tb; t += NT) {
        const uint32_t c = __ldg(cnt + t);
        ovf |= c > cap;
        pad += (c + 3u) & ~3u;
      }
      ovf = block_sum<NT>(ovf, sh.tmp);
      pad = block_sum<NT>(pad, sh.tmp);
      const bool stageable2 =
          tb - ta <= kSelectWindow && lo_key >= (1u << 20) && pad <= stage_cap;
      C::sync();  // every CTA has read the first exchange
      if (tid == 0) sh.xch[1] = ovf && !stageable2;
      C::sync();
      any_bad = 0;
#pragma unroll
      for (int q = 0; q < CL; ++q) any_bad |= C::remote(sh.xch, q)[1];
      fast = !any_bad;
    }
  }
  if (!fast && rank == 0 && tid == 0) atomicAdd(dp.status + kStatusFallbacks, 1u);

  const uint32_t ea = ld.off + (uint32_t)((uint64_t)ld.d * rank / CL);
  const uint32_t eb = ld.off + (uint32_t)((uint64_t)ld.d * (rank + 1) / CL);
  const uint64_t cbase = (uint64_t)p * dp.C + ld.slot_base;

  // Visit this CTA's share in index order, NT entries per round; every thread
  // calls fn(valid, idx, val) once per round, so fn may contain barriers.
  // `stream_candidates` walks the candidate slots tile by tile (gathering
  // through a window of tile prefix sums); once the share has been copied to
  // shared memory (`staged`) the walks read it from there.
  auto stream_candidates = [&](auto&& fn) {
    uint32_t seen = 0;  // candidates of earlier windows
    for (uint32_t w0 = ta; w0 < tb; w0 += kSelectWindow) {
      const uint32_t nw = min(kSelectWindow, tb - w0);
      constexpr int PER = kSelectWindow / NT;
      uint32_t c[PER], sum = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const uint32_t q = tid * PER + i;
        c[i] = q < nw ? __ldg(cnt + w0 + q) : 0u;
        sum += c[i];
      }
      uint32_t wtotal;
      uint32_t ex = block_excl_scan<NT>(sum, sh.tmp, &wtotal);
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const uint32_t q = tid * PER + i;
        if (q < nw) sh.tpre[q] = ex;
        ex += c[i];
      }
      __syncthreads();
      for (uint32_t b = 0; b < wtotal; b += NT) {
        const uint32_t v = b + tid;
        bool valid = v < wtotal;
        uint32_t idx = 0;
        float val = 0.f;
        if (valid) {
          uint32_t lo = 0, hi = nw - 1;
          while (lo < hi) {
            const uint32_t mid = (lo + hi + 1) >> 1;
            if (sh.tpre[mid] <= v) lo = mid; else hi = mid - 1;
          }
          const uint32_t in_tile = v - sh.tpre[lo];
          if (in_tile < cap) {
            const uint64_t slot = cbase + (uint64_t)(w0 + lo - ld.tile_begin) * cap + in_tile;
            idx = __ldg(cand_idx + slot);
            val = __ldg(cand_val + slot);
          } else {
            // an overflowed tile walked from its slots (only after a staging
            // timeout): the slots end at cap, so report and skip the rest
            atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
            valid = false;
          }
        }
        fn(valid, seen + v, idx, val);
      }
      seen += wtotal;
      __syncthreads();
    }
  };
  // Staged share: this CTA's candidate runs (one per tile, in index order) are
  // copied to shared memory by the bulk-copy engine, one cp.async.bulk per
  // tile and array, completing on one mbarrier.  Each run is padded to a
  // 16-byte multiple with entries of magnitude key 0; the share is staged only
  // when the candidate threshold is at least 2^20 (level-0 bin >= 1), so every
  // real candidate outranks the padding and the padding is never counted into
  // a pick, a tie or the bin holding the k-th largest key.
  bool staged = false, stage_timeout = false;
  uint32_t my_pad = 0;  // staged entries, padding included
  if (fast && tb - ta <= kSelectWindow && lo_key >= (1u << 20)) {
    const uint32_t nw = tb - ta;
    constexpr int PER = kSelectWindow / NT;
    uint32_t c[PER], sum = 0, bulk = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const uint32_t q = tid * PER + i;
      const uint32_t raw = q < nw ? __ldg(cnt + ta + q) : 0u;
      c[i] = (raw + 3u) & ~3u;
      sum += c[i];
      // entries the bulk copies bring: every run except an overflowed tile's
      if (raw <= cap) bulk += c[i];
    }
    uint32_t ex = block_excl_scan<NT>(sum, sh.tmp, &my_pad);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const uint32_t q = tid * PER + i;
      if (q < nw) sh.tpre[q] = ex;
      ex += c[i];
    }
    staged = my_pad <= stage_cap;  // block-uniform (== stageable)
    bulk = block_sum<NT>(bulk, sh.tmp);  // (from this thread's own counts, not tpre)
    if (tid == 0) {
      sh.tpre[nw] = my_pad;
      mbar_init(&stage_bar, 1);
      mbar_init_fence();
      if (staged) mbar_arrive_expect_tx(&stage_bar, bulk * (VO ? 4u : 8u));  // before any copy
    }
    __syncthreads();
    if (staged) {
      for (uint32_t q = tid; q < nw; q += NT) {
        const uint32_t n = sh.tpre[q + 1] - sh.tpre[q];
        if (n == 0 || __ldg(cnt + ta + q) > cap) continue;
        const uint64_t slot = cbase + (uint64_t)(ta + q - ld.tile_begin) * cap;
        bulk_load(stage_val + sh.tpre[q], cand_val + slot, n * 4u, &stage_bar);
        if constexpr (!VO) bulk_load(stage_idx + sh.tpre[q], cand_idx + slot, n * 4u, &stage_bar);
      }
      if (ovf) {
        // overflowed tiles: the CTA recompacts the entries with key >= lo_key
        // from the tile's acc, in index order (each thread a contiguous run)
        constexpr uint32_t PT = kTile / NT;
        for (uint32_t q = 0; q < nw; ++q) {
          const uint32_t n = __ldg(cnt + ta + q);  // block-uniform
          if (n <= cap) continue;
          const TileDesc tq = dp.tiles[ta + q];
          const uint32_t e0 = tq.start + tid * PT;
          const uint32_t mine = tid * PT < tq.len ? min(PT, tq.len - tid * PT) : 0u;
          uint32_t c = 0;
          for (uint32_t j = 0; j < mine; ++j) c += mag_key(r[e0 + j]) >= lo_key;
          uint32_t found;
          uint32_t at = block_excl_scan<NT>(c, sh.tmp, &found);
          const uint32_t room = sh.tpre[q + 1] - sh.tpre[q];
          if (tid == 0 && found != n) atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
          for (uint32_t j = 0; j < mine; ++j) {  // (the run is in L1 from the count)
            const float x = r[e0 + j];
            if (mag_key(x) >= lo_key) {
              if (at < room) {
                stage_val[sh.tpre[q] + at] = x;
                if constexpr (!VO) stage_idx[sh.tpre[q] + at] = e0 + j;
              }
              ++at;
            }
          }
          // if the self-check failed with fewer entries than counted, the rest
          // of the run is padding, never uninitialised shared memory
          for (uint32_t j = min(found, room) + tid; j < room; j += NT) {
            stage_val[sh.tpre[q] + j] = 0.0f;
            if constexpr (!VO) stage_idx[sh.tpre[q] + j] = 0xFFFFFFFFu;
          }
        }
      }
      const bool ok = mbar_wait_bounded(&stage_bar, 0, dp.stage_spin);
      if (__syncthreads_or(!ok)) {
        // the copies did not complete: report, and select from global memory
        // (the share's acc, see walk_share below)
        if (tid == 0) atomicOr(dp.status + kStatusFlags, LAGS_FLAG_TIMEOUT);
        staged = false;
        stage_timeout = true;
      } else {
        for (uint32_t q = tid; q < nw; q += NT) {  // padding: key 0, no index
          const uint32_t real = __ldg(cnt + ta + q);
          for (uint32_t j = sh.tpre[q] + real; j < sh.tpre[q + 1]; ++j) {
            stage_val[j] = 0.0f;
            if constexpr (!VO) stage_idx[j] = 0xFFFFFFFFu;
          }
        }
        __syncthreads();
      }
    }
  }
  // (Candidate lists and counts are read through the read-only path: nothing
  // writes them during this kernel, and plain loads would be ordered behind the
  // emission's scattered stores, which measured 6x slower.)
  // Unstaged shares: every pass walks the candidates (or, on the exhaustive
  // path, the layer's acc) from global memory.
  // After a staging timeout the share's candidates are taken from its acc
  // instead of the slots (a tile that overflowed its slots has only part of
  // its candidates there): every entry of the share with key >= lo_key, one
  // entry per thread and round, in index order.  Slower, same candidates.
  uint32_t sa = 0, sb = 0;
  if (stage_timeout && ta < tb) {
    sa = __ldg(&dp.tiles[ta].start);
    sb = __ldg(&dp.tiles[tb - 1].start) + __ldg(&dp.tiles[tb - 1].len);
  }
  auto walk_share = [&](auto&& fn) {
    for (uint32_t b = sa; b < sb; b += NT) {
      const uint32_t e = b + tid;
      const float x = e < sb ? r[e] : 0.0f;
      fn(e < sb && mag_key(x) >= lo_key, e, x);
    }
  };
  auto traverse = [&](auto&& fn) {
    if (stage_timeout) {
      walk_share(fn);
    } else {
      stream_candidates(
          [&](bool valid, uint32_t, uint32_t idx, float val) { fn(valid, idx, val); });
    }
  };
  // Exhaustive path: the CTA's element share [ea, eb) of the layer's acc, in
  // rounds of NT * kExhV elements; each thread takes kExhV consecutive
  // elements per round (index order = thread order within a round).
  constexpr uint32_t kExhV = 4;
  auto exh_load = [&](uint32_t base, float (&v)[kExhV]) {
#pragma unroll
    for (uint32_t j = 0; j < kExhV; ++j) {
      const uint32_t e = base + tid * kExhV + j;
      v[j] = e < eb ? r[e] : 0.f;
    }
  };

  // One radix level: histogram of digit (key >> dshift) & dmask over the keys
  // whose prefix key >> mshift equals mval (all keys when mshift == 32), in
  // this CTA's hist (cleared for each level after the first).
  // staged share, for the ordered emission: warp w owns the contiguous
  // positions [wb, we) and walks them 32 at a time
  constexpr uint32_t NW = NT / 32;
  const uint32_t warp = tid >> 5;
  const uint32_t wspan = (my_pad + NW - 1) / NW;
  const uint32_t wb = min(my_pad, warp * wspan), we = min(my_pad, wb + wspan);
  const unsigned lanes_below = (1u << lane) - 1u;

  auto hist_level = [&](int level, int mshift, uint32_t mval, int dshift, uint32_t dmask) {
    uint32_t* hl = hist;
    if (level > 0) {  // (the previous level's reads of it ended in its search)
      for (int i = tid; i < (int)kBins; i += NT) hl[i] = 0;
      __syncthreads();
    }
    if (staged) {
      for (uint32_t i = tid; i < my_pad; i += NT) {
        const uint32_t key = mag_key(stage_val[i]);
        if (mshift >= 32 || (key >> mshift) == mval)
          atomicAdd(&hl[(key >> dshift) & dmask], 1u);
      }
    } else if (fast) {
      traverse([&](bool valid, uint32_t, float val) {
        // candidates sit in the sparse tail: few collisions
        const uint32_t key = mag_key(val);
        if (valid && (mshift >= 32 || (key >> mshift) == mval))
          atomicAdd(&hl[(key >> dshift) & dmask], 1u);
      });
    } else {
      // a whole layer: keys crowd into few bins, add once per warp and bin
      for (uint32_t base = ea; base < eb; base += NT * kExhV) {
        float v[kExhV];
        exh_load(base, v);
#pragma unroll
        for (uint32_t j = 0; j < kExhV; ++j) {
          const uint32_t key = mag_key(v[j]);
          const bool m = base + tid * kExhV + j < eb && (mshift >= 32 || (key >> mshift) == mval);
          const uint32_t dig = m ? ((key >> dshift) & dmask) : 0xFFFFFFFFu;
          const unsigned peers = __match_any_sync(kFull, dig);
          if (m && lane == __ffs(peers) - 1) atomicAdd(&hl[dig], (uint32_t)__popc(peers));
        }
      }
    }
  };
  // The cluster-wide histogram of a level (the CTAs add their nonzero bins
  // into CTA 0's merged copy through distributed shared memory) and the bin
  // holding the r-th largest key; thread t reads bins [t PER, t PER + PER)
  // into registers for the search.
  auto merge_find = [&](int level, auto nb, uint32_t r) {
    constexpr int NB = decltype(nb)::value;
    static_assert(NB % NT == 0 || NT % NB == 0, "bins per thread");
    constexpr int PER = NB >= NT ? NB / NT : 1;
    __syncthreads();  // this CTA's histogram is complete
    const uint32_t* src = hist;
    if constexpr (CL > 1) {
      uint32_t* dst = C::remote(merged[level], 0);
      for (int i = tid; i < NB; i += NT) {
        const uint32_t h = hist[i];
        if (h) atomicAdd(dst + i, h);
      }
      C::sync();
      src = C::remote(merged[level], 0);
    }
    uint32_t h[PER];
    const int b0 = tid * PER;
    if constexpr (PER == 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(src + b0);
      h[0] = x.x;
      h[1] = x.y;
      h[2] = x.z;
      h[3] = x.w;
    } else {
#pragma unroll
      for (int i = 0; i < PER; ++i) h[i] = b0 < NB ? src[b0 + i] : 0u;
    }
    return block_find_bin_regs<NT, PER>(h, r, sh.tmp);
  };

  // ---- radix select ----
  uint32_t rem = ld.k;
  int fshift;
  uint32_t fpfx;
  {
    hist_level(0, 32, 0, kDigitShift0, 0x7FFu);
    BinPick b = merge_find(0, std::integral_constant<int, kBins>(), rem);
    rem -= b.above;
    fpfx = b.bin;
    fshift = kDigitShift0;
    if (b.count != rem) {
      hist_level(1, kDigitShift0, fpfx, kDigitShift1, 0x7FFu);
      b = merge_find(1, std::integral_constant<int, kBins>(), rem);
      rem -= b.above;
      fpfx = (fpfx << 11) | b.bin;
      fshift = kDigitShift1;
      if (b.count != rem) {
        hist_level(2, kDigitShift1, fpfx, kDigitShift2, 0x1FFu);
        b = merge_find(2, std::integral_constant<int, 512>(), rem);
        rem -= b.above;
        fpfx = (fpfx << 9) | b.bin;
        fshift = kDigitShift2;
      }
    }
  }
  const uint32_t need = rem;

  // ---- count strict picks and ties of this CTA, exchange prefixes ----
  uint32_t na = 0, nb = 0, warp_ex = 0;
  if (staged) {
    uint32_t ca = 0, ct = 0;
    for (uint32_t i = wb + lane; i < we; i += 32) {
      const uint32_t s = mag_key(stage_val[i]) >> fshift;
      ca += s > fpfx;
      ct += s == fpfx;
    }
    // per-CTA counts <= my_pad <= stage_cap < 2^16: pack strict | ties
    const uint32_t wsum = __reduce_add_sync(kFull, (ca << 16) | ct);
    if (lane == 0) sh.tmp[warp] = wsum;
    __syncthreads();
    if (warp == 0) {
      const uint32_t x = lane < NW ? sh.tmp[lane] : 0u;
      const uint32_t incl = warp_incl_scan(x);
      if (lane < NW) sh.tmp[NW + lane] = incl - x;
      if (lane == NW - 1) sh.tmp[2 * NW] = incl;
    }
    __syncthreads();
    warp_ex = sh.tmp[NW + warp];
    const uint32_t tot = sh.tmp[2 * NW];
    na = tot >> 16;
    nb = tot & 0xFFFFu;
    __syncthreads();
  } else if (fast) {
    traverse([&](bool valid, uint32_t, float val) {
      const uint32_t s = mag_key(val) >> fshift;
      na += valid && s > fpfx;
      nb += valid && s == fpfx;
    });
    na = block_sum<NT>(na, sh.tmp);
    nb = block_sum<NT>(nb, sh.tmp);
  } else {
    for (uint32_t base = ea; base < eb; base += NT * kExhV) {
      float v[kExhV];
      exh_load(base, v);
#pragma unroll
      for (uint32_t j = 0; j < kExhV; ++j) {
        const bool valid = base + tid * kExhV + j < eb;
        const uint32_t s = mag_key(v[j]) >> fshift;
        na += valid && s > fpfx;
        nb += valid && s == fpfx;
      }
    }
    na = block_sum<NT>(na, sh.tmp);
    nb = block_sum<NT>(nb, sh.tmp);
  }
  if (tid == 0) {
    sh.xch[2] = na;
    sh.xch[3] = nb;
  }
  C::sync();
  uint32_t a_run = 0, b_run = 0;
  for (uint32_t q = 0; q < rank; ++q) {
    const uint32_t* x = C::remote(sh.xch, q);
    a_run += x[2];
    b_run += x[3];
  }
  C::arrive();  // the last read of a peer's shared memory (see C::wait below)

  // ---- ordered emission: pos = strict_before + min(need, ties_before) ----
  const uint64_t ob = (uint64_t)p * dp.K + ld.koff;
  auto emit = [&](uint32_t pos, uint32_t idx, float val, bool zero_residual) {
    if (pos < ld.k) {
      out_idx[ob + pos] = idx;
      out_val[ob + pos] = val;
      if (zero_residual) r[idx] = 0.0f;
    } else {
      atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
    }
  };
  // values-only staging: one bit per staged entry marks the picks for the
  // index pass (in this CTA's histogram, free once the search is done: no
  // peer reads it)
  uint32_t* const picked = hist;
  static_assert(kSelectStageMaxValues <= kBins * 32, "one bit per staged entry fits the histogram");
  if constexpr (VO) {
    if (staged) {
      for (uint32_t w = tid; w < (my_pad + 31) / 32; w += NT) picked[w] = 0u;
      __syncthreads();
    }
  }
  bool restage_timeout = false;
  if (staged) {
    // warp rounds of 32 consecutive positions: ballots give each lane its
    // strict and tie ranks, so the pick-list stores are coalesced and no
    // block barrier is needed; the emitted index (VO: the pick's position)
    // replaces the staged value (0xFFFFFFFF marks "not emitted") for the
    // residual zeroing (VO: the index lookup) below
    uint32_t at = a_run + (warp_ex >> 16), bt = b_run + (warp_ex & 0xFFFFu);
    for (uint32_t b0 = wb; b0 < we; b0 += 32) {
      const uint32_t i = b0 + lane;
      const bool valid = i < we;
      const float val = valid ? stage_val[i] : 0.f;
      const uint32_t s = mag_key(val) >> fshift;
      const bool st = valid && s > fpfx, ti = valid && s == fpfx;
      const unsigned mst = __ballot_sync(kFull, st), mti = __ballot_sync(kFull, ti);
      const uint32_t sb = at + __popc(mst & lanes_below), tb_ = bt + __popc(mti & lanes_below);
      uint32_t mark = 0xFFFFFFFFu;
      if (st || (ti && tb_ < need)) {
        const uint32_t pos = st ? sb + min(need, tb_) : sb + tb_;
        if constexpr (VO) {
          if (pos < ld.k) {
            out_val[ob + pos] = val;
            mark = pos;
            atomicOr(&picked[i >> 5], 1u << (i & 31));
          } else {
            atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
          }
        } else {
          const uint32_t idx = stage_idx[i];
          emit(pos, idx, val, false);
          mark = idx;
        }
      }
      if (valid) stage_val[i] = __uint_as_float(mark);
      at += __popc(mst);
      bt += __popc(mti);
    }
    if constexpr (VO) {
      // the picks' indices, tile by tile (the walks cross the warps' ranges)
      fence_proxy_async_shared();  // the marks above, before the copies below
      __syncthreads();
      const uint32_t nw = tb - ta;
      if (!ovf) {
        // every run came from the slots: copy the runs' indices over the
        // stage (the picks' positions follow from the bits), then write each
        // warp's picks in index order, coalesced, and zero their residuals
        if (tid == 0) mbar_arrive_expect_tx(&stage_bar, my_pad * 4u);
        __syncthreads();
        for (uint32_t q = tid; q < nw; q += NT) {
          const uint32_t n = sh.tpre[q + 1] - sh.tpre[q];
          if (n == 0) continue;
          const uint64_t slot = cbase + (uint64_t)(ta + q - ld.tile_begin) * cap;
          bulk_load(stage_val + sh.tpre[q], cand_idx + slot, n * 4u, &stage_bar);
        }
        const bool ok = mbar_wait_bounded(&stage_bar, 1, dp.index_spin);
        restage_timeout = __syncthreads_or(!ok);
        if (restage_timeout && tid == 0) atomicOr(dp.status + kStatusFlags, LAGS_FLAG_TIMEOUT);
        // picks before this warp's range: strict ones plus the first `need` ties
        uint32_t pos = a_run + (warp_ex >> 16) + min(need, b_run + (warp_ex & 0xFFFFu));
        for (uint32_t b0 = wb; b0 < we; b0 += 32) {
          const uint32_t i = b0 + lane;
          const bool pk = i < we && ((picked[i >> 5] >> (i & 31)) & 1u);
          const unsigned mp = __ballot_sync(kFull, pk);
          if (pk) {
            const uint32_t at_ = pos + __popc(mp & lanes_below);
            uint32_t x;
            if (!restage_timeout) {
              x = __float_as_uint(stage_val[i]);
            } else {
              // the copies did not complete: the slot from the tile prefix
              uint32_t lo_q = 0, hi_q = nw - 1;
              while (lo_q < hi_q) {
                const uint32_t mid = (lo_q + hi_q + 1) >> 1;
                if (sh.tpre[mid] <= i) lo_q = mid; else hi_q = mid - 1;
              }
              x = __ldg(cand_idx + cbase + (uint64_t)(ta + lo_q - ld.tile_begin) * cap +
                        (i - sh.tpre[lo_q]));
            }
            if (at_ < ld.k && x - ld.off < ld.d) {
              out_idx[ob + at_] = x;
              r[x] = 0.0f;
            } else {
              atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
            }
          }
          pos += __popc(mp);
        }
      } else {
      // tiles the bulk copies brought: the index of staged entry j of tile q
      // is in the tile's slot j
      // (eight entries at a time: their index loads in flight together)
      constexpr uint32_t B = 8;
      for (uint32_t q = tid; q < nw; q += NT) {
        const uint32_t n = __ldg(cnt + ta + q);
        if (n > cap) continue;
        const uint64_t slot = cbase + (uint64_t)(ta + q - ld.tile_begin) * cap;
        const uint32_t b = sh.tpre[q];
        for (uint32_t j0 = 0; j0 < n; j0 += B) {
          uint32_t m[B], x[B];
#pragma unroll
          for (uint32_t u = 0; u < B; ++u)
            m[u] = j0 + u < n ? __float_as_uint(stage_val[b + j0 + u]) : 0xFFFFFFFFu;
#pragma unroll
          for (uint32_t u = 0; u < B; ++u)
            x[u] = m[u] != 0xFFFFFFFFu ? __ldg(cand_idx + slot + j0 + u) : 0u;
#pragma unroll
          for (uint32_t u = 0; u < B; ++u) {
            if (m[u] == 0xFFFFFFFFu) continue;
            out_idx[ob + m[u]] = x[u];
            if (x[u] - ld.off < ld.d) r[x[u]] = 0.0f;  // an emitted index lies in the layer
            else atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
          }
        }
      }
      if (ovf) {
        // recompacted tiles: the tile's acc walked again in the recompaction's
        // order (each thread a contiguous run); its j-th entry with key >=
        // lo_key sits at stage tpre[q] + j.  Only these tiles' residuals are
        // written here, each after it is read.
        constexpr uint32_t PT = kTile / NT;
        for (uint32_t q = 0; q < nw; ++q) {
          const uint32_t n = __ldg(cnt + ta + q);  // block-uniform
          if (n <= cap) continue;
          const TileDesc tq = dp.tiles[ta + q];
          const uint32_t e0 = tq.start + tid * PT;
          const uint32_t mine = tid * PT < tq.len ? min(PT, tq.len - tid * PT) : 0u;
          uint32_t c = 0;
          for (uint32_t j = 0; j < mine; ++j) c += mag_key(r[e0 + j]) >= lo_key;
          uint32_t found;
          uint32_t rank_in = block_excl_scan<NT>(c, sh.tmp, &found);
          const uint32_t room = sh.tpre[q + 1] - sh.tpre[q];
          for (uint32_t j = 0; j < mine; ++j) {
            const float x = r[e0 + j];
            if (mag_key(x) >= lo_key) {
              if (rank_in < room) {
                const uint32_t m = __float_as_uint(stage_val[sh.tpre[q] + rank_in]);
                if (m != 0xFFFFFFFFu) {
                  out_idx[ob + m] = e0 + j;
                  r[e0 + j] = 0.0f;
                }
              }
              ++rank_in;
            }
          }
        }
      }
      }  // (overflowed share)
    } else {
      __syncwarp();
      for (uint32_t i = wb + lane; i < we; i += 32) {
        const uint32_t x = __float_as_uint(stage_val[i]);
        if (x == 0xFFFFFFFFu) continue;
        if (x - ld.off < ld.d) r[x] = 0.0f;  // an emitted index lies in the layer
        else atomicOr(dp.status + kStatusFlags, LAGS_FLAG_INTERNAL);
      }
    }
  } else if (fast) {
    traverse([&](bool valid, uint32_t idx, float val) {
      const uint32_t s = mag_key(val) >> fshift;
      const bool st = valid && s > fpfx;
      const bool ti = valid && s == fpfx;
      uint32_t tot;
      const uint32_t ex = block_excl_scan<NT>(((uint32_t)st << 16) | (uint32_t)ti, sh.tmp, &tot);
      const uint32_t at = a_run + (ex >> 16), bt = b_run + (ex & 0xFFFFu);
      if (st) emit(at + min(need, bt), idx, val, true);
      else if (ti && bt < need) emit(at + bt, idx, val, true);
      a_run += tot >> 16;
      b_run += tot & 0xFFFFu;
    });
  } else {
    // one block scan per round of NT * kExhV elements (< 2^16, so strict and
    // tie counts pack into one word); the next round's loads are issued
    // before this round's stores, which would otherwise hold them back
    float v[kExhV];
    exh_load(ea, v);
    for (uint32_t base = ea; base < eb; base += NT * kExhV) {
      float nv[kExhV];
      exh_load(base + NT * kExhV, nv);
      uint32_t cst = 0, cti = 0;
#pragma unroll
      for (uint32_t j = 0; j < kExhV; ++j) {
        const bool valid = base + tid * kExhV + j < eb;
        const uint32_t s = mag_key(v[j]) >> fshift;
        cst += valid && s > fpfx;
        cti += valid && s == fpfx;
      }
      uint32_t tot;
      const uint32_t ex = block_excl_scan<NT>((cst << 16) | cti, sh.tmp, &tot);
      uint32_t at = a_run + (ex >> 16), bt = b_run + (ex & 0xFFFFu);
#pragma unroll
      for (uint32_t j = 0; j < kExhV; ++j) {
        const uint32_t e = base + tid * kExhV + j;
        const uint32_t s = mag_key(v[j]) >> fshift;
        if (e < eb && s > fpfx) {
          emit(at + min(need, bt), e, v[j], true);
          ++at;
        } else if (e < eb && s == fpfx) {
          if (bt < need) emit(at + bt, e, v[j], true);
          ++bt;
        }
      }
      a_run += tot >> 16;
      b_run += tot & 0xFFFFu;
#pragma unroll
      for (uint32_t j = 0; j < kExhV; ++j) v[j] = nv[j];
    }
  }
  if (stage_timeout && tid == 0)  // give copies still in flight a bounded chance to land
    mbar_wait_bounded(&stage_bar, 0, kSelectSpinLimit);
  if (restage_timeout && tid == 0)
    mbar_wait_bounded(&stage_bar, 1, kSelectSpinLimit);
  C::wait();  // no CTA leaves while another may still read its shared memory
}

// Dynamic shared memory of a select launch staging `cap` candidates (values
// and indices, or values only).
inline size_t stage_smem_bytes(uint32_t cap, bool values_only = false) {
  return (size_t)cap * (values_only ? 4 : 8);
}

cudaError_t configure_select() {
  const int most = (int)stage_smem_bytes(kSelectStageMax);
  cudaError_t e = cudaFuncSetAttribute(k_select<1, kSelectThreadsSmall, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, most);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_select<kSelectCluster, kSelectThreads, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, most);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_select<kSelectClusterMid, kSelectThreads, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)stage_smem_bytes(kSelectStageMaxValues, true));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_select<kSelectClusterHuge, kSelectThreads, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, most);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_select<kSelectClusterHuge, kSelectThreads, false>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

namespace {
// Whether the current device can run one 16-CTA select cluster with `smem`
// bytes of dynamic shared memory per CTA (cached per device and size, under a
// lock: several host threads may launch on several devices).
bool huge_clusters_fit(size_t smem) {
  struct Fit {
    size_t smem;
    bool fit;
  };
  static std::mutex mu;
  static std::vector<Fit> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (const Fit& f : cache[dev])
    if (f.smem == smem) return f.fit;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSelectClusterHuge);
  cfg.blockDim = dim3(kSelectThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSelectClusterHuge;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(
      &clusters, k_select<kSelectClusterHuge, kSelectThreads, false>, &cfg);
  if (e != cudaSuccess) cudaGetLastError();  // clear; use 8-CTA clusters instead
  const bool fit = e == cudaSuccess && clusters > 0;
  cache[dev].push_back(Fit{smem, fit});
  return fit;
}
}  // namespace

cudaError_t launch_select(const DevPlan& dp, const WorkerPtrs& wp, uint32_t* out_idx,
                          float* out_val, cudaStream_t s) {
  if (dp.n_small) {
    cudaError_t e = launch_pdl(k_select<1, kSelectThreadsSmall, false>, dim3(dp.n_small, dp.P),
                               dim3(kSelectThreadsSmall), stage_smem_bytes(dp.stage_small), s, 1,
                               dp, wp, dp.sel_small, dp.stage_small, out_idx, out_val);
    if (e != cudaSuccess) return e;
  }
  if (dp.n_mid) {
    cudaError_t e = launch_pdl(k_select<kSelectClusterMid, kSelectThreads, true>,
                               dim3(dp.n_mid * kSelectClusterMid, dp.P), dim3(kSelectThreads),
                               stage_smem_bytes(dp.stage_mid, true), s, kSelectClusterMid, dp, wp,
                               dp.sel_mid, dp.stage_mid, out_idx, out_val);
    if (e != cudaSuccess) return e;
  }
  if (dp.n_large) {
    cudaError_t e = launch_pdl(k_select<kSelectCluster, kSelectThreads, false>,
                               dim3(dp.n_large * kSelectCluster, dp.P), dim3(kSelectThreads),
                               stage_smem_bytes(dp.stage_large), s, kSelectCluster, dp, wp,
                               dp.sel_large, dp.stage_large, out_idx, out_val);
    if (e != cudaSuccess) return e;
  }
  if (dp.n_huge) {
    const size_t smem = stage_smem_bytes(dp.stage_huge);
    if (huge_clusters_fit(smem))
      return launch_pdl(k_select<kSelectClusterHuge, kSelectThreads, false>,
                        dim3(dp.n_huge * kSelectClusterHuge, dp.P), dim3(kSelectThreads), smem, s,
                        kSelectClusterHuge, dp, wp, dp.sel_huge, dp.stage_huge, out_idx, out_val);
    // 8-CTA clusters with the same staging: shares that do not fit are read
    // from global memory on every pass (slower, same result)
    return launch_pdl(k_select<kSelectCluster, kSelectThreads, false>,
                      dim3(dp.n_huge * kSelectCluster, dp.P), dim3(kSelectThreads), smem, s,
                      kSelectCluster, dp, wp, dp.sel_huge, dp.stage_huge, out_idx, out_val);
  }
  return cudaSuccess;
}

}  // namespace lags
