// Exact block-wide top-K selection on 32-bit order keys.
//
// The K entries with the largest keys are kept; among equal keys the earlier
// entry wins (entries are always presented in ascending key-index order, so
// "earlier" is "lower index", the tie rule of the method).  The rule is found
// by an MSB-first radix select that starts at the highest key bit that varies
// among the entries (bits above it are a common prefix) and consumes up to 11
// bits per pass with a 2048-bin shared histogram, stopping as soon as the
// boundary bin is taken whole.  The selected entries are emitted in entry order
// with their output slot, so every output row comes out ascending.
#pragma once

#include "ptx.cuh"

namespace pivot {

template <int NT>
struct SelectSmem {
  int hist[2048];
  int warp_tot[NT / 32];
  unsigned red[NT / 32];
  int bstar, above, cntb;
};

// Exclusive block-wide prefix sum of one int per thread (all NT threads call).
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < NT / 32) ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < NT / 32) warp_tot[lane] = wi - w;  // exclusive warp offsets
    int tot = __shfl_sync(0xffffffffu, wi, NT / 32 - 1);
    if (lane == 0 && total) *total = tot;
  }
  __syncthreads();
  return warp_tot[warp] + incl - x;
}

// Block-wide OR of one value per thread.
template <int NT>
__device__ __forceinline__ unsigned block_or(unsigned x, unsigned* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x |= __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  unsigned r = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) r |= red[w];
  return r;
}

// Selects the top K of n entries (K <= n) and calls emit(slot, e) for each
// selected entry e, slot = its rank in entry order (0..K-1).
template <int NT, class Fetch, class Emit>
__device__ void block_select_emit(int n, int K, Fetch fetch, Emit emit, SelectSmem<NT>& sm) {
  if (K <= 0) return;
  if (K >= n) {
    for (int e = threadIdx.x; e < n; e += NT) emit(e, e);
    return;
  }
  // bits that vary among the keys
  const uint32_t key0 = fetch(0);
  unsigned diff = 0;
  for (int e = threadIdx.x; e < n; e += NT) diff |= fetch(e) ^ key0;
  diff = block_or<NT>(diff, sm.red);
  int sh = 32 - __clz(diff);                     // bits [sh, 32) are common to all keys
  uint32_t tmask = sh >= 32 ? 0u : (0xFFFFFFFFu << sh);
  uint32_t thr = key0 & tmask;
  int rank = K;                                  // how many keys at or above thr to take
  bool whole = false;
  bool ties = (sh == 0);                         // all keys equal: first K in order
#pragma unroll 1
  while (sh > 0) {
    const int width = sh >= 11 ? 11 : sh;
    sh -= width;
    const int nbn = 1 << width;
    for (int b = threadIdx.x; b < nbn; b += NT) sm.hist[b] = 0;
    if (threadIdx.x == 0) {
      sm.bstar = 0;
      sm.above = 0;
      sm.cntb = 0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += NT) {
      const uint32_t key = fetch(e);
      if ((key & tmask) == thr) red_shared_add(smem_u32(&sm.hist[(key >> sh) & (nbn - 1)]), 1u);
    }
    __syncthreads();
    // thread t owns bins [top - per + 1, top], scanned from the top
    const int per = (nbn + NT - 1) / NT;
    const int top = nbn - 1 - per * static_cast<int>(threadIdx.x);
    int s = 0;
    for (int t = 0; t < per; ++t)
      if (top - t >= 0) s += sm.hist[top - t];
    const int excl = block_exclusive_scan<NT>(s, sm.warp_tot, nullptr);
    if (excl < rank && rank <= excl + s) {
      int cum = excl;
      for (int t = 0; t < per; ++t) {
        const int cb = sm.hist[top - t];
        if (cum + cb >= rank) {
          sm.bstar = top - t;
          sm.above = cum;
          sm.cntb = cb;
          break;
        }
        cum += cb;
      }
    }
    __syncthreads();
    thr |= static_cast<uint32_t>(sm.bstar) << sh;
    tmask |= static_cast<uint32_t>(nbn - 1) << sh;
    rank -= sm.above;
    whole = (sm.cntb == rank);
    __syncthreads();
    if (whole) break;          // every key of the boundary bin is taken
    if (sh == 0) ties = true;  // equal keys, only `rank` of them are taken
  }

  // Each thread owns a contiguous run of entries so that entry order is kept.
  const int per = (n + NT - 1) / NT;
  const int e0 = min(n, static_cast<int>(threadIdx.x) * per);
  const int e1 = min(n, e0 + per);
  int eq_before = 0;
  if (ties) {
    int n_eq = 0;
    for (int e = e0; e < e1; ++e) n_eq += (fetch(e) == thr);
    eq_before = block_exclusive_scan<NT>(n_eq, sm.warp_tot, nullptr);
  }
  auto take = [&](uint32_t key, int& seen) -> bool {
    if (!ties) return (key & tmask) >= thr;
    if (key > thr) return true;
    if (key == thr) return (eq_before + seen++) < rank;
    return false;
  };
  int n_sel = 0, seen = 0;
  for (int e = e0; e < e1; ++e) n_sel += take(fetch(e), seen);
  int slot = block_exclusive_scan<NT>(n_sel, sm.warp_tot, nullptr);
  seen = 0;
  for (int e = e0; e < e1; ++e)
    if (take(fetch(e), seen)) emit(slot++, e);
}

}  // namespace pivot
