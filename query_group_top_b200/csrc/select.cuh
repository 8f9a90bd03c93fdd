// Exact block-wide top-K selection on 32-bit order keys.
//
// The K entries with the largest keys are kept; among equal keys the earlier
// entry wins (entries are always presented in ascending key-index order, so
// "earlier" is "lower index", the tie rule of the method).  The threshold key
// T (the K-th largest) is found by a 4-pass MSB-first radix select with
// 256-bin shared histograms; the selected entries are then emitted in entry
// order with their output slot, so every output row comes out ascending.
#pragma once

#include "ptx.cuh"

namespace pivot {

template <int NT>
struct SelectSmem {
  int hist[256];
  int warp_tot[NT / 32];
  int bstar;
  int above;
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

// Finds, among entries e < n whose key matches (key & mask) == prefix, the
// digit b at `shift` such that the number of matching entries with digit > b
// is < rank <= that number plus the count of digit b.  Returns b; *above
// receives the count with digit > b.
template <int NT, class Fetch>
__device__ __forceinline__ int radix_digit(int n, Fetch fetch, uint32_t prefix, uint32_t mask, int shift,
                                           int rank, SelectSmem<NT>& sm, int* above) {
  const int lane = threadIdx.x & 31;
  for (int b = threadIdx.x; b < 256; b += NT) sm.hist[b] = 0;
  if (threadIdx.x == 0) {
    sm.bstar = 0;
    sm.above = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += NT) {
    const int e = base + threadIdx.x;
    int digit = 256 + lane;  // unique sentinel: matches nobody
    if (e < n) {
      const uint32_t key = fetch(e);
      if ((key & mask) == prefix) digit = (key >> shift) & 255;
    }
    const unsigned same = __match_any_sync(0xffffffffu, digit);
    if (digit < 256 && lane == __ffs(same) - 1) atomicAdd(&sm.hist[digit], __popc(same));
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // lane l owns bins [8*(31-l), 8*(31-l)+8): lane 0 holds the top bins.
    const int hi_bin = 255 - 8 * lane;
    int c[8];
    int s = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = sm.hist[hi_bin - t];
      s += c[t];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - s;
    const unsigned hit = __ballot_sync(0xffffffffu, excl < rank && rank <= incl);
    if (hit && lane == __ffs(hit) - 1) {
      int cum = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (cum + c[t] >= rank) {
          sm.bstar = hi_bin - t;
          sm.above = cum;
          break;
        }
        cum += c[t];
      }
    }
  }
  __syncthreads();
  const int b = sm.bstar;
  *above = sm.above;
  __syncthreads();
  return b;
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
  uint32_t prefix = 0, mask = 0;
  int rank = K;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    int above;
    const int b = radix_digit<NT>(n, fetch, prefix, mask, shift, rank, sm, &above);
    prefix |= static_cast<uint32_t>(b) << shift;
    mask |= 0xFFu << shift;
    rank -= above;
  }
  const uint32_t T = prefix;   // K-th largest key
  const int need_eq = rank;    // how many entries equal to T are taken (earliest first)

  // Each thread owns a contiguous run of entries so that entry order is kept.
  const int per = (n + NT - 1) / NT;
  const int e0 = min(n, static_cast<int>(threadIdx.x) * per);
  const int e1 = min(n, e0 + per);
  int n_eq = 0;
  for (int e = e0; e < e1; ++e) n_eq += (fetch(e) == T);
  const int eq_before = block_exclusive_scan<NT>(n_eq, sm.warp_tot, nullptr);
  int n_sel = 0, seen = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = fetch(e);
    if (key > T) {
      ++n_sel;
    } else if (key == T) {
      n_sel += (eq_before + seen < need_eq);
      ++seen;
    }
  }
  const int sel_before = block_exclusive_scan<NT>(n_sel, sm.warp_tot, nullptr);
  int slot = sel_before;
  seen = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = fetch(e);
    bool take = false;
    if (key > T) {
      take = true;
    } else if (key == T) {
      take = (eq_before + seen < need_eq);
      ++seen;
    }
    if (take) emit(slot++, e);
  }
}

}  // namespace pivot
