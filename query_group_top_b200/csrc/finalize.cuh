// Exact top-K per proxy row from the scan's spill lists, and the exact
// fallback for rows whose sampled threshold missed.
//
// Method: the candidate set C = top-Kc of the proxy scores ("PIVOT explained",
// "How It Works": C = top-K(scores), K = 2 x top_k); for Reuse the members
// share the proxy's top-k ("Show Me The Code", pivot_reuse); the dense indexer
// keeps each query's own top-k.  Ties go to the lower key index; rows are
// written in ascending key order, padded with -1.
#pragma once

#include "ptx.cuh"
#include "scan.cuh"
#include "select.cuh"

namespace pivot {

struct FinalizeParams {
  int G, L, H, g, bound_kind;
  int K_sel;       // keys kept per row
  int cap;         // spill capacity per row
  int width;       // output row width: top_k for index rows; for candidate
                   // rows the row stride, cand_row_words(K_sel)
  int broadcast;   // 0: write the candidate row; 1: write the row to every member's output row
  const uint2* spill;
  const int4* cnt;   // per row: the four runs' entry counts (layout in ScanParams)
  int32_t* cand;   // [H*G][width] when broadcast == 0
  int32_t* out;    // [L][H][width] when broadcast == 1
  float* out_scores;  // [L][H][width] or null (broadcast == 1 only)
  int* fb_list;    // rows handed to the fallback kernel
  int* fb_count;
  int* status;
  // fallback only: the scan's operand, one of
  const float* proxy32;   // [G][H][d] fp32 proxies (PIVOT)
  const uint16_t* proxy16;  // [G][H][d] bf16 bits (dense: the queries)
  const uint16_t* keys;   // [L][H][d] bf16 bits
  int d;
  uint32_t* fb_scratch;   // [gridDim.x][L] order keys
};

constexpr int kFinNT = 512;
constexpr int kFbNT = 512;

// Copies the K selected key indices (staged in shared memory) to their
// destination: a candidate row, or every member's index row, coalesced, with
// -1 padding to `width`.
__device__ __forceinline__ void write_rows(const FinalizeParams& p, int h, int i, const int32_t* sel,
                                           const uint32_t* selk, int K) {
  if (!p.broadcast) {
    write_cand_row(p.cand + (static_cast<long long>(h) * p.G + i) * p.width, sel, K);
    return;
  }
  const int s = i * p.g, e = min(s + p.g, p.L);
  for (int pos = s; pos < e; ++pos) {
    int32_t* dst = p.out + (static_cast<long long>(pos) * p.H + h) * p.width;
    for (int t = threadIdx.x; t < p.width; t += blockDim.x) dst[t] = t < K ? sel[t] : -1;
    if (p.out_scores) {
      float* ds = p.out_scores + (static_cast<long long>(pos) * p.H + h) * p.width;
      for (int t = threadIdx.x; t < p.width; t += blockDim.x)
        ds[t] = t < K ? key_score(selk[t]) : __int_as_float(0x7fc00000);
    }
  }
}

__global__ void __launch_bounds__(kFinNT) finalize_kernel(FinalizeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ SelectSmem<kFinNT> sm;
  uint2* ent = reinterpret_cast<uint2*>(smem_raw);
  int32_t* sel = reinterpret_cast<int32_t*>(smem_raw + static_cast<size_t>(p.cap) * sizeof(uint2));
  uint32_t* selk = reinterpret_cast<uint32_t*>(sel + p.K_sel);

  const long long row_id = blockIdx.x;
  const int h = static_cast<int>(row_id / p.G), i = static_cast<int>(row_id % p.G);
  ScanParams sp{};
  sp.G = p.G; sp.L = p.L; sp.g = p.g; sp.bound_kind = p.bound_kind;
  const int bound = row_bound(sp, i);
  const int K = min(p.K_sel, bound);
  const int4 c4 = p.cnt[row_id];
  const int capH = p.cap / 2;
  const int n = c4.x + c4.y + c4.z + c4.w;
  // a spill region that overflowed, or too few survivors of a thresholded row
  if (c4.x + c4.y > capH || c4.z + c4.w > capH || (bound > capH && n < K)) {
    if (threadIdx.x == 0) {
      const int slot = atomicAdd(p.fb_count, 1);
      p.fb_list[slot] = static_cast<int>(row_id);
    }
    return;
  }
  // runs 0..3 cover ascending quarters of the keys; odd runs were stored
  // downward from the end of their region: copied in this order, the entries
  // are in ascending key-index order.  Every copy of the row is in flight at
  // once; then the scores become order keys.
  const uint2* src = p.spill + row_id * p.cap;
  const int o1 = c4.x, o2 = o1 + c4.y, o3 = o2 + c4.z;
  for (int e = threadIdx.x; e < n; e += kFinNT) {
    const int at = e < o1 ? e : (e < o2 ? capH - 1 - (e - o1) : (e < o3 ? capH + (e - o2) : p.cap - 1 - (e - o3)));
    cp_async_8(smem_u32(&ent[e]), src + at);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += kFinNT) ent[e].x = score_key(__uint_as_float(ent[e].x));
  const int nn = n;
  __syncthreads();
  if (!p.broadcast) {
    // candidate row: each selected index goes straight to its word of the
    // row (no staging, so the kernel needs only the entries' shared memory)
    int32_t* dst = p.cand + row_id * p.width;
    block_select_emit<kFinNT>(
        nn, K, [&](int e) { return ent[e].x; },
        [&](int slot, int e) { dst[slot] = static_cast<int32_t>(ent[e].y); }, sm);
    const int words = (K + 127) / 128 * 128;
    for (int t = K + static_cast<int>(threadIdx.x); t < words; t += kFinNT) dst[t] = -1;
    return;
  }
  block_select_emit<kFinNT>(
      nn, K, [&](int e) { return ent[e].x; },
      [&](int slot, int e) {
        sel[slot] = static_cast<int32_t>(ent[e].y);
        selk[slot] = ent[e].x;
      },
      sm);
  __syncthreads();
  write_rows(p, h, i, sel, selk, K);
}

// Exact path for rows the filter could not settle: recompute the row's scores
// over its whole prefix (CUDA cores, fp32 proxy times bf16 keys, fp32
// accumulation) and select from all of them.
__global__ void __launch_bounds__(kFbNT) fallback_kernel(FinalizeParams p) {
  __shared__ SelectSmem<kFbNT> sm;
  __shared__ float pv[128];
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  int32_t* sel = reinterpret_cast<int32_t*>(smem_raw);
  uint32_t* selk = reinterpret_cast<uint32_t*>(sel + p.K_sel);
  uint32_t* sc = p.fb_scratch + static_cast<long long>(blockIdx.x) * p.L;
  const int total = *p.fb_count;
  if (blockIdx.x == 0 && threadIdx.x == 0 && total > 0) atomicOr(p.status, kStFallback);
  ScanParams sp{};
  sp.G = p.G; sp.L = p.L; sp.g = p.g; sp.bound_kind = p.bound_kind;
  for (int w = blockIdx.x; w < total; w += gridDim.x) {
    const int row_id = p.fb_list[w];
    const int h = row_id / p.G, i = row_id % p.G;
    const int bound = row_bound(sp, i);
    const int K = min(p.K_sel, bound);
    __syncthreads();
    for (int c = threadIdx.x; c < p.d; c += kFbNT) {
      const long long o = (static_cast<long long>(i) * p.H + h) * p.d + c;
      pv[c] = p.proxy32 ? p.proxy32[o] : __uint_as_float(static_cast<uint32_t>(p.proxy16[o]) << 16);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < bound; j += kFbNT) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.keys + (static_cast<long long>(j) * p.H + h) * p.d);
      float acc = 0.f;
      for (int c8 = 0; c8 < p.d / 8; ++c8) {
        const uint4 u = kr[c8];
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc = fmaf(pv[c8 * 8 + 2 * t], __uint_as_float(w4[t] << 16), acc);
          acc = fmaf(pv[c8 * 8 + 2 * t + 1], __uint_as_float(w4[t] & 0xFFFF0000u), acc);
        }
      }
      sc[j] = score_key(acc);
    }
    __syncthreads();
    block_select_emit<kFbNT>(
        bound, K, [&](int e) { return sc[e]; },
        [&](int slot, int e) {
          sel[slot] = e;
          selk[slot] = sc[e];
        },
        sm);
    __syncthreads();
    write_rows(p, h, i, sel, selk, K);
  }
}

}  // namespace pivot
