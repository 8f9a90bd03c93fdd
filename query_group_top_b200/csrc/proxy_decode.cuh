// Proxy build (prefill and decode) and the decode-side scan and select.
//
// Proxy: "PIVOT explained", "How It Works": proxy_q = mean(group); the mean is
// accumulated in fp64 in member order, divided by the member count and
// rounded to fp32: the fp32 mean is the scan's operand.  A partial last group
// averages over its actual members.  For the tensor-core scan the fp32 mean is
// split exactly into three bf16 terms, p = hi + mid + lo: hi = bf16(p), mid =
// bf16(p - hi), lo = p - hi - mid.  Each difference is exact in fp32 (the
// operands lie within a factor of two of each other), p - hi carries at most
// 16 significant bits and p - hi - mid at most 8, so lo is a bf16 value and
// the three terms sum to p exactly (for |p| >= 2^-110 or p = 0, where lo is
// not a bf16 subnormal that loses bits).  Three MMAs over the same key tile
// then accumulate p . k with only fp32 accumulation error.  The variant
// flag rounds the fp32 mean to bf16 and scans with that value alone.
//
// Decode (paper abstract: in decode a group is "the queries decoded together
// in one multi-token prediction step"): one group per sequence, members at
// positions n_b .. n_b+g-1 of a packed key cache.  With a single proxy row per
// (sequence, head) the scan is a matrix-vector product bound by HBM: each warp
// streams 16-byte slices of consecutive key rows, multiplies them by the fp32
// proxy, reduces each row's dot product with shuffles and writes one 32-bit
// order key per key (4 bytes per 256 key bytes read).  An exact block select
// then keeps the top-K per (sequence, head).
#pragma once

#include <cuda_bf16.h>

#include "decode_cache.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

// Proxy of unit u (u < G), head h: P32[u][h][:] fp32 and, when P3 is not
// null, its three bf16 terms P3[t][u][h][:] (t = 0 hi, 1 mid, 2 lo).
// Prefill: members are positions u*g .. min(u*g+g, L)-1 of q [L][H][d].
// Decode (decode != 0): members are rows u*g .. u*g+g-1 of q [B*g][H][d].
// bf16_proxy != 0: the proxy is the fp32 mean rounded to bf16 (P32 holds that
// value, hi is it, mid and lo are zero).
__global__ void proxy_kernel(const uint16_t* __restrict__ q, float* __restrict__ P32, uint16_t* __restrict__ P3,
                             int G, int H, int d, int g, int L, int decode, int bf16_proxy) {
  const long long total = static_cast<long long>(G) * H * (d / 8);
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const int c8 = static_cast<int>(t % (d / 8));
  const long long uh = t / (d / 8);
  const int h = static_cast<int>(uh % H);
  const int u = static_cast<int>(uh / H);
  const long long row0 = static_cast<long long>(u) * g;
  const int n = decode ? g : min(u * g + g, L) - u * g;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int m = 0; m < n; ++m) {
    const uint4 v = *reinterpret_cast<const uint4*>(q + ((row0 + m) * H + h) * d + c8 * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[2 * k] += static_cast<double>(__uint_as_float(w[k] << 16));
      acc[2 * k + 1] += static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u));
    }
  }
  float pm[8];
  uint32_t th[8], tm[8], tl[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float p = __double2float_rn(__ddiv_rn(acc[k], static_cast<double>(n)));
    if (bf16_proxy) p = __bfloat162float(__float2bfloat16_rn(p));
    pm[k] = p;
    const __nv_bfloat16 hi = __float2bfloat16_rn(p);
    const float r1 = __fsub_rn(p, __bfloat162float(hi));      // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = __fsub_rn(r1, __bfloat162float(mid));    // exact, a bf16 value
    th[k] = __bfloat16_as_ushort(hi);
    tm[k] = __bfloat16_as_ushort(mid);
    tl[k] = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
  }
  const long long o = (static_cast<long long>(u) * H + h) * d + c8 * 8;
  reinterpret_cast<float4*>(P32 + o)[0] = make_float4(pm[0], pm[1], pm[2], pm[3]);
  reinterpret_cast<float4*>(P32 + o)[1] = make_float4(pm[4], pm[5], pm[6], pm[7]);
  if (P3) {
    const long long term = static_cast<long long>(G) * H * d;
    *reinterpret_cast<uint4*>(P3 + o) =
        make_uint4(th[0] | th[1] << 16, th[2] | th[3] << 16, th[4] | th[5] << 16, th[6] | th[7] << 16);
    *reinterpret_cast<uint4*>(P3 + term + o) =
        make_uint4(tm[0] | tm[1] << 16, tm[2] | tm[3] << 16, tm[4] | tm[5] << 16, tm[6] | tm[7] << 16);
    *reinterpret_cast<uint4*>(P3 + 2 * term + o) =
        make_uint4(tl[0] | tl[1] << 16, tl[2] | tl[3] << 16, tl[4] | tl[5] << 16, tl[6] | tl[7] << 16);
  }
}

// The listing's per-member Refine scans each member's own prefix with its
// group's proxy ("Show Me The Code", pivot_refine: k[:pos] per member).  The
// scan then treats positions as its rows, so every position gets a copy of
// its group's proxy: P32e [L][H][d] fp32 and the bf16 terms P3e [3][L][H][d]
// from P32 [G][H][d] and P3 [3][G][H][d].  One thread per (position, head,
// 8 channels): 32-byte and three 16-byte copies.
__global__ void proxy_expand_kernel(const float* __restrict__ P32, const uint16_t* __restrict__ P3,
                                    float* __restrict__ P32e, uint16_t* __restrict__ P3e, int G, int L, int H,
                                    int d, int g) {
  const long long total = static_cast<long long>(L) * H * (d / 8);
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const int c8 = static_cast<int>(t % (d / 8));
  const long long ph = t / (d / 8);
  const int h = static_cast<int>(ph % H);
  const long long pos = ph / H;
  const long long src = ((pos / g) * H + h) * d + c8 * 8;
  const long long dst = (pos * H + h) * d + c8 * 8;
  reinterpret_cast<float4*>(P32e + dst)[0] = reinterpret_cast<const float4*>(P32 + src)[0];
  reinterpret_cast<float4*>(P32e + dst)[1] = reinterpret_cast<const float4*>(P32 + src)[1];
  const long long tg = static_cast<long long>(G) * H * d, te = static_cast<long long>(L) * H * d;
#pragma unroll
  for (int term = 0; term < 3; ++term)
    *reinterpret_cast<uint4*>(P3e + term * te + dst) = *reinterpret_cast<const uint4*>(P3 + term * tg + src);
}

struct DecodeParams {
  const uint16_t* kcache;   // packed [rows][H][d] or paged [pages][page_size][H][d]
  const float* P;           // [B][H][d] fp32 proxies
  CacheIndex ci;            // where each sequence's keys live
  uint32_t* scores;         // [H*B][max_seqlen] order keys
  int32_t* cand;            // [H][B][cand_row_words(K_sel)] candidate rows (Refine)
  int32_t* out;             // [B][g][H][width] (Reuse)
  float* out_scores;        // [B][g][H][width] or null (Reuse)
  int B, H, d, g;
  int mode;                 // 0 Refine (scan j < n_b+g-1, keep Kc), 1 Reuse (scan j < n_b, keep top_k)
  int K_sel, width, max_seqlen;
  int* status;
};

constexpr int kDecChunk = 2048;   // keys per scan CTA
constexpr int kDecNT = 256;

__device__ __forceinline__ bool decode_unit(const DecodeParams& p, int b, int& n_b, int& bound) {
  const int len = p.ci.len(b);
  n_b = len - p.g;
  bound = p.mode == 0 ? n_b + p.g - 1 : n_b;
  return len <= p.max_seqlen && n_b >= 0;
}

// PAGED selects the cache layout at compile time, so the packed layout's
// loop carries no page lookups.
template <int D, bool PAGED>
__global__ void __launch_bounds__(kDecNT) decode_scan_kernel(DecodeParams p) {
  constexpr int LPK = D / 8;          // lanes per key row (16 bytes each)
  constexpr int KPW = 32 / LPK;       // key rows per warp step
  constexpr int NW = kDecNT / 32;
  const int b = blockIdx.z, h = blockIdx.y;
  int n_b, bound;
  if (!decode_unit(p, b, n_b, bound)) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) atomicOr(p.status, kStBadLen);
    return;
  }
  const int j_begin = blockIdx.x * kDecChunk;
  if (j_begin >= bound) return;
  const int j_end = min(bound, j_begin + kDecChunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPK, part = lane % LPK;
  float pf[8];
  {
    const float4* pp = reinterpret_cast<const float4*>(p.P + (static_cast<long long>(b) * p.H + h) * D + part * 8);
    const float4 a = pp[0], c = pp[1];
    pf[0] = a.x; pf[1] = a.y; pf[2] = a.z; pf[3] = a.w;
    pf[4] = c.x; pf[5] = c.y; pf[6] = c.z; pf[7] = c.w;
  }
  // packed: rows from the sequence's first cache row; paged: rows from the
  // cache start, found through the block table
  const long long r0 = PAGED ? 0 : static_cast<long long>(p.ci.cu[b]);
  const uint16_t* kb = p.kcache + (r0 * p.H + h) * D + part * 8;
  const long long kstride = static_cast<long long>(p.H) * D;
  uint32_t* srow = p.scores + (static_cast<long long>(h) * p.B + b) * p.max_seqlen;
  constexpr int UNROLL = 4;
  for (int base = j_begin + warp * KPW; base < j_end; base += NW * KPW * UNROLL) {
    uint4 kv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int j = base + u * NW * KPW + sub;
      if constexpr (PAGED)
        kv[u] = (j < j_end) ? __ldg(reinterpret_cast<const uint4*>(kb + p.ci.row(b, 0, j) * kstride))
                            : make_uint4(0, 0, 0, 0);
      else
        kv[u] = (j < j_end) ? __ldg(reinterpret_cast<const uint4*>(kb + j * kstride)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const uint32_t w[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc = fmaf(pf[2 * k], __uint_as_float(w[k] << 16), acc);
        acc = fmaf(pf[2 * k + 1], __uint_as_float(w[k] & 0xFFFF0000u), acc);
      }
#pragma unroll
      for (int o = LPK / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int j = base + u * NW * KPW + sub;
      if (part == 0 && j < j_end) srow[j] = score_key(acc);
    }
  }
}

constexpr int kDecSelNT = 1024;

// Exact top-K per (sequence, head) over the materialised order keys.
__global__ void __launch_bounds__(kDecSelNT) decode_select_kernel(DecodeParams p) {
  __shared__ SelectSmem<kDecSelNT> sm;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  int32_t* sel = reinterpret_cast<int32_t*>(smem_raw);
  uint32_t* selk = reinterpret_cast<uint32_t*>(sel + p.K_sel);
  const int h = blockIdx.x / p.B, b = blockIdx.x % p.B;
  int n_b, bound;
  if (!decode_unit(p, b, n_b, bound)) {
    // skipped sequence (reported by the scan): Reuse rows are empty; the
    // refine kernel gives Refine members empty rows without reading a
    // candidate row
    if (p.mode != 0) {
      for (int m = 0; m < p.g; ++m) {
        const long long o = ((static_cast<long long>(b) * p.g + m) * p.H + h) * p.width;
        for (int t = threadIdx.x; t < p.width; t += kDecSelNT) {
          p.out[o + t] = -1;
          if (p.out_scores) p.out_scores[o + t] = __int_as_float(0x7fc00000);
        }
      }
    }
    return;
  }
  const int K = min(p.K_sel, bound);
  const uint32_t* srow = p.scores + (static_cast<long long>(h) * p.B + b) * p.max_seqlen;
  block_select_emit<kDecSelNT>(
      bound, K, [&](int e) { return srow[e]; },
      [&](int slot, int e) {
        sel[slot] = e;
        selk[slot] = srow[e];
      },
      sm);
  __syncthreads();
  if (p.mode == 0) {
    write_cand_row(p.cand + (static_cast<long long>(h) * p.B + b) * cand_row_words(p.K_sel), sel, K);
  } else {
    for (int m = 0; m < p.g; ++m) {
      int32_t* dst = p.out + ((static_cast<long long>(b) * p.g + m) * p.H + h) * p.width;
      for (int t = threadIdx.x; t < p.width; t += kDecSelNT) dst[t] = t < K ? sel[t] : -1;
      if (p.out_scores) {
        float* ds = p.out_scores + ((static_cast<long long>(b) * p.g + m) * p.H + h) * p.width;
        for (int t = threadIdx.x; t < p.width; t += kDecSelNT)
          ds[t] = t < K ? key_score(selk[t]) : __int_as_float(0x7fc00000);
      }
    }
  }
}

}  // namespace pivot
