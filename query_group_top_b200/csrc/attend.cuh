// The sparse attention that consumes the index rows ("PIVOT explained",
// "Show Me The Code": the demo after pivot_refine computes, per position and
// head, softmax(q . k[sel] * d^-1/2) @ v[sel] over the selected indices).
// For query row r, head h and the valid entries J of its index row (>= 0;
// -1 is padding):
//     s_j = (q . k_j) * d^-1/2,  out = sum_j softmax(s)_j v_j   (fp32)
// and a row without a valid index (position 0) gets zeros, as the demo
// leaves out[0].
//
// Memory-bound gather: every selected key and value row is read once (2 *
// top_k * d * 2 bytes per query head).  One 128-thread CTA per (row, head);
// a key row is d/8 lanes wide (16 bytes each), so a warp takes 32/(d/8) keys
// per step and the CTA runs 4 * 32/(d/8) independent key streams, each with
// an online softmax (running max, sum and accumulator over its slice of
// channels), four keys at a time so that their loads are in flight
// together; the streams are merged by shuffles, then across warps in shared
// memory.
#pragma once

#include "ptx.cuh"

namespace pivot {

struct AttendParams {
  const uint16_t* q;     // [R][H][d] bf16
  const uint16_t* k;     // prefill [R][H][d]; decode packed cache [rows][H][d]
  const uint16_t* v;     // same layout as k
  const int32_t* idx;    // [R][H][top_k]
  const int32_t* cu;     // decode: [B+1] cache row offsets (row r is member r % g of sequence r / g); null: prefill
  float* out;            // [R][H][d]
  int R, H, g, top_k;
  float scale;           // d^-1/2
};

constexpr int kAttNT = 128;

// Merges softmax state (m2, l2, a2) into (m, l, a); m = -inf means empty.
__device__ __forceinline__ void attend_merge(float& m, float& l, float (&a)[8], float m2, float l2,
                                             const float (&a2)[8]) {
  const float mn = fmaxf(m, m2);
  if (mn == -__int_as_float(0x7f800000)) return;   // both empty
  const float c1 = (m == mn) ? 1.f : __expf(m - mn);
  const float c2 = (m2 == mn) ? 1.f : __expf(m2 - mn);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int c = 0; c < 8; ++c) a[c] = a[c] * c1 + a2[c] * c2;
  m = mn;
}

template <int D>
__global__ void __launch_bounds__(kAttNT) sparse_attention_kernel(AttendParams p) {
  constexpr int LPK = D / 8;          // lanes per key row
  constexpr int KPW = 32 / LPK;       // keys per warp step
  constexpr int NW = kAttNT / 32;
  constexpr int STREAMS = NW * KPW;
  constexpr int U = 4;                // keys per stream per step
  const float kNegInf = -__int_as_float(0x7f800000);
  __shared__ float sm_m[NW][LPK], sm_l[NW][LPK], sm_a[NW][LPK][8];

  const long long rh = blockIdx.x;
  const int r = static_cast<int>(rh / p.H), h = static_cast<int>(rh % p.H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPK, part = lane % LPK;

  float qf[8];
  {
    const uint4 u = *reinterpret_cast<const uint4*>(p.q + rh * D + part * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      qf[2 * c] = __uint_as_float(w[c] << 16) * p.scale;
      qf[2 * c + 1] = __uint_as_float(w[c] & 0xFFFF0000u) * p.scale;
    }
  }
  const long long base = p.cu ? static_cast<long long>(p.cu[r / p.g]) : 0;
  const long long rstride = static_cast<long long>(p.H) * D;
  const uint16_t* kb = p.k + (base * p.H + h) * D + part * 8;
  const uint16_t* vb = p.v + (base * p.H + h) * D + part * 8;
  const int32_t* row = p.idx + rh * p.top_k;

  float m = kNegInf, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;

  // the trip count follows the warp's first stream, so that every lane of a
  // warp runs the same iterations (the key reductions are warp shuffles);
  // entries past top_k read as empty
  for (int tw = warp * KPW; tw < p.top_k; tw += STREAMS * U) {
    const int t0 = tw + sub;
    int j[U];
    uint4 kv[U], vv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u * STREAMS;
      j[u] = t < p.top_k ? __ldg(row + t) : -1;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      kv[u] = j[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(kb + j[u] * rstride)) : make_uint4(0, 0, 0, 0);
      vv[u] = j[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(vb + j[u] * rstride)) : make_uint4(0, 0, 0, 0);
    }
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      float x = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        x = fmaf(qf[2 * c], __uint_as_float(w[c] << 16), x);
        x = fmaf(qf[2 * c + 1], __uint_as_float(w[c] & 0xFFFF0000u), x);
      }
#pragma unroll
      for (int o = LPK / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      s[u] = j[u] >= 0 ? x : kNegInf;
    }
    float mn = m;
#pragma unroll
    for (int u = 0; u < U; ++u) mn = fmaxf(mn, s[u]);
    if (mn == kNegInf) continue;   // nothing valid in this stream yet (uniform per key group)
    const float cs = (m == mn) ? 1.f : __expf(m - mn);
    l *= cs;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= cs;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float w8 = j[u] >= 0 ? __expf(s[u] - mn) : 0.f;
      l += w8;
      const uint32_t w[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[2 * c] = fmaf(w8, __uint_as_float(w[c] << 16), acc[2 * c]);
        acc[2 * c + 1] = fmaf(w8, __uint_as_float(w[c] & 0xFFFF0000u), acc[2 * c + 1]);
      }
    }
    m = mn;
  }

  // merge the warp's key streams (lanes part, part + LPK, ...)
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    float a2[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) a2[c] = __shfl_xor_sync(0xffffffffu, acc[c], o);
    attend_merge(m, l, acc, m2, l2, a2);
  }
  if (sub == 0) {
    sm_m[warp][part] = m;
    sm_l[warp][part] = l;
#pragma unroll
    for (int c = 0; c < 8; ++c) sm_a[warp][part][c] = acc[c];
  }
  __syncthreads();
  if (warp == 0 && sub == 0) {
#pragma unroll
    for (int w2 = 1; w2 < NW; ++w2) {
      float a2[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) a2[c] = sm_a[w2][part][c];
      attend_merge(m, l, acc, sm_m[w2][part], sm_l[w2][part], a2);
    }
    float* o = p.out + rh * D + part * 8;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    reinterpret_cast<float4*>(o)[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    reinterpret_cast<float4*>(o)[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

}  // namespace pivot
