// PIVOT-Refine: every member of a group re-scores the group's candidate set
// with its own query and keeps its own top-k ("PIVOT explained", "How It
// Works": refine_scores = q . K[C], final_indices[q] = top-k(refine_scores);
// paper abstract: "re-scores the candidate set with the indexer of each query
// and then selects an individual top-k").  Member pos only keeps candidates
// j < pos (causality).
//
// One CTA per (group, head).  The candidate keys are gathered 128 at a time
// with 16-byte cp.async into the 128-byte-swizzled K-major layout, and one
// thread issues tcgen05.mma with M = 128 candidates, N = 16 member queries,
// K = d, accumulating chunk c's scores into TMEM columns [16c, 16c+16).  With
// Kc <= 4096 the whole candidates x members score block (4096 x 16 fp32 =
// 256 KB) stays in TMEM, and the per-member exact select reads it from there:
// the 8 warps split into two halves of 4 (one per TMEM lane quarter), each half
// selecting for alternate members with a 4-pass radix select over its 128
// threads, then writing the selected candidates in ascending order.
#pragma once

#include "ptx.cuh"

namespace pivot {

struct RefineParams {
  const uint16_t* q;      // prefill [L][H][d]; decode [B][g][H][d]
  const uint16_t* keys;   // prefill [L][H][d]; decode packed cache [rows][H][d]
  const int32_t* cand;    // [H][G][Kc], ascending, -1 padded
  int32_t* out;           // prefill [L][H][top_k]; decode [B][g][H][top_k]
  float* out_scores;      // same shape as out, or null
  const int32_t* cu;      // decode: [B+1] cache row offsets; null for prefill
  int G, L, H, g, top_k, Kc, d;
  uint32_t tmem_cols;
  int* status;
};

struct HalfSel {
  int hist[256];
  int eq[128];
  int sel[128];
  int bstar, above;
};

template <int D>
struct RefineCfg {
  static constexpr int NT = 256;
  static constexpr int NS = 4;                          // gather stages
  static constexpr int KATOMS = D / 64;
  static constexpr int ATOM_A = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int STAGE = KATOMS * ATOM_A;
  static constexpr int ATOM_B = 16 * 128;               // 16 member rows x 128 bytes
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = NS * STAGE;
  static constexpr int OFF_C = OFF_B + KATOMS * ATOM_B + 1024 - (KATOMS * ATOM_B) % 1024;
  // candidate indices are staged for whole 128-row chunks (-1 past the set)
  __host__ __device__ static int cidx_bytes(int Kc) { return ((Kc + 127) / 128) * 128 * 4; }
  static int smem_bytes(int Kc) {
    return OFF_C + cidx_bytes(Kc) + 2 * static_cast<int>(sizeof(HalfSel)) + 64 + 1024;
  }
};

__device__ __forceinline__ void half_sync(int half) { named_barrier(1 + half, 128); }

template <int D>
__global__ void __launch_bounds__(256, 1) refine_kernel(RefineParams p) {
  using C = RefineCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  int32_t* cidx = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  const int off_hs = C::OFF_C + C::cidx_bytes(p.Kc);
  HalfSel* hs = reinterpret_cast<HalfSel*>(smem + off_hs);
  uint8_t* tail = smem + off_hs + 2 * sizeof(HalfSel);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);            // NS mma-done barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 8 * C::NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 8 * C::NS + 8);
  const uint32_t bar0 = smem_u32(bars);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x / p.G, u = blockIdx.x % p.G;

  // ---- the unit: members, their positions, where keys and outputs live
  int nm, pos0;
  long long key_row0 = 0;      // cache row of key index 0
  long long qrow0, orow0;      // row (before *H) of member 0's query / output
  if (p.cu == nullptr) {
    const int s = u * p.g;
    nm = min(s + p.g, p.L) - s;
    pos0 = s;
    qrow0 = s;
    orow0 = s;
  } else {
    nm = p.g;
    key_row0 = p.cu[u];
    pos0 = p.cu[u + 1] - p.cu[u] - p.g;
    qrow0 = static_cast<long long>(u) * p.g;
    orow0 = qrow0;
  }
  const int last = pos0 + nm - 1;
  const int nc = min(p.Kc, max(last, 0));
  const int nch = (nc + 127) / 128;

  if (tid == 0) {
    for (int s = 0; s < C::NS; ++s) mbar_init(bar0 + 8u * s, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  const int32_t* crow = p.cand + (static_cast<long long>(h) * p.G + u) * p.Kc;
  for (int t = tid; t < nch * 128; t += C::NT) cidx[t] = (t < nc) ? crow[t] : -1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint16_t* kbase = p.keys + (key_row0 * p.H + h) * static_cast<long long>(D);
  auto issue_gather = [&](int c, int stage) {
    const uint32_t dst0 = sA + stage * C::STAGE;
#pragma unroll
    for (int it = 0; it < (128 * D / 8) / C::NT; ++it) {
      const int id = tid + it * C::NT;
      const int r = id / (D / 8), piece = id % (D / 8);
      const int a = piece >> 3, p8 = piece & 7;
      const int j = cidx[c * 128 + r];
      const uint16_t* src = kbase + (j >= 0 ? static_cast<long long>(j) * p.H * D : 0) + piece * 8;
      const uint32_t dst = dst0 + a * C::ATOM_A + r * 128 + ((p8 ^ (r & 7)) << 4);
      cp_async_16(dst, src, j >= 0 ? 16u : 0u);
    }
  };

  constexpr uint32_t idesc = umma_idesc_bf16(128, 16);
  int seq = 0;  // chunks issued so far (all member batches), drives stage/parity
  int last_commit = -1;  // thread 0: last chunk whose MMAs were committed
  bool ok = true;
  const int half = warp >> 2, quarter = warp & 3;
  const int r_lane = quarter * 32 + lane;  // TMEM lane = candidate row within a chunk
  HalfSel& S = hs[half];

  for (int mb = 0; mb < nm && ok; mb += 16) {
    const int nb = min(16, nm - mb);
    // ---- member queries -> B operand (16 rows, swizzled), zero rows past nb
    for (int id = tid; id < 16 * (D / 8); id += C::NT) {
      const int r = id / (D / 8), piece = id % (D / 8);
      const int a = piece >> 3, p8 = piece & 7;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nb)
        v = *reinterpret_cast<const uint4*>(p.q + ((qrow0 + mb + r) * p.H + h) * static_cast<long long>(D) + piece * 8);
      *reinterpret_cast<uint4*>(smem + C::OFF_B + a * C::ATOM_B + r * 128 + ((p8 ^ (r & 7)) << 4)) = v;
    }
    // ---- gather + MMA pipeline over candidate chunks
    const int seq0 = seq;
    // always NS-1 groups in the prologue, so that wait_group<NS-1> below
    // means "chunk c has landed" whatever nch is
    for (int c = 0; c < C::NS - 1; ++c) {
      if (c < nch) issue_gather(c, (seq0 + c) % C::NS);
      cp_async_commit();
    }
    for (int c = 0; c < nch; ++c) {
      const int cn = c + C::NS - 1;
      if (cn < nch) {
        if (c >= 1) {
          const int prev = seq0 + c - 1;  // chunk whose stage is refilled now
          if (!mbar_wait(bar0 + 8u * (prev % C::NS), (prev / C::NS) & 1, abort_flag, p.status)) {
            ok = false;
          }
        }
        if (ok) issue_gather(cn, (seq0 + cn) % C::NS);
      }
      cp_async_commit();
      cp_async_wait<C::NS - 1>();
      fence_proxy_async_smem();
      if (__syncthreads_or(!ok)) {
        ok = false;
        break;
      }
      if (tid == 0) {
        tc_fence_after();
        const int st = (seq0 + c) % C::NS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int a = kk >> 2, k4 = kk & 3;
          const uint64_t adesc = sw128_kmajor_desc(sA + st * C::STAGE + a * C::ATOM_A + k4 * 32);
          const uint64_t bdesc = sw128_kmajor_desc(sB + a * C::ATOM_B + k4 * 32);
          umma_bf16(tmem + c * 16, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar0 + 8u * st);
        last_commit = seq0 + c;
      }
    }
    cp_async_wait<0>();
    seq = seq0 + nch;
    if (nch > 0) {
      const int lastc = seq - 1;
      if (!mbar_wait(bar0 + 8u * (lastc % C::NS), (lastc / C::NS) & 1, abort_flag, p.status)) ok = false;
    }
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    tc_fence_after();

    // ---- per-member exact top-k, two halves of 128 threads in parallel
    for (int m = mb + half; m < mb + nb; m += 2) {
      const int pos = pos0 + m;
      const int col = m - mb;
      uint32_t key[32];
      uint32_t valid = 0;  // bit c: candidate (c, r_lane) is usable by this member
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        key[c] = 0;
        if (c < nch) {
          uint32_t v;
          tmem_ld_32x32b_x1(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c * 16 + col, v);
          key[c] = v;
        }
      }
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        reg_fence(key[c]);
        if (c < nch) {
          const int j = cidx[c * 128 + r_lane];
          if (j >= 0 && j < pos) valid |= 1u << c;
          key[c] = score_key(__uint_as_float(key[c]));
        }
      }
      // number of usable candidates
      int nv = __popc(valid);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
      if (lane == 0) S.eq[quarter] = nv;
      half_sync(half);
      nv = S.eq[0] + S.eq[1] + S.eq[2] + S.eq[3];
      const int K = min(p.top_k, nv);
      half_sync(half);

      uint32_t T = 0;
      int need_eq = 0;
      if (K > 0 && K < nv) {
        uint32_t prefix = 0, mask = 0;
        int rank = K;
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
          for (int b = r_lane; b < 256; b += 128) S.hist[b] = 0;
          if (r_lane == 0) { S.bstar = 0; S.above = 0; }
          half_sync(half);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < nch) {
              int digit = 256 + lane;
              if (((valid >> c) & 1u) && (key[c] & mask) == prefix) digit = (key[c] >> shift) & 255;
              const unsigned same = __match_any_sync(0xffffffffu, digit);
              if (digit < 256 && lane == __ffs(same) - 1) atomicAdd(&S.hist[digit], __popc(same));
            }
          }
          half_sync(half);
          if (quarter == 0) {
            const int hi_bin = 255 - 8 * lane;
            int cb[8], s = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) { cb[t] = S.hist[hi_bin - t]; s += cb[t]; }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += y;
            }
            const int excl = incl - s;
            const unsigned hit = __ballot_sync(0xffffffffu, excl < rank && rank <= incl);
            if (hit && lane == __ffs(hit) - 1) {
              int cum = excl;
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                if (cum + cb[t] >= rank) { S.bstar = hi_bin - t; S.above = cum; break; }
                cum += cb[t];
              }
            }
          }
          half_sync(half);
          prefix |= static_cast<uint32_t>(S.bstar) << shift;
          mask |= 0xFFu << shift;
          rank -= S.above;
          half_sync(half);
        }
        T = prefix;
        need_eq = rank;
      }
      // ---- ordered emission: entry order is (chunk, quarter, lane) = ascending key index
      const unsigned lt = (1u << lane) - 1u;
      int32_t* orow = p.out + ((orow0 + m) * p.H + h) * static_cast<long long>(p.top_k);
      float* srow = p.out_scores ? p.out_scores + ((orow0 + m) * p.H + h) * static_cast<long long>(p.top_k) : nullptr;
      uint32_t eqm[32];
      if (K > 0) {
        const bool take_all = (K >= nv);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          eqm[c] = 0;
          if (c < nch) {
            const bool v = (valid >> c) & 1u;
            const unsigned eb = __ballot_sync(0xffffffffu, v && !take_all && key[c] == T);
            eqm[c] = eb;
            if (lane == 0) S.eq[c * 4 + quarter] = __popc(eb);
          }
        }
        half_sync(half);
        // exclusive scan of S.eq[0..4*nch) over the half's 128 threads (one entry each)
        {
          const int x = (r_lane < 4 * nch) ? S.eq[r_lane] : 0;
          int incl = x;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (lane == 31) S.hist[quarter] = incl;
          half_sync(half);
          int off = 0;
          for (int w = 0; w < quarter; ++w) off += S.hist[w];
          half_sync(half);
          if (r_lane < 4 * nch) S.eq[r_lane] = off + incl - x;
          half_sync(half);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < nch) {
            const bool v = (valid >> c) & 1u;
            bool take = false;
            if (v) {
              if (take_all || key[c] > T) take = true;
              else if (key[c] == T) take = (S.eq[c * 4 + quarter] + __popc(eqm[c] & lt)) < need_eq;
            }
            const unsigned sb = __ballot_sync(0xffffffffu, take);
            eqm[c] = sb;  // reuse: selection mask of this warp for chunk c
            if (lane == 0) S.sel[c * 4 + quarter] = __popc(sb);
          }
        }
        half_sync(half);
        {
          const int x = (r_lane < 4 * nch) ? S.sel[r_lane] : 0;
          int incl = x;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (lane == 31) S.hist[4 + quarter] = incl;
          half_sync(half);
          int off = 0;
          for (int w = 0; w < quarter; ++w) off += S.hist[4 + w];
          half_sync(half);
          if (r_lane < 4 * nch) S.sel[r_lane] = off + incl - x;
          half_sync(half);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < nch && ((eqm[c] >> lane) & 1u)) {
            const int slot = S.sel[c * 4 + quarter] + __popc(eqm[c] & lt);
            orow[slot] = cidx[c * 128 + r_lane];
            if (srow) {
              const uint32_t kk = key[c];
              const uint32_t bits = (kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk;
              srow[slot] = __uint_as_float(bits);
            }
          }
        }
      }
      for (int t = K + r_lane; t < p.top_k; t += 128) {
        orow[t] = -1;
        if (srow) srow[t] = __int_as_float(0x7fc00000);
      }
      half_sync(half);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // On an aborted run, let the MMAs already issued finish before TMEM is freed.
  if (tid == 0 && !ok && last_commit >= 0)
    mbar_wait_cleanup(bar0 + 8u * (last_commit % C::NS), (last_commit / C::NS) & 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace pivot
