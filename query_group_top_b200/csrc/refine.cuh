// PIVOT-Refine: every member of a group re-scores the group's candidate set
// with its own query and keeps its own top-k ("PIVOT explained", "How It
// Works": refine_scores = q . K[C], final_indices[q] = top-k(refine_scores);
// paper abstract: "re-scores the candidate set with the indexer of each query
// and then selects an individual top-k").  Member pos only keeps candidates
// j < pos (causality).
//
// One CTA per (group, head), 16 warps.  With nc candidates and
// nch = ceil(nc/128) chunks, chunk c's MMA row r holds candidate r*nch + c, so
// TMEM lane r ends up with the contiguous, ascending block of candidates
// [r*nch, r*nch + nch).  The keys are gathered 128 rows per chunk with 16-byte
// cp.async into the 128-byte-swizzled K-major layout, and one thread issues
// tcgen05.mma with M = 128 candidate rows, N = 16 member queries, K = d; chunk
// c's scores land in TMEM columns [16c, 16c+16).  With Kc <= 4096 the whole
// candidates x members block (4096 x 16 fp32 = 256 KB) stays in TMEM.
//
// Selection: the 16 warps form 4 groups of 4 (one warp per TMEM lane quarter,
// so each group sees all 128 lanes); group q takes members q, q+4, ...  For a
// member, thread r loads its block's scores, and an exact radix select on the
// 32-bit order keys finds the k-th largest key: it starts at the highest key
// bit that varies across the member's candidates (a group-wide AND/OR), takes
// up to 11 bits per pass with a shared histogram and stops as soon as the
// boundary bin is taken whole.
// Because every thread owns an ascending run of candidates, one exclusive scan
// over the 128 threads orders the output, ascending by key index.
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

struct GroupSel {
  int hist[2048];
  int wsum[4];
  int wsum2[4];
  uint32_t wand[4];
  uint32_t wor[4];
  int bstar, above, cntb;
};

template <int D>
struct RefineCfg {
  static constexpr int NT = 512;
  static constexpr int NS = 5;                          // gather stages
  static constexpr int LA = 3;                          // chunks in flight ahead of the MMA
  static constexpr int KATOMS = D / 64;
  static constexpr int ATOM_A = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int STAGE = KATOMS * ATOM_A;
  static constexpr int ATOM_B = 16 * 128;               // 16 member rows x 128 bytes
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = NS * STAGE;
  static constexpr int OFF_C = OFF_B + ((KATOMS * ATOM_B + 1023) / 1024) * 1024;
  // candidate indices are staged for whole 128-row chunks (-1 past the set)
  __host__ __device__ static int cidx_bytes(int Kc) { return ((Kc + 127) / 128) * 128 * 4; }
  static int smem_bytes(int Kc) {
    return OFF_C + cidx_bytes(Kc) + 4 * static_cast<int>(sizeof(GroupSel)) + 64 + 1024;
  }
};

__device__ __forceinline__ void group_sync(int grp) { named_barrier(1 + grp, 128); }

// Exclusive prefix sum over the 128 threads of a group (thread order = r).
__device__ __forceinline__ int group_exclusive_scan(int x, int* wsum, int grp, int quarter, int lane,
                                                   int* total) {
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[quarter] = incl;
  group_sync(grp);
  int off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int s = wsum[w];
    off += (w < quarter) ? s : 0;
    tot += s;
  }
  group_sync(grp);
  if (total) *total = tot;
  return off + incl - x;
}

template <int D>
__global__ void __launch_bounds__(512, 1) refine_kernel(RefineParams p) {
  using C = RefineCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  int32_t* cidx = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  const int off_gs = C::OFF_C + C::cidx_bytes(p.Kc);
  GroupSel* gsel = reinterpret_cast<GroupSel*>(smem + off_gs);
  uint8_t* tail = smem + off_gs + 4 * sizeof(GroupSel);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);            // NS mma-done barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 8 * C::NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 8 * C::NS + 8);
  const uint32_t bar0 = smem_u32(bars);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x / p.G, u = blockIdx.x % p.G;

  // ---- the unit: members, their positions, where keys and outputs live
  int nm, pos0;
  long long key_row0 = 0;      // cache row of key index 0
  long long qrow0;             // row (before *H) of member 0's query and output
  if (p.cu == nullptr) {
    const int s = u * p.g;
    nm = min(s + p.g, p.L) - s;
    pos0 = s;
    qrow0 = s;
  } else {
    nm = p.g;
    key_row0 = p.cu[u];
    pos0 = p.cu[u + 1] - p.cu[u] - p.g;
    qrow0 = static_cast<long long>(u) * p.g;
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
  // chunk c, MMA row r  <->  candidate r*nch + c
  auto issue_gather = [&](int c, int stage) {
    const uint32_t dst0 = sA + stage * C::STAGE;
#pragma unroll
    for (int it = 0; it < (128 * D / 8) / C::NT; ++it) {
      const int id = tid + it * C::NT;
      const int rr = id / (D / 8), piece = id % (D / 8);
      const int a = piece >> 3, p8 = piece & 7;
      const int j = cidx[rr * nch + c];
      const uint16_t* src = kbase + (j >= 0 ? static_cast<long long>(j) * p.H * D : 0) + piece * 8;
      const uint32_t dst = dst0 + a * C::ATOM_A + rr * 128 + ((p8 ^ (rr & 7)) << 4);
      cp_async_16(dst, src, j >= 0 ? 16u : 0u);
    }
  };

  constexpr uint32_t idesc = umma_idesc_bf16(128, 16);
  int seq = 0;           // chunks issued so far (all member batches), drives stage/parity
  int last_commit = -1;  // thread 0: last chunk whose MMAs were committed
  bool ok = true;
  const int grp = warp >> 2, quarter = warp & 3;
  const int r = quarter * 32 + lane;  // TMEM lane: this thread's candidate block
  GroupSel& S = gsel[grp];

  for (int mb = 0; mb < nm && ok; mb += 16) {
    const int nb = min(16, nm - mb);
    // ---- member queries -> B operand (16 rows, swizzled), zero rows past nb
    for (int id = tid; id < 16 * (D / 8); id += C::NT) {
      const int rr = id / (D / 8), piece = id % (D / 8);
      const int a = piece >> 3, p8 = piece & 7;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (rr < nb)
        v = *reinterpret_cast<const uint4*>(p.q + ((qrow0 + mb + rr) * p.H + h) * static_cast<long long>(D) +
                                            piece * 8);
      *reinterpret_cast<uint4*>(smem + C::OFF_B + a * C::ATOM_B + rr * 128 + ((p8 ^ (rr & 7)) << 4)) = v;
    }
    // ---- gather + MMA pipeline over candidate chunks
    const int seq0 = seq;
    // always LA groups in the prologue, so that wait_group<LA> below means
    // "chunk c has landed" whatever nch is
    for (int c = 0; c < C::LA; ++c) {
      if (c < nch) issue_gather(c, (seq0 + c) % C::NS);
      cp_async_commit();
    }
    for (int c = 0; c < nch; ++c) {
      const int cn = c + C::LA;
      if (cn < nch) {
        // the stage refilled now last held chunk cn - NS = c - 2, whose MMAs
        // were issued two iterations ago
        if (cn >= C::NS) {
          const int prev = seq0 + cn - C::NS;
          if (!mbar_wait(bar0 + 8u * (prev % C::NS), (prev / C::NS) & 1, abort_flag, p.status)) ok = false;
        }
        if (ok) issue_gather(cn, (seq0 + cn) % C::NS);
      }
      cp_async_commit();
      cp_async_wait<C::LA>();
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
    if (ok && nch > 0) {
      const int lastc = seq - 1;
      if (!mbar_wait(bar0 + 8u * (lastc % C::NS), (lastc / C::NS) & 1, abort_flag, p.status)) ok = false;
    }
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    tc_fence_after();

    // ---- per-member exact top-k, four groups of 128 threads in parallel
    const int32_t* myc = cidx + r * nch;   // this thread's ascending candidate run
    for (int m = mb + grp; m < mb + nb; m += 4) {
      const int pos = pos0 + m;
      const int col = m - mb;
      uint32_t key[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        key[c] = 0;
        if (c < nch) tmem_ld_32x32b_x1(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c * 16 + col, key[c]);
      }
      // usable candidates of this thread: the ascending prefix with 0 <= j < pos
      int lo = 0, hi = nch;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int j = myc[mid];
        if (j >= 0 && j < pos) lo = mid + 1;
        else hi = mid;
      }
      const int nvt = lo;
      tmem_ld_wait();
      uint32_t kand = 0xFFFFFFFFu, kor = 0u;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        reg_fence(key[c]);
        key[c] = score_key(__uint_as_float(key[c]));
        if (c < nvt) {
          kand &= key[c];
          kor |= key[c];
        }
      }
      // group totals: usable count, and which key bits vary across the member
      {
        const int wn = __reduce_add_sync(0xffffffffu, nvt);
        const uint32_t wa = __reduce_and_sync(0xffffffffu, kand);
        const uint32_t wo = __reduce_or_sync(0xffffffffu, kor);
        if (lane == 0) {
          S.wsum[quarter] = wn;
          S.wand[quarter] = wa;
          S.wor[quarter] = wo;
        }
        group_sync(grp);
      }
      const int nv = S.wsum[0] + S.wsum[1] + S.wsum[2] + S.wsum[3];
      const uint32_t gand = S.wand[0] & S.wand[1] & S.wand[2] & S.wand[3];
      const uint32_t gor = S.wor[0] | S.wor[1] | S.wor[2] | S.wor[3];
      group_sync(grp);
      const int K = min(p.top_k, nv);

      // selection rule: take keys whose bits under `tmask` exceed `thr`, and
      // those equal to it -- all of them, or (ties) the first `rank` in order.
      // Bits above the highest varying bit are common to every usable key.
      int sh = 32 - __clz(gor ^ gand);
      uint32_t tmask = sh >= 32 ? 0u : (0xFFFFFFFFu << sh);
      uint32_t thr = gand & tmask;
      int rank = K;
      bool ties = (sh == 0);
      if (K > 0 && K < nv) {
        bool first = true;
#pragma unroll 1
        while (sh > 0) {
          const int width = sh >= 11 ? 11 : sh;
          sh -= width;
          const int nbn = 1 << width;
          for (int b = r; b < nbn; b += 128) S.hist[b] = 0;
          group_sync(grp);
          if (first) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < nvt) atomicAdd(&S.hist[(key[c] >> sh) & (nbn - 1)], 1);
          } else {
            // only the few keys inside the current boundary bin take part
            uint32_t mm = 0;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < nvt && (key[c] & tmask) == thr) mm |= 1u << c;
            if (mm) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if ((mm >> c) & 1u) atomicAdd(&S.hist[(key[c] >> sh) & (nbn - 1)], 1);
            }
          }
          first = false;
          group_sync(grp);
          // thread r owns bins [top - per + 1, top]; the reads are rotated by r
          // to keep the 32 lanes on different banks
          const int per = nbn >= 128 ? nbn / 128 : 1;
          const int top = nbn - 1 - per * r;
          int s = 0;
          if (top >= 0)
            for (int t = 0; t < per; ++t) s += S.hist[top - ((t + r) & (per - 1))];
          const int excl = group_exclusive_scan(s, S.wsum2, grp, quarter, lane, nullptr);
          if (top >= 0 && excl < rank && rank <= excl + s) {
            int cum = excl;
            for (int t = 0; t < per; ++t) {
              const int cb = S.hist[top - t];
              if (cum + cb >= rank) {
                S.bstar = top - t;
                S.above = cum;
                S.cntb = cb;
                break;
              }
              cum += cb;
            }
          }
          group_sync(grp);
          thr |= static_cast<uint32_t>(S.bstar) << sh;
          tmask |= static_cast<uint32_t>(nbn - 1) << sh;
          rank -= S.above;
          const bool whole = (S.cntb == rank);
          group_sync(grp);
          if (whole) break;           // every key of the boundary bin is taken
          if (sh == 0) ties = true;   // equal keys, only `rank` of them are taken
        }
      }
      // ---- selection flags and ordered emission
      uint32_t sel = 0;
      if (K > 0) {
        if (K >= nv) {
          sel = nvt >= 32 ? 0xFFFFFFFFu : ((1u << nvt) - 1u);
        } else if (!ties) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nvt && (key[c] & tmask) >= thr) sel |= 1u << c;
        } else {
          int neq = 0;
#pragma unroll
          for (int c = 0; c < 32; ++c) neq += (c < nvt && key[c] == thr) ? 1 : 0;
          int eq_before = group_exclusive_scan(neq, S.wsum2, grp, quarter, lane, nullptr);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < nvt) {
              if (key[c] > thr) {
                sel |= 1u << c;
              } else if (key[c] == thr) {
                if (eq_before < rank) sel |= 1u << c;
                ++eq_before;
              }
            }
          }
        }
      }
      int slot = group_exclusive_scan(__popc(sel), S.wsum2, grp, quarter, lane, nullptr);
      int32_t* orow = p.out + ((qrow0 + m) * p.H + h) * static_cast<long long>(p.top_k);
      float* srow = p.out_scores ? p.out_scores + ((qrow0 + m) * p.H + h) * static_cast<long long>(p.top_k) : nullptr;
      if (srow) {
        int sslot = slot;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if ((sel >> c) & 1u) srow[sslot++] = key_score(key[c]);
      }
      for (uint32_t bits = sel; bits; bits &= bits - 1) orow[slot++] = myc[__ffs(bits) - 1];
      for (int t = K + r; t < p.top_k; t += 128) {
        orow[t] = -1;
        if (srow) srow[t] = __int_as_float(0x7fc00000);
      }
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
