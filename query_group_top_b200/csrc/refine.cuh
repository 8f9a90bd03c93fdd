// PIVOT-Refine: every member of a group re-scores the group's candidate set
// with its own query and keeps its own top-k ("PIVOT explained", "How It
// Works": refine_scores = q . K[C], final_indices[q] = top-k(refine_scores);
// paper abstract: "re-scores the candidate set with the indexer of each query
// and then selects an individual top-k").  Member pos only keeps candidates
// j < pos (causality).
//
// One CTA per (group, head), 16 warps.  With nc candidates and
// nch = ceil(nc/128) chunks, chunk c's MMA row r holds candidate
// t = r*nch + c, so TMEM lane r ends up with the contiguous, ascending block of
// candidates [r*nch, r*nch + nch).  The keys are gathered 128 rows per chunk
// with 16-byte cp.async into the 128-byte-swizzled K-major layout, and one
// thread issues tcgen05.mma with M = 128 candidate rows, N = 16 member queries,
// K = d; chunk c's scores land in TMEM columns [16c, 16c+16).  With Kc <= 4096
// the whole candidates x members block (4096 x 16 fp32 = 256 KB) stays in TMEM.
//
// Selection (exact, on 32-bit order keys, ties to the lower index):
//  * Warp group grp (4 warps, one per TMEM lane quarter) owns members
//    4grp..4grp+3, read with one 4-column TMEM load per chunk.
//  * Round 0 runs inside the gather/MMA loop, two chunks behind the MMA: chunk
//    0 is a 128-candidate sample spread over the whole set; its key range sets
//    a linear 2048-bin histogram (monotone in the key, clamped at both ends),
//    and every chunk is counted into it as soon as its scores exist.
//  * After the loop, warp m finds member m's boundary bin with a two-level scan
//    and inverts the bin function to key thresholds [kl, kh); one TMEM pass
//    then marks each thread's candidates "above" (key >= kh) or "boundary".
//  * A boundary of up to kListCap keys is ranked exactly from a shared list;
//    larger boundaries are narrowed by further histogram rounds over their own
//    key range, and a boundary of equal keys takes its first keys in order.
//  * Output: one group scan gives every thread its output slot; each warp
//    stages its slice of the row in shared memory and writes it coalesced.
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

// member selection modes
enum : int {
  kMNone = 0,    // takes nothing (no usable candidate)
  kMAll = 1,     // takes every usable candidate (top_k >= usable count)
  kMSel = 2,     // narrowing: the boundary bin of the current round is open
  kMWhole = 3,   // every key of the boundary bin is taken
  kMList = 4,    // boundary ranked from the shared list: (tk, need_eq) known
  kMNarrow = 5,  // boundary too large for the list: another round
  kMTies = 6,    // boundary keys all equal: the first need_eq in order
};

constexpr int kRefBins = 2048;
constexpr int kListCap = 256;

struct MemberSel {
  int nv;           // usable candidates: the ascending prefix with j < pos
  int K;            // min(top_k, nv)
  int mode;
  int active;       // takes part in the current round
  int need;         // keys still to take from the current candidate interval
  int cnt;          // keys in the boundary bin
  uint32_t lo;      // bin function: origin (a key, or a score's bits) and scale
  float scale;
  int vmode;        // bins linear in the score (1) or in the order key (0)
  uint32_t kl, kh;  // boundary bin = keys in [kl, kh); kh_inf: no upper edge
  int kh_inf;
  uint32_t bmin, bmax;
  uint32_t tk;      // final rule: keys > tk, then keys == tk in order up to need_eq
  int need_eq;
  int nlist;
};

struct RefineMisc {
  MemberSel ms[16];
  uint32_t pmin[4][16], pmax[4][16];
  int gscan[4][4][8];
  uint64_t bars[8];
  uint32_t tmem_slot;
  int abort_flag;
  int more;
};

template <int D>
struct RefineCfg {
  static constexpr int NT = 512;
  static constexpr int NS = 4;                          // gather stages
  static constexpr int LA = 2;                          // chunks in flight ahead of the MMA
  static_assert(NS == LA + 2, "stage reuse and score reads both trail the MMA by two chunks");
  static constexpr int KATOMS = D / 64;
  static constexpr int ATOM_A = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int STAGE = KATOMS * ATOM_A;
  static constexpr int ATOM_B = 16 * 128;               // 16 member rows x 128 bytes
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = NS * STAGE;
  static constexpr int OFF_C = OFF_B + ((KATOMS * ATOM_B + 1023) / 1024) * 1024;
  // histograms: 16 members x 2048 bins of 16-bit counts (two per word); the
  // same bytes later hold the boundary lists and the per-warp output staging
  static constexpr int HIST_BYTES = 16 * (kRefBins / 2) * 4;
  static_assert(16 * 2 * kListCap * 4 <= HIST_BYTES, "lists alias the histograms");
  static_assert(16 * 1024 * 4 <= HIST_BYTES, "output staging aliases the histograms");
  // candidate indices are staged for whole 128-row chunks (-1 past the set)
  __host__ __device__ static int cidx_bytes(int Kc) { return ((Kc + 127) / 128) * 128 * 4; }
  static int smem_bytes(int Kc) {
    return OFF_C + cidx_bytes(Kc) + HIST_BYTES + static_cast<int>(sizeof(RefineMisc)) + 1024;
  }
};

// Linear bin of an order key over [lo, ...) with `scale` bins per key unit,
// clamped to [0, 2047].  Every step (difference, conversion, product,
// truncation, clamp) is non-decreasing in the key, so the bins are ordered
// like the keys and equal keys share a bin.
__device__ __forceinline__ int key_bin(uint32_t key, uint32_t lo, float scale) {
  const uint32_t dl = key > lo ? key - lo : 0u;
  const uint32_t b = __float2uint_rz(__uint2float_rn(dl) * scale);
  return static_cast<int>(min(b, static_cast<uint32_t>(kRefBins - 1)));
}

// Linear bin of a score over [lo, ...), clamped to [0, 2047]; explicit
// roundings keep every step non-decreasing in the score, and -0 and +0 share
// a bin.  Scores of real data spread evenly over such bins, while order keys
// of scores on both sides of zero crowd into a few of the key-linear ones.
__device__ __forceinline__ int value_bin(float s, float lo, float scale) {
  const float x = __fmul_rn(__fsub_rn(s, lo), scale);
  return min(max(__float2int_rz(x), 0), kRefBins - 1);
}

// Bin of an order key under either bin function; key patterns beyond the
// infinities (no score has them) clamp to the infinities.
__device__ __forceinline__ int bin_of_key(uint32_t key, uint32_t lo, float scale, bool vmode) {
  if (!vmode) return key_bin(key, lo, scale);
  const uint32_t kc = min(max(key, 0x007FFFFFu), 0xFF800000u);
  return value_bin(key_score(kc), __uint_as_float(lo), scale);
}

// Smallest key whose bin is >= b (1 <= b <= 2047), searched by the whole warp
// 32 ways at a time; false when no key reaches bin b.
__device__ __forceinline__ bool warp_first_key_of_bin(int b, uint32_t lo, float scale, bool vmode, int lane,
                                                      uint32_t* out) {
  if (bin_of_key(0xFFFFFFFFu, lo, scale, vmode) < b) return false;
  unsigned long long base = 0, span = 1ull << 32;
  while (span > 1) {
    const unsigned long long stride = (span + 31) / 32;
    const unsigned long long first = base + static_cast<unsigned long long>(lane) * stride;
    bool ge = true;  // empty sub-ranges count as "beyond"
    if (first < base + span) {
      const unsigned long long last = min(first + stride, base + span) - 1;
      ge = bin_of_key(static_cast<uint32_t>(last), lo, scale, vmode) >= b;
    }
    const int j = __ffs(__ballot_sync(0xffffffffu, ge)) - 1;
    const unsigned long long nb = base + static_cast<unsigned long long>(j) * stride;
    span = min(stride, base + span - nb);
    base = nb;
  }
  *out = static_cast<uint32_t>(base);
  return true;
}

__device__ __forceinline__ void group_sync(int grp) { named_barrier(1 + grp, 128); }

template <int D>
__global__ void __launch_bounds__(512, 1) refine_kernel(RefineParams p) {
  using C = RefineCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  int32_t* cidx = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  const int off_h = C::OFF_C + C::cidx_bytes(p.Kc);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + off_h);
  RefineMisc* M = reinterpret_cast<RefineMisc*>(smem + off_h + C::HIST_BYTES);
  volatile int* abort_flag = &M->abort_flag;
  const uint32_t bar0 = smem_u32(&M->bars[0]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, quarter = warp & 3;
  const int r = quarter * 32 + lane;  // TMEM lane: this thread's candidate block
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
    tmem_alloc(smem_u32(&M->tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  // candidate t = r*nch + c lives at cidx[c*128 + ((r + c) & 127)]: conflict-free
  // both along a chunk (fixed c) and along a thread's block (fixed r)
  const int32_t* crow = p.cand + (static_cast<long long>(h) * p.G + u) * p.Kc;
  for (int t = tid; t < nch * 128; t += C::NT) {
    const int rr = t / nch, c = t - rr * nch;
    cidx[c * 128 + ((rr + c) & 127)] = (t < nc) ? crow[t] : -1;
  }
  auto cand_at = [&](int c, int rr) -> int { return cidx[c * 128 + ((rr + c) & 127)]; };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M->tmem_slot;
  const uint32_t tlane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);

  const uint16_t* kbase = p.keys + (key_row0 * p.H + h) * static_cast<long long>(D);
  // chunk c, MMA row r  <->  candidate r*nch + c
  auto issue_gather = [&](int c, int stage) {
    const uint32_t dst0 = sA + stage * C::STAGE;
#pragma unroll
    for (int it = 0; it < (128 * D / 8) / C::NT; ++it) {
      const int id = tid + it * C::NT;
      const int rr = id / (D / 8), piece = id % (D / 8);
      const int a = piece >> 3, p8 = piece & 7;
      const int j = cand_at(c, rr);
      const uint16_t* src = kbase + (j >= 0 ? static_cast<long long>(j) * p.H * D : 0) + piece * 8;
      const uint32_t dst = dst0 + a * C::ATOM_A + rr * 128 + ((p8 ^ (rr & 7)) << 4);
      cp_async_16(dst, src, j >= 0 ? 16u : 0u);
    }
  };

  constexpr uint32_t idesc = umma_idesc_bf16(128, 16);
  int seq = 0;           // chunks issued so far (all member batches), drives stage/parity
  int last_commit = -1;  // thread 0: last chunk whose MMAs were committed
  bool ok = true;

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
    // ---- per-member usable counts (the candidate set is ascending) and modes
    if (tid < 16) {
      MemberSel& S = M->ms[tid];
      int nv = 0;
      if (tid < nb) {
        const int pos = pos0 + mb + tid;
        int lo = 0, hi = nc;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          const int q8 = mid / max(nch, 1);
          if (cand_at(mid - q8 * nch, q8) < pos) lo = mid + 1;
          else hi = mid;
        }
        nv = lo;
      }
      const int K = min(p.top_k, nv);
      S.nv = nv;
      S.K = K;
      S.mode = K == 0 ? kMNone : (K == nv ? kMAll : kMSel);
      S.active = S.mode == kMSel;
      S.need = K;
      S.cnt = nv;
      S.nlist = 0;
      S.bmin = 0xFFFFFFFFu;
      S.bmax = 0u;
      S.need_eq = 0;
      S.tk = 0;
      S.vmode = 0;
    }
    for (int i = tid; i < C::HIST_BYTES / 16; i += C::NT) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    // this thread's view of its four members (member 4*grp + i of the batch)
    uint32_t um[4];       // usable chunks of this thread's block
    uint32_t hm = 0;      // members counted in the round-0 histogram
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const MemberSel& S = M->ms[4 * grp + i];
      const int nvt = min(max(S.nv - r * nch, 0), nch);
      um[i] = nvt >= 32 ? 0xFFFFFFFFu : ((1u << nvt) - 1u);
      hm |= (S.mode == kMSel ? 1u : 0u) << i;
    }
    uint32_t lo4[4] = {0, 0, 0, 0};
    float sc4[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t vm4 = 0;     // members whose round-0 bins are linear in the score

    // round 0, chunk 0: the sample's key range, per lane quarter
    auto sample_range = [&]() {
      uint32_t v[4];
      tmem_ld_32x32b_x4(tlane + 4 * grp, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        reg_fence(v[i]);
        const bool use = ((hm >> i) & 1u) && (um[i] & 1u);
        const uint32_t key = score_key(__uint_as_float(v[i]));
        const uint32_t mn = __reduce_min_sync(0xffffffffu, use ? key : 0xFFFFFFFFu);
        const uint32_t mx = __reduce_max_sync(0xffffffffu, use ? key : 0u);
        if (lane == 0) {
          M->pmin[quarter][4 * grp + i] = mn;
          M->pmax[quarter][4 * grp + i] = mx;
        }
      }
    };
    // bins over the sample's range (every thread of the group computes the same)
    auto set_range = [&]() {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * grp + i;
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          mn = min(mn, M->pmin[qq][m]);
          mx = max(mx, M->pmax[qq][m]);
        }
        const float vmin = key_score(mn), vmax = key_score(mx);
        const float vsc = static_cast<float>(kRefBins) / __fsub_rn(vmax, vmin);
        const bool vm = mn < mx && isfinite(vmin) && isfinite(vmax) && isfinite(vsc) && vsc > 0.f;
        if (vm) {
          lo4[i] = __float_as_uint(vmin);
          sc4[i] = vsc;
          vm4 |= 1u << i;
        } else if (mn > mx) {
          lo4[i] = 0u;
          sc4[i] = 0.f;
        } else {
          lo4[i] = mn;
          sc4[i] = static_cast<float>(kRefBins) / (__uint2float_rn(mx - mn) + 1.0f);
        }
        if (quarter == 0 && lane == 0) {
          M->ms[m].lo = lo4[i];
          M->ms[m].scale = sc4[i];
          M->ms[m].vmode = vm ? 1 : 0;
        }
      }
    };
    auto hist_chunk = [&](int c) {
      uint32_t v[4];
      tmem_ld_32x32b_x4(tlane + c * 16 + 4 * grp, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        reg_fence(v[i]);
        if (((hm >> i) & 1u) && ((um[i] >> c) & 1u)) {
          const float f = __uint_as_float(v[i]);
          const int b = ((vm4 >> i) & 1u) ? value_bin(f, __uint_as_float(lo4[i]), sc4[i])
                                          : key_bin(score_key(f), lo4[i], sc4[i]);
          atomicAdd(&hist[(4 * grp + i) * (kRefBins / 2) + (b >> 1)], 1u << ((b & 1) * 16));
        }
      }
    };
    auto process_chunk = [&](int c) {
      if (hm == 0) return;
      if (c == 0) {
        sample_range();
      } else {
        if (c == 1) {
          set_range();
          hist_chunk(0);
        }
        hist_chunk(c);
      }
    };

    // ---- gather + MMA pipeline over candidate chunks, round-0 histogram two
    //      chunks behind the MMA
    const int seq0 = seq;
    // always LA groups in the prologue, so that wait_group<LA> below means
    // "chunk c has landed" whatever nch is
    for (int c = 0; c < C::LA; ++c) {
      if (c < nch) issue_gather(c, (seq0 + c) % C::NS);
      cp_async_commit();
    }
    for (int c = 0; c < nch; ++c) {
      if (c >= 2) {
        // chunk c-2's MMAs are done: its stage may be refilled (with chunk
        // c + LA) and its scores read
        const int pv = seq0 + c - 2;
        if (ok && !mbar_wait(bar0 + 8u * (pv % C::NS), (pv / C::NS) & 1, abort_flag, p.status)) ok = false;
      }
      const int cn = c + C::LA;
      if (ok && cn < nch) issue_gather(cn, (seq0 + cn) % C::NS);
      cp_async_commit();
      if (c >= 2) {
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          process_chunk(c - 2);
        }
      }
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
    if (!ok) break;
    for (int pp = max(0, nch - 2); pp < nch; ++pp) {
      const int pv = seq0 + pp;
      if (ok && !mbar_wait(bar0 + 8u * (pv % C::NS), (pv / C::NS) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        process_chunk(pp);
      }
      if (pp == 0 && __syncthreads_or(!ok)) ok = false;  // the sample ranges are visible
    }
    if (ok && nch == 1 && hm != 0) {
      set_range();
      hist_chunk(0);
    }
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }

    // ---- selection rounds
    uint32_t gt[4] = {0, 0, 0, 0};   // taken: above the boundary
    uint32_t bnd[4] = {0, 0, 0, 0};  // in the current boundary bin
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (M->ms[4 * grp + i].mode == kMAll) gt[i] = um[i];

#pragma unroll 1
    for (int round = 0;; ++round) {
      // (a) warp m: member m's boundary bin and its key thresholds
      if (warp < nb && M->ms[warp].active) {
        MemberSel& S = M->ms[warp];
        const uint32_t* hw = hist + warp * (kRefBins / 2);
        const int need = S.need;
        // lane l owns words [1024 - 32(l+1), 1024 - 32l): bins in descending order
        const int w0 = kRefBins / 2 - 32 * (lane + 1);
        int s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 x = reinterpret_cast<const uint4*>(hw + w0)[(i + lane) & 7];
          s += (x.x & 0xFFFFu) + (x.x >> 16) + (x.y & 0xFFFFu) + (x.y >> 16) + (x.z & 0xFFFFu) + (x.z >> 16) +
               (x.w & 0xFFFFu) + (x.w >> 16);
        }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int L = __ffs(__ballot_sync(0xffffffffu, incl >= need)) - 1;
        const int exclL = __shfl_sync(0xffffffffu, incl - s, L);
        // lane i: word (1024 - 32L - 1 - i), holding bins 2w+1 (upper half) and 2w
        const int w = kRefBins / 2 - 32 * L - 1 - lane;
        const uint32_t wv = hw[w];
        const int chi = static_cast<int>(wv >> 16), clo = static_cast<int>(wv & 0xFFFFu);
        const int s2 = chi + clo;
        int incl2 = s2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl2, o);
          if (lane >= o) incl2 += y;
        }
        const int i2 = __ffs(__ballot_sync(0xffffffffu, exclL + incl2 >= need)) - 1;
        int bstar = 0, above = 0, cntb = 0;
        if (lane == i2) {
          const int before = exclL + incl2 - s2;
          if (before + chi >= need) {
            bstar = 2 * w + 1;
            above = before;
            cntb = chi;
          } else {
            bstar = 2 * w;
            above = before + chi;
            cntb = clo;
          }
        }
        bstar = __shfl_sync(0xffffffffu, bstar, i2);
        above = __shfl_sync(0xffffffffu, above, i2);
        cntb = __shfl_sync(0xffffffffu, cntb, i2);
        const uint32_t lo = S.lo;
        const float sc = S.scale;
        const bool vm = S.vmode != 0;
        uint32_t kl = 0, kh = 0;
        bool has_kl = true, has_kh = false;
        if (bstar > 0) has_kl = warp_first_key_of_bin(bstar, lo, sc, vm, lane, &kl);
        if (bstar < kRefBins - 1) has_kh = warp_first_key_of_bin(bstar + 1, lo, sc, vm, lane, &kh);
        if (lane == 0) {
          const int need2 = need - above;
          S.need = need2;
          S.cnt = cntb;
          S.kl = has_kl ? kl : 0u;
          S.kh = kh;
          S.kh_inf = has_kh ? 0 : 1;
          S.mode = (cntb == need2) ? kMWhole : (cntb <= kListCap ? kMList : kMNarrow);
          S.nlist = 0;
          S.bmin = 0xFFFFFFFFu;
          S.bmax = 0u;
        }
      }
      __syncthreads();

      // (b) one pass over the scores: above / boundary, boundary lists and ranges
      {
        uint32_t act = 0, lst = 0, nar = 0;
        uint32_t kl4[4], kh4[4];
        bool khinf4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const MemberSel& S = M->ms[4 * grp + i];
          const bool a = S.active != 0;
          act |= (a ? 1u : 0u) << i;
          lst |= (a && S.mode == kMList ? 1u : 0u) << i;
          nar |= (a && S.mode == kMNarrow ? 1u : 0u) << i;
          kl4[i] = S.kl;
          kh4[i] = S.kh;
          khinf4[i] = S.kh_inf != 0;
        }
        uint32_t cand4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          cand4[i] = ((act >> i) & 1u) ? (round == 0 ? um[i] : bnd[i]) : 0u;
          if ((act >> i) & 1u) bnd[i] = 0u;
        }
        uint32_t bmn[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
        uint32_t bmx[4] = {0u, 0u, 0u, 0u};
        const uint32_t any = __reduce_or_sync(0xffffffffu, cand4[0] | cand4[1] | cand4[2] | cand4[3]);
        if (act != 0) {
#pragma unroll 1
          for (int cb = 0; cb < nch; cb += 8) {
            if (((any >> cb) & 0xFFu) == 0u) continue;
            uint32_t v[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (cb + j < nch) tmem_ld_32x32b_x4(tlane + (cb + j) * 16 + 4 * grp, v[j]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                reg_fence(v[j][i]);
                const int c = cb + j;
                if (c < nch && ((cand4[i] >> c) & 1u)) {
                  const uint32_t key = score_key(__uint_as_float(v[j][i]));
                  if (!khinf4[i] && key >= kh4[i]) {
                    gt[i] |= 1u << c;
                  } else if (key >= kl4[i]) {
                    bnd[i] |= 1u << c;
                    bmn[i] = min(bmn[i], key);
                    bmx[i] = max(bmx[i], key);
                    if ((lst >> i) & 1u) {
                      const int m = 4 * grp + i;
                      const int at = atomicAdd(&M->ms[m].nlist, 1);
                      if (at < kListCap) {
                        hist[m * 2 * kListCap + at] = key;
                        hist[m * 2 * kListCap + kListCap + at] = static_cast<uint32_t>(r * nch + c);
                      }
                    }
                  }
                }
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if ((nar >> i) & 1u) {
              const uint32_t mn = __reduce_min_sync(0xffffffffu, bmn[i]);
              const uint32_t mx = __reduce_max_sync(0xffffffffu, bmx[i]);
              if (lane == 0) {
                atomicMin(&M->ms[4 * grp + i].bmin, mn);
                atomicMax(&M->ms[4 * grp + i].bmax, mx);
              }
            }
          }
        }
      }
      if (tid == 0) M->more = 0;
      __syncthreads();

      // (c) warp m closes member m's round: rank the list, or detect equal
      //     keys, or set up the next round over the boundary's own range
      if (warp < nb && M->ms[warp].active) {
        MemberSel& S = M->ms[warp];
        const int mode = S.mode;
        const int need = S.need;
        if (mode == kMWhole) {
          if (lane == 0) {
            S.need_eq = 0x7FFFFFFF;
            S.active = 0;
          }
        } else if (mode == kMList) {
          const int n = min(S.nlist, kListCap);
          const uint32_t* lk = hist + warp * 2 * kListCap;
          // the need-th largest key (with multiplicity) and how many of its
          // copies are taken
          for (int e = lane; e < n; e += 32) {
            const uint32_t ke = lk[e];
            int ngt = 0, neq = 0;
            for (int f = 0; f < n; ++f) {
              const uint32_t kf = lk[f];
              ngt += kf > ke ? 1 : 0;
              neq += kf == ke ? 1 : 0;
            }
            if (ngt < need && need <= ngt + neq) {
              S.tk = ke;             // every such lane writes the same values
              S.need_eq = need - ngt;
            }
          }
          __syncwarp();
          if (lane == 0) S.active = 0;
        } else {  // kMNarrow
          if (lane == 0) {
            const uint32_t mn = S.bmin, mx = S.bmax;
            if (mn == mx) {
              S.mode = kMTies;
              S.tk = mn;
              S.need_eq = need;
              S.active = 0;
            } else {
              S.lo = mn;
              S.scale = static_cast<float>(kRefBins) / (__uint2float_rn(mx - mn) + 1.0f);
              S.vmode = 0;
              S.mode = kMSel;
              M->more = 1;
            }
          }
        }
      }
      __syncthreads();
      if (!M->more) break;

      // (d) another histogram round over the open boundaries (rare: more than
      //     kListCap keys in one bin with distinct values)
      for (int i = tid; i < C::HIST_BYTES / 16; i += C::NT) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
      __syncthreads();
      {
        uint32_t act = 0;
        uint32_t lo_[4];
        float sc_[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const MemberSel& S = M->ms[4 * grp + i];
          act |= (S.active ? 1u : 0u) << i;
          lo_[i] = S.lo;
          sc_[i] = S.scale;
        }
        uint32_t c4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) c4[i] = ((act >> i) & 1u) ? bnd[i] : 0u;
        const uint32_t any = __reduce_or_sync(0xffffffffu, c4[0] | c4[1] | c4[2] | c4[3]);
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          if (((any >> c) & 1u) == 0u) continue;
          uint32_t v[4];
          tmem_ld_32x32b_x4(tlane + c * 16 + 4 * grp, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reg_fence(v[i]);
            if ((c4[i] >> c) & 1u) {
              const int b = key_bin(score_key(__uint_as_float(v[i])), lo_[i], sc_[i]);
              atomicAdd(&hist[(4 * grp + i) * (kRefBins / 2) + (b >> 1)], 1u << ((b & 1) * 16));
            }
          }
        }
      }
      __syncthreads();
    }

    // ---- final rule per member: gt, plus the first need_eq of eq in order
    uint32_t eq[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const MemberSel& S = M->ms[4 * grp + i];
      const int mode = S.mode;
      if (mode == kMWhole || mode == kMTies) {
        eq[i] = bnd[i];
      } else if (mode == kMList) {
        // re-read the few boundary keys and split them around tk
        const uint32_t tk = S.tk;
        uint32_t any = __reduce_or_sync(0xffffffffu, bnd[i]);
        while (any) {
          const int c = __ffs(any) - 1;
          any &= any - 1;
          uint32_t v;
          tmem_ld_32x32b_x1(tlane + c * 16 + 4 * grp + i, v);
          tmem_ld_wait();
          if ((bnd[i] >> c) & 1u) {
            const uint32_t key = score_key(__uint_as_float(v));
            if (key > tk) gt[i] |= 1u << c;
            else if (key == tk) eq[i] |= 1u << c;
          }
        }
      }
    }
    // group scan (thread order = candidate order) of (|gt|, |eq|) for 4 members
    int ex[8];
    {
      int incl[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        incl[i] = __popc(gt[i]);
        incl[4 + i] = __popc(eq[i]);
      }
      int own[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) own[k] = incl[k];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int y = __shfl_up_sync(0xffffffffu, incl[k], o);
          if (lane >= o) incl[k] += y;
        }
      }
      if (lane == 31) {
#pragma unroll
        for (int k = 0; k < 8; ++k) M->gscan[grp][quarter][k] = incl[k];
      }
      group_sync(grp);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        int off = 0;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) off += (qq < quarter) ? M->gscan[grp][qq][k] : 0;
        ex[k] = off + incl[k] - own[k];
      }
    }
    // the histogram bytes become per-warp output staging (1024 entries a warp)
    uint32_t* stg = hist + warp * 1024;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 4 * grp + i;
      if (m >= nb) continue;
      const MemberSel& S = M->ms[m];
      const int K = S.K, need_eq = S.need_eq;
      const int eqb = ex[4 + i];
      const int neq = __popc(eq[i]);
      const int take = min(max(need_eq - eqb, 0), neq);
      uint32_t sel = gt[i];
      if (take == neq) {
        sel |= eq[i];
      } else {
        uint32_t e = eq[i];
        for (int k = 0; k < take; ++k) {
          sel |= e & (0u - e);  // lowest remaining equal key
          e &= e - 1;
        }
      }
      const int slot = ex[i] + min(eqb, need_eq);
      const int wb = __shfl_sync(0xffffffffu, slot, 0);
      const int wc = __shfl_sync(0xffffffffu, slot + __popc(sel), 31) - wb;
      const long long orow_off = ((qrow0 + mb + m) * p.H + h) * static_cast<long long>(p.top_k);
      int32_t* orow = p.out + orow_off;
      {
        int o = slot - wb;
        for (uint32_t bits = sel; bits; bits &= bits - 1) {
          const int c = __ffs(bits) - 1;
          stg[o++] = static_cast<uint32_t>(cand_at(c, r));
        }
      }
      __syncwarp();
      for (int x = lane; x < wc; x += 32) orow[wb + x] = static_cast<int32_t>(stg[x]);
      __syncwarp();
      if (p.out_scores) {
        float* srow = p.out_scores + orow_off;
        uint32_t any = __reduce_or_sync(0xffffffffu, sel);
        int o = slot - wb;
        while (any) {
          const int c = __ffs(any) - 1;
          any &= any - 1;
          uint32_t v;
          tmem_ld_32x32b_x1(tlane + c * 16 + 4 * grp + i, v);
          tmem_ld_wait();
          if ((sel >> c) & 1u) stg[o++] = v;
        }
        __syncwarp();
        for (int x = lane; x < wc; x += 32) srow[wb + x] = __uint_as_float(stg[x]);
        __syncwarp();
        for (int x = K + r; x < p.top_k; x += 128) srow[x] = __int_as_float(0x7fc00000);
      }
      for (int x = K + r; x < p.top_k; x += 128) orow[x] = -1;
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
