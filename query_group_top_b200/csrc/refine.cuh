// PIVOT-Refine: every member of a group re-scores the group's candidate set
// with its own query and keeps its own top-k ("PIVOT explained", "How It
// Works": refine_scores = q . K[C], final_indices[q] = top-k(refine_scores);
// paper abstract: "re-scores the candidate set with the indexer of each query
// and then selects an individual top-k").  Member pos only keeps candidates
// j < pos (causality).
//
// Persistent, warp-specialised kernel: one CTA per SM walks the work items
// (unit = (group, head), in batches of up to 16 members) with three roles
// that run concurrently, so that one unit's selection overlaps the next
// unit's gather and MMAs:
//  * producers (warps 0-2) fetch the unit's candidate row with one bulk copy
//    and gather the candidate keys 128 rows per chunk with 16-byte cp.async
//    into the 128-byte-swizzled K-major layout (plus the member queries as the
//    B operand); each thread's arrival on the stage's mbarrier fires once its
//    copies have landed;
//  * the MMA warp (warp 3) issues tcgen05.mma with M = 128 candidate rows,
//    N = 16 member queries, K = d, into TMEM columns [16c, 16c+16) for chunk
//    c, and signals "chunk c scored" on a per-chunk mbarrier;
//  * the select warps (4-19, four per TMEM lane quarter; group grp of four
//    warps owns members 4grp..4grp+3) select every member's exact top-k and
//    write the rows.
// Chunk c's MMA row r holds candidate t = r*nch + c, so TMEM lane r owns the
// contiguous, ascending candidates [r*nch, r*nch + nch).  With Kc <= 4096 a
// unit's scores (4096 x 16 fp32 = 256 KB) fill TMEM; the select warps read
// each chunk's columns once and give them back at once, so the MMA warp can
// write the next unit into them while this unit is still being selected.
//
// Selection (exact, on 32-bit order keys, ties to the lower index), in one
// pass over the scores:
//  * a member with at most kCap usable candidates sends all of them to its
//    boundary list;
//  * otherwise the first kSample chunks (a stride sample of the candidate
//    set, since chunk c holds every nch-th candidate) give an interval
//    [lo, hi) that holds the member's k-th score with overwhelming
//    probability: a histogram linear in the score over chunk 0's range, and
//    sample ranks kZ standard deviations on either side of the expected one;
//  * one pass over all chunks marks candidates >= hi in per-thread bit masks
//    and appends those in [lo, hi) to the member's list, and gives each
//    chunk's TMEM columns back as soon as it is read;
//  * the list is ranked exactly (a warp radix select: the need-th largest key
//    and how many of its copies are taken, ties in candidate order), and its
//    decisions go to a per-member bitmap;
//  * one group scan gives every thread its output slots; each warp stages its
//    slice of an output row in shared memory and writes it coalesced.
// A member whose k-th score fell outside its interval, whose list overflowed,
// or whose sample had no score range is not written here: it is recorded in a
// miss list and refine_fallback_kernel redoes it exactly afterwards.
#pragma once

#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

struct RefineParams {
  const uint16_t* q;      // prefill [L][H][d]; decode [B][g][H][d]
  const uint16_t* keys;   // prefill [L][H][d]; decode packed cache [rows][H][d]
  const int32_t* cand;    // [H][G][cand_row_words(Kc)] candidate rows in read order (ptx.cuh)
  int32_t* out;           // prefill [L][H][top_k]; decode [B][g][H][top_k]
  float* out_scores;      // same shape as out, or null
  const int32_t* cu;      // decode: [B+1] cache row offsets; null for prefill
  int G, L, H, g, top_k, Kc, d;
  int max_seqlen;         // decode: sequences with more cache rows (or fewer than g) are skipped
  int n_items;            // H * G units x member batches
  int nbatch;             // member batches of up to 16 per unit
  uint32_t tmem_cols;
  int2* miss_list;        // (item, member within the item) for refine_fallback_kernel
  int* miss_count;        // zeroed before the launch
  int miss_cap;
  int* status;
};

// member selection modes
enum : int {
  kMNone = 0,   // takes nothing (no usable candidate)
  kMAll = 1,    // takes every usable candidate (top_k >= usable count)
  kMList = 2,   // few usable candidates: all of them go to the list
  kMBand = 3,   // sampled interval: >= hi taken, [lo, hi) to the list
  kMMiss = 4,   // redone by refine_fallback_kernel
};

constexpr int kBins = 512;          // sample histogram bins per member
// 2^23: a float in [2^23, 2^24) is an integer, held in its low mantissa bits
constexpr float kMagic = 8388608.0f;
constexpr int kCap = 512;           // boundary list entries per member
constexpr int kSample = 16;         // sampled chunks
constexpr float kZ = 4.0f;          // interval half-width, in standard deviations of the sample rank

struct MemberSel {
  int nv;           // usable candidates: the ascending prefix with j < pos
  int K;            // min(top_k, nv)
  int mode;
  int nlist;        // list entries appended (may exceed kCap: overflow)
  int nabove;       // candidates >= hi
  int nsamp;        // usable sampled scores
  float lo, hi;     // list interval [lo, hi); hi = +inf: no "above" region
  uint32_t kmin, kmax;  // chunk 0's usable score range as order keys
  uint32_t tk, tmask;   // list rule: (key & tmask) > tk, or == tk and among the first need_eq
  int need_eq;
};

struct RefineMisc {
  MemberSel ms[16];
  int gscan[4][4][4];
  uint64_t full[4], empty[4], cready[2], cfree[2], drain;
  uint64_t tready[32], tfree[32];
  uint32_t tmem_slot;
  int abort_flag;
};

template <int D>
struct RefineCfg {
  static constexpr int NPROD = 96;                      // producer threads (warps 0-2)
  static constexpr int MMA_WARP = 3;
  static constexpr int SEL_WARP0 = 4;                   // select warps 4-19
  static constexpr int NSEL = 512;
  static constexpr int NT = 640;
  static constexpr int NS = 3;                          // gather stages
  static constexpr int KATOMS = D / 64;
  static constexpr int ATOM_A = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int STAGE = KATOMS * ATOM_A;
  static constexpr int ATOM_B = 16 * 128;               // 16 member rows x 128 bytes
  static constexpr int B_BYTES = ((KATOMS * ATOM_B + 1023) / 1024) * 1024;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = NS * STAGE;              // two B buffers (item parity)
  static constexpr int OFF_C = OFF_B + 2 * B_BYTES;     // two candidate lists
  // per member kBins 32-bit words: the sample histogram; later the list's
  // 256-bin radix histogram (words 0..255) and the decision bitmap (words
  // 256..383, one bit per candidate)
  static constexpr int HIST_BYTES = 16 * kBins * 4;
  static constexpr int LK_BYTES = 16 * kCap * 4;        // list keys
  static constexpr int LT_BYTES = 16 * kCap * 2;        // list candidate slots
  // output staging entries per select warp: the list bytes, once ranked
  static constexpr int STGE = (LK_BYTES + LT_BYTES) / 4 / 16;
  __host__ __device__ static int nch_max(int Kc) { return (Kc + 127) / 128; }
  __host__ __device__ static int cidx_words(int Kc) { return nch_max(Kc) * 128; }
  __host__ __device__ static int off_hist(int Kc) { return OFF_C + 2 * cidx_words(Kc) * 4; }
  static int smem_bytes(int Kc) {
    return off_hist(Kc) + HIST_BYTES + LK_BYTES + LT_BYTES + static_cast<int>(sizeof(RefineMisc)) + 1024;
  }
  static_assert(kBins >= 256 + 128, "radix histogram and bitmap fit a member's histogram words");
};

// Linear bin of a score, round(s * scale + off) clamped to [0, kBins-1], with
// offm = off + 2^23 (as a float): the fma rounds s*scale + offm to an integer
// in [2^23, 2^23 + kBins-1] after the clamps, and the bin is its low mantissa
// bits.  One rounding of a function increasing in s, then monotone clamps, so
// the bins are ordered like the scores, and -0 and +0 share a bin.
__device__ __forceinline__ int value_bin(float s, float scale, float offm) {
  const float t = fminf(fmaxf(__fmaf_rn(s, scale, offm), kMagic), kMagic + static_cast<float>(kBins - 1));
  return static_cast<int>(__float_as_uint(t) & static_cast<uint32_t>(kBins - 1));
}

// Bin of an order key; key patterns beyond the infinities (no score has them)
// clamp to the infinities.
__device__ __forceinline__ int bin_of_key(uint32_t key, float scale, float offm) {
  const uint32_t kc = min(max(key, 0x007FFFFFu), 0xFF800000u);
  return value_bin(key_score(kc), scale, offm);
}

// Smallest order key whose bin is >= b (1 <= b <= kBins-1), found by the whole
// warp (every key reaches the top bin at +inf).  A 32-key probe around the
// bin's nominal edge usually brackets it; otherwise a 32-way search over all
// keys does.
__device__ __forceinline__ uint32_t warp_first_key_of_bin(int b, float scale, float offm, int lane) {
  // the score where round(s * scale + offm) reaches 2^23 + b
  const uint32_t guess = score_key(static_cast<float>(
      (static_cast<double>(kMagic) + b - 0.5 - static_cast<double>(offm)) / static_cast<double>(scale)));
  const long long p0 = static_cast<long long>(guess) - 16;
  const long long pk = min(max(p0 + lane, 0ll), 4294967295ll);
  const unsigned ge = __ballot_sync(0xffffffffu, bin_of_key(static_cast<uint32_t>(pk), scale, offm) >= b);
  if ((ge & 1u) == 0u && (ge >> 31) != 0u && p0 >= 0 && p0 + 31 <= 4294967295ll)
    return static_cast<uint32_t>(p0 + __ffs(ge) - 1);
  unsigned long long base = 0, span = 1ull << 32;
  while (span > 1) {
    const unsigned long long stride = (span + 31) / 32;
    const unsigned long long first = base + static_cast<unsigned long long>(lane) * stride;
    bool g = true;  // empty sub-ranges count as "beyond"
    if (first < base + span) {
      const unsigned long long last = min(first + stride, base + span) - 1;
      g = bin_of_key(static_cast<uint32_t>(last), scale, offm) >= b;
    }
    const int j = __ffs(__ballot_sync(0xffffffffu, g)) - 1;
    const unsigned long long nb = base + static_cast<unsigned long long>(j) * stride;
    span = min(stride, base + span - nb);
    base = nb;
  }
  return static_cast<uint32_t>(base);
}

// The bin that holds the r-th largest of the counts in h[0..nbins) (1 <= r <=
// total), found by the whole warp: the largest b with sum(h[b..]) >= r.  Lane
// l sums the nbins/32 bins just below nbins - (nbins/32)*l.  *above receives
// sum(h[b+1..]).
template <int NBINS>
__device__ __forceinline__ int warp_rank_bin(const uint32_t* h, int r, int lane, int* above) {
  constexpr int PER = NBINS / 32;
  const int b0 = NBINS - PER * (lane + 1);
  int s = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) s += static_cast<int>(h[b0 + i]);
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= r);
  const int L = hit ? __ffs(hit) - 1 : 31;
  int cum = __shfl_sync(0xffffffffu, incl - s, L);
  int bin = NBINS - PER * L - PER;  // (the counts always reach r)
  const int bL = NBINS - PER * (L + 1);
  for (int i = PER - 1; i >= 0; --i) {
    const int c = static_cast<int>(h[bL + i]);
    if (cum + c >= r) {
      bin = bL + i;
      break;
    }
    cum += c;
  }
  *above = cum;
  return bin;
}

// One work item: a unit's batch of up to 16 members.
struct RefineItem {
  int h, u, mb, nb, pos0, nc, nch;
  int jlim;             // candidate key indices lie in [0, jlim): the scan's bound
  long long key_row0;   // cache row of key index 0
  long long qrow0;      // row (before *H) of member 0's query and output
};

__device__ __forceinline__ RefineItem refine_item(const RefineParams& p, int item) {
  RefineItem it;
  const int ui = item / p.nbatch;
  it.mb = (item - ui * p.nbatch) * 16;
  it.h = ui / p.G;
  it.u = ui - it.h * p.G;
  int nm;
  if (p.cu == nullptr) {
    const int s = it.u * p.g;
    nm = min(s + p.g, p.L) - s;
    it.pos0 = s;
    it.key_row0 = 0;
    it.qrow0 = s;
  } else {
    nm = p.g;
    it.key_row0 = p.cu[it.u];
    const int len = p.cu[it.u + 1] - p.cu[it.u];
    it.pos0 = len - p.g;
    it.qrow0 = static_cast<long long>(it.u) * p.g;
    if (len > p.max_seqlen || it.pos0 < 0) {
      // A sequence the decode scan skipped (longer than max_seqlen, or
      // shorter than one step) has no candidate row: its members get
      // empty rows and no key is read.
      it.nb = min(16, nm - it.mb);
      it.nc = 0;
      it.nch = 0;
      it.jlim = 0;
      return it;
    }
  }
  it.nb = min(16, nm - it.mb);
  const int last = it.pos0 + nm - 1;
  it.nc = min(p.Kc, max(last, 0));
  it.nch = (it.nc + 127) / 128;
  it.jlim = max(last, 0);
  return it;
}

// candidate t = r*nch + c of a list lives at word c*128 + ((r + c) & 127):
// conflict-free both along a chunk (fixed c) and along a thread's block (fixed r)
__device__ __forceinline__ int cidx_pos(int c, int r) { return c * 128 + ((r + c) & 127); }

template <int D>
__global__ void __launch_bounds__(640, 1) refine_kernel(RefineParams p) {
  using C = RefineCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  const int NCH = C::nch_max(p.Kc);
  const int CW = C::cidx_words(p.Kc);
  int32_t* cidx0 = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::off_hist(p.Kc));
  uint32_t* lkeys = hist + C::HIST_BYTES / 4;                                   // [16][kCap]
  uint16_t* lslot = reinterpret_cast<uint16_t*>(lkeys + C::LK_BYTES / 4);       // [16][kCap]
  RefineMisc* M = reinterpret_cast<RefineMisc*>(lslot + C::LT_BYTES / 2);
  volatile int* abort_flag = &M->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(smem_u32(&M->full[s]), C::NPROD);
      mbar_init(smem_u32(&M->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&M->cready[b]), 1);
      mbar_init(smem_u32(&M->cfree[b]), C::NSEL / 32);
    }
    for (int c = 0; c < 32; ++c) {
      mbar_init(smem_u32(&M->tready[c]), 1);
      mbar_init(smem_u32(&M->tfree[c]), C::NSEL / 32);
    }
    mbar_init(smem_u32(&M->drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(&M->tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M->tmem_slot;

  if (warp < C::MMA_WARP) {
    // ======================================================== producers
    // Thread 0 fetches each unit's candidate row (stored in this kernel's
    // read order) with one bulk copy; then all 96 producer threads gather the
    // candidate key rows of each chunk with 16-byte cp.async into the
    // 128-byte-swizzled K-major layout, and each thread's arrival on the
    // stage's "full" barrier fires once its own copies have landed, so no
    // producer ever waits for a copy before issuing the next chunk.
    const int pt = tid;
    int sseq = 0;     // chunks issued so far (all items)
    int kk = 0;       // items processed so far
    bool ok = true;
    constexpr int RSTEP = C::NPROD / 8;
    const int p8 = pt & 7, rr0 = pt >> 3;   // 16-byte piece p8 (of each K atom) of rows rr0, rr0 + RSTEP, ...
    const long long rowstride = static_cast<long long>(p.H) * D;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const RefineItem it = refine_item(p, item);
      if (it.nb <= 0) continue;
      const int buf = kk & 1;
      const int32_t* cx = cidx0 + buf * CW;
      const uint32_t cbar = smem_u32(&M->cready[buf]);
      // the list and B buffers of this parity are free once the select warps
      // are done with the item two back
      if (kk >= 2 && ok && warp == 0)
        ok = mbar_wait(smem_u32(&M->cfree[buf]), ((kk >> 1) - 1) & 1, abort_flag, p.status);
      ok = !named_barrier_or(1, C::NPROD, !ok);
      if (ok && pt == 0) {
        const uint32_t bytes = static_cast<uint32_t>(it.nch) * 128u * 4u;
        mbar_arrive_expect_tx(cbar, bytes);
        if (bytes) bulk_copy_g2s(smem_u32(cx), p.cand + (static_cast<long long>(it.h) * p.G + it.u) * CW, bytes, cbar);
      }
      if (ok) ok = mbar_wait(cbar, (kk >> 1) & 1, abort_flag, p.status);
      const uint16_t* kbase = p.keys + (it.key_row0 * p.H + it.h) * static_cast<long long>(D) + p8 * 8;
      const uint32_t bB = sB + buf * C::B_BYTES;
      for (int c = 0; c < it.nch; ++c) {
        const int s = sseq % C::NS;
        // one warp watches the stage; the others sleep on the named barrier
        if (sseq >= C::NS && ok && warp == 0)
          ok = mbar_wait(smem_u32(&M->empty[s]), ((sseq / C::NS) - 1) & 1, abort_flag, p.status);
        ok = !named_barrier_or(1, C::NPROD, !ok);
        if (ok) {
          const uint32_t dst0 = sA + s * C::STAGE;
          const int32_t* cxc = cx + c * 128;
          for (int rr = rr0; rr < 128; rr += RSTEP) {
            const int j = cxc[(rr + c) & 127];
            // a missing candidate (-1 padding) reads as zeros; so would an
            // index outside the scan's bound, which no candidate row holds
            const bool in = j >= 0 && j < it.jlim;
            const uint16_t* src = kbase + (in ? j : 0) * rowstride;
            const uint32_t dst = dst0 + rr * 128 + ((p8 ^ (rr & 7)) << 4);
            const uint32_t nbytes = in ? 16u : 0u;
#pragma unroll
            for (int a = 0; a < C::KATOMS; ++a) cp_async_16(dst + a * C::ATOM_A, src + a * 64, nbytes);
          }
          if (c == 0) {
            // member queries of this batch -> B operand, zero rows past nb
            for (int id = pt; id < 16 * (D / 8); id += C::NPROD) {
              const int rr = id / (D / 8), piece = id % (D / 8);
              const int a = piece >> 3, q8 = piece & 7;
              const bool real = rr < it.nb;
              const uint16_t* src =
                  p.q + (real ? ((it.qrow0 + it.mb + rr) * p.H + it.h) * static_cast<long long>(D) + piece * 8 : 0);
              cp_async_16(bB + a * C::ATOM_B + rr * 128 + ((q8 ^ (rr & 7)) << 4), src, real ? 16u : 0u);
            }
          }
          cp_async_arrive_noinc(smem_u32(&M->full[s]));
        }
        ++sseq;
      }
      ++kk;
      if (named_barrier_or(1, C::NPROD, !ok)) break;
    }
    // never leave the CTA with a copy still landing in its shared memory
    cp_async_wait<0>();
    if (pt == 0)
      for (int q = max(0, kk - 2); q < kk; ++q) mbar_wait_cleanup(smem_u32(&M->cready[q & 1]), (q >> 1) & 1);
  } else if (warp == C::MMA_WARP) {
    // ======================================================== MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16(128, 16);
    int sseq = 0, kk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const RefineItem it = refine_item(p, item);
      if (it.nb <= 0) continue;
      const uint32_t bB = sB + (kk & 1) * C::B_BYTES;
      for (int c = 0; c < NCH && ok; ++c) {
        // the previous item's select warps are done with these columns
        if (kk >= 1) ok = mbar_wait(smem_u32(&M->tfree[c]), (kk - 1) & 1, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && c < it.nch) {
          const int s = sseq % C::NS;
          ok = mbar_wait(smem_u32(&M->full[s]), (sseq / C::NS) & 1, abort_flag, p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (ok && lane == 0) {
            tc_fence_after();
            // the stage was written by other threads' cp.async (generic proxy)
            // and is read by the MMAs (async proxy)
            fence_proxy_async_smem();
#pragma unroll
            for (int kq = 0; kq < D / 16; ++kq) {
              const int a = kq >> 2, k4 = kq & 3;
              const uint64_t adesc = sw128_kmajor_desc(sA + s * C::STAGE + a * C::ATOM_A + k4 * 32);
              const uint64_t bdesc = sw128_kmajor_desc(bB + a * C::ATOM_B + k4 * 32);
              umma_bf16(tmem + c * 16, adesc, bdesc, idesc, kq > 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(&M->empty[s]));
          }
          ++sseq;
        }
        if (ok && lane == 0) umma_commit(smem_u32(&M->tready[c]));
        __syncwarp();
      }
      ++kk;
    }
    // every MMA issued has finished before TMEM can be freed
    if (lane == 0) {
      umma_commit(smem_u32(&M->drain));
      mbar_wait_cleanup(smem_u32(&M->drain), 0);
    }
    __syncwarp();
  } else {
    // ======================================================== select
    const int sw = warp - C::SEL_WARP0;   // 0..15: also the member whose list this warp ranks
    const int grp = sw >> 2;              // member group: members 4grp..4grp+3
    const int quarter = warp & 3;         // TMEM lane quarter
    const int r = quarter * 32 + lane;    // this thread's candidate block
    const int stid = sw * 32 + lane;      // 0..511
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 4 * grp;
    const float kInf = __int_as_float(0x7f800000);
    auto sel_sync = [&]() { named_barrier(2, C::NSEL); };
    int kk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const RefineItem it = refine_item(p, item);
      if (it.nb <= 0) continue;
      const int buf = kk & 1;
      const int nch = it.nch, nb = it.nb;
      const int32_t* cx = cidx0 + buf * CW;
      if (ok) ok = mbar_wait(smem_u32(&M->cready[buf]), (kk >> 1) & 1, abort_flag, p.status);
      // ---- per-member usable counts (the candidate set is ascending) and modes
      if (stid < 16 && ok) {
        MemberSel& S = M->ms[stid];
        int nv = 0;
        if (stid < nb) {
          const int pos = it.pos0 + it.mb + stid;
          int lo = 0, hi = it.nc;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            const int rr = mid / nch;
            if (cx[cidx_pos(mid - rr * nch, rr)] < pos) lo = mid + 1;
            else hi = mid;
          }
          nv = lo;
        }
        const int K = min(p.top_k, nv);
        S.nv = nv;
        S.K = K;
        S.mode = K == 0 ? kMNone : (K == nv ? kMAll : (nv <= kCap ? kMList : kMBand));
        S.nlist = 0;
        S.nabove = 0;
        S.nsamp = 0;
        S.lo = -kInf;
        S.hi = kInf;
        S.kmin = 0xFFFFFFFFu;
        S.kmax = 0u;
        S.tk = 0u;
        S.tmask = 0u;
        S.need_eq = 0x7FFFFFFF;
      }
      for (int i = stid; i < C::HIST_BYTES / 16; i += C::NSEL) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
      if (named_barrier_or(2, C::NSEL, !ok)) break;

      // this thread's view of its four members (member 4*grp + i)
      uint32_t um[4];       // usable chunks of this thread's block (a low-bit prefix)
      uint32_t bandm = 0;   // this group's members with a sampled interval
      bool anyb = false;    // the item has such a member (uniform)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const MemberSel& S = M->ms[4 * grp + i];
        const int nvt = min(max(S.nv - r * nch, 0), nch);
        um[i] = nvt >= 32 ? 0xFFFFFFFFu : ((1u << nvt) - 1u);
        bandm |= (S.mode == kMBand ? 1u : 0u) << i;
      }
      for (int m = 0; m < 16; ++m) anyb |= M->ms[m].mode == kMBand;
      const int s_ch = min(nch, kSample);

      // ---- sample: chunk 0's score range, then a histogram of the first s_ch chunks
      if (anyb) {
        if (ok) ok = mbar_wait(smem_u32(&M->tready[0]), kk & 1, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && bandm != 0u) {
          tc_fence_after();
          uint32_t v[4];
          tmem_ld_32x32b_x4(tl, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reg_fence(v[i]);
            const bool use = ((bandm >> i) & um[i] & 1u) != 0u;
            const uint32_t key = score_key(__uint_as_float(v[i]));
            const uint32_t mn = __reduce_min_sync(0xffffffffu, use ? key : 0xFFFFFFFFu);
            const uint32_t mx = __reduce_max_sync(0xffffffffu, use ? key : 0u);
            if (lane == 0 && ((bandm >> i) & 1u)) {
              red_shared_min(smem_u32(&M->ms[4 * grp + i].kmin), mn);
              red_shared_max(smem_u32(&M->ms[4 * grp + i].kmax), mx);
            }
          }
        }
        sel_sync();
        // bins linear in the score over chunk 0's range (every thread for its
        // members, the same values in all warps of a group)
        float sc4[4], of4[4];
        uint32_t vm = 0;   // members with a usable score range
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const MemberSel& S = M->ms[4 * grp + i];
          const float vmin = key_score(S.kmin), vmax = key_score(S.kmax);
          sc4[i] = __fdiv_rn(static_cast<float>(kBins), __fsub_rn(vmax, vmin));
          of4[i] = __fadd_rn(__fmul_rn(-vmin, sc4[i]), kMagic);
          const bool good = ((bandm >> i) & 1u) && S.kmin < S.kmax && isfinite(vmin) && isfinite(vmax) &&
                            isfinite(sc4[i]) && sc4[i] > 0.f && isfinite(of4[i]);
          vm |= (good ? 1u : 0u) << i;
        }
        uint32_t hrow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) hrow[i] = smem_u32(hist + (4 * grp + i) * kBins);
        int ns[4] = {0, 0, 0, 0};
        for (int c = 0; c < s_ch; ++c) {
          if (c > 0) {
            if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
          }
          if (ok && vm != 0u) {
            tc_fence_after();
            uint32_t v[4];
            tmem_ld_32x32b_x4(tl + c * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              reg_fence(v[i]);
              if (((vm >> i) & (um[i] >> c) & 1u) != 0u) {
                red_shared_add(hrow[i] + 4u * value_bin(__uint_as_float(v[i]), sc4[i], of4[i]), 1u);
                ++ns[i];
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if ((vm >> i) & 1u) {
            const int s = __reduce_add_sync(0xffffffffu, ns[i]);
            if (lane == 0) atom_shared_add(smem_u32(&M->ms[4 * grp + i].nsamp), static_cast<uint32_t>(s));
          }
        }
        if (named_barrier_or(2, C::NSEL, !ok)) break;
        // warp sw: member sw's interval from its sample -- sample ranks kZ
        // standard deviations either side of the expected rank of the k-th
        // score (hypergeometric: the sample is drawn without replacement)
        if (sw < nb && M->ms[sw].mode == kMBand) {
          MemberSel& S = M->ms[sw];
          const float vmin = key_score(S.kmin), vmax = key_score(S.kmax);
          const float vsc = __fdiv_rn(static_cast<float>(kBins), __fsub_rn(vmax, vmin));
          const float voff = __fadd_rn(__fmul_rn(-vmin, vsc), kMagic);
          const bool good = S.kmin < S.kmax && isfinite(vmin) && isfinite(vmax) && isfinite(vsc) && vsc > 0.f &&
                            isfinite(voff);
          if (!good) {
            if (lane == 0) S.mode = kMMiss;
          } else {
            const int n_s = S.nsamp;
            const float pk = static_cast<float>(S.K) / static_cast<float>(S.nv);
            const float e = pk * static_cast<float>(n_s);
            const float fpc = fmaxf(0.f, 1.f - static_cast<float>(n_s) / static_cast<float>(S.nv));
            const float dlt = kZ * sqrtf(static_cast<float>(n_s) * pk * (1.f - pk) * fpc) + 2.f;
            const int r_hi = static_cast<int>(floorf(e - dlt));
            const int r_lo = static_cast<int>(ceilf(e + dlt));
            const uint32_t* hm = hist + sw * kBins;
            float hi = kInf, lo = -kInf;
            int ab;
            if (r_hi >= 1) {
              // above = bins over the one holding the r_hi-th largest sample
              const int b = warp_rank_bin<kBins>(hm, r_hi, lane, &ab);
              if (b < kBins - 1) hi = key_score(warp_first_key_of_bin(b + 1, vsc, voff, lane));
            }
            if (r_lo <= n_s) {
              // list = down to the bin holding the r_lo-th largest sample
              const int b = warp_rank_bin<kBins>(hm, r_lo, lane, &ab);
              if (b > 0) lo = key_score(warp_first_key_of_bin(b, vsc, voff, lane));
            }
            if (lane == 0) {
              S.lo = lo;
              S.hi = hi;
            }
          }
          __syncwarp();
        }
        sel_sync();
      }

      // ---- one pass: candidates >= hi to the per-thread masks, [lo, hi) to
      //      the member's list; each batch of chunks is given back at once
      //      (unless the scores are written out, which reads them again)
      const bool keep_tmem = p.out_scores != nullptr;
      float th4[4], tl4[4];
      uint32_t cm[4];            // chunks to classify, per member
      uint32_t gt[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const MemberSel& S = M->ms[4 * grp + i];
        cm[i] = (S.mode == kMList || S.mode == kMBand) ? um[i] : 0u;
        th4[i] = S.hi;
        tl4[i] = S.lo;
      }
      const uint32_t anyc = __reduce_or_sync(0xffffffffu, cm[0] | cm[1] | cm[2] | cm[3]);
      const int waited = anyb ? s_ch : 0;   // chunks whose "scored" barrier the sample already took
      int released = 0;                     // chunks whose TMEM columns this warp has given back
      auto release_upto = [&](int upto) {
        if (upto <= released) return;
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int c = released; c < upto; ++c) mbar_arrive(smem_u32(&M->tfree[c]));
        released = upto;
      };
#pragma unroll 1
      for (int cb = 0; cb < nch; cb += 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = cb + j;
          if (c < nch && c >= waited && ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (((anyc >> cb) & 15u) != 0u) {
          tc_fence_after();
          uint32_t v[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (cb + j < nch) tmem_ld_32x32b_x4(tl + (cb + j) * 16, v[j]);
          tmem_ld_wait();
          uint32_t lb[4] = {0u, 0u, 0u, 0u};   // this batch's list entries (bit j: chunk cb + j)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = cb + j;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              reg_fence(v[j][i]);
              const float f = __uint_as_float(v[j][i]);
              const uint32_t in = c < nch ? (cm[i] >> c) & 1u : 0u;
              const uint32_t above = f >= th4[i] ? in : 0u;
              const uint32_t inlist = f >= tl4[i] ? in : 0u;
              gt[i] |= above << c;
              lb[i] |= (inlist & ~above) << j;
            }
          }
          // append to the lists: one shared atomic per warp and member
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (__any_sync(0xffffffffu, lb[i] != 0u)) {
              const int m = 4 * grp + i;
              const int cnt = __popc(lb[i]);
              int incl = cnt;
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
              }
              int base = 0;
              if (lane == 31) base = static_cast<int>(atom_shared_add(smem_u32(&M->ms[m].nlist), static_cast<uint32_t>(incl)));
              base = __shfl_sync(0xffffffffu, base, 31);
              int at = base + incl - cnt;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if ((lb[i] >> j) & 1u) {
                  if (at < kCap) {
                    lkeys[m * kCap + at] = score_key(__uint_as_float(v[j][i]));
                    lslot[m * kCap + at] = static_cast<uint16_t>(r * nch + cb + j);
                  }
                  ++at;
                }
              }
            }
          }
        }
        if (!keep_tmem) release_upto(min(cb + 4, nch));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = __reduce_add_sync(0xffffffffu, __popc(gt[i]));
        if (lane == 0 && n > 0) atom_shared_add(smem_u32(&M->ms[4 * grp + i].nabove), static_cast<uint32_t>(n));
      }
      if (named_barrier_or(2, C::NSEL, !ok)) break;

      // ---- warp sw ranks member sw's list exactly: the need-th largest key
      //      (radix select from the highest bit that varies) and how many of
      //      its copies are taken; decisions to the member's bitmap
      if (sw < nb) {
        MemberSel& S = M->ms[sw];
        int mode = S.mode;
        if (mode == kMList || mode == kMBand) {
          const int n = S.nlist, need = S.K - S.nabove;
          if (n > kCap || need < 1 || need > n) {
            mode = kMMiss;   // the k-th score fell outside the interval, or the list overflowed
          } else {
            const uint32_t* lk = lkeys + sw * kCap;
            const uint16_t* ls = lslot + sw * kCap;
            uint32_t* rh = hist + sw * kBins;   // radix histogram (256 words)
            uint32_t* bs = rh + 256;            // decision bitmap (one bit per candidate slot)
            for (int w = lane; w < 128; w += 32) bs[w] = 0u;
            uint32_t tk = 0u, tmask = 0u;
            int need_eq = 0x7FFFFFFF;
            if (need < n) {
              const uint32_t k0 = lk[0];
              uint32_t diff = 0u;
              for (int e = lane; e < n; e += 32) diff |= lk[e] ^ k0;
              diff = __reduce_or_sync(0xffffffffu, diff);
              int sh = 32 - __clz(diff);   // bits [sh, 32) are common to every key
              tmask = sh >= 32 ? 0u : (0xFFFFFFFFu << sh);
              tk = k0 & tmask;
              int rank = need;             // keys matching tk on tmask still to take
              bool whole = false;
#pragma unroll 1
              while (sh > 0) {
                const int width = min(8, sh);
                sh -= width;
                const uint32_t nbm = (1u << width) - 1u;
                for (int b = lane; b < 256; b += 32) rh[b] = 0u;
                __syncwarp();
                for (int e = lane; e < n; e += 32) {
                  const uint32_t key = lk[e];
                  if ((key & tmask) == tk) red_shared_add(smem_u32(&rh[(key >> sh) & nbm]), 1u);
                }
                __syncwarp();
                int above;
                const int b = warp_rank_bin<256>(rh, rank, lane, &above);
                const int cntb = static_cast<int>(rh[b]);
                __syncwarp();
                tk |= static_cast<uint32_t>(b) << sh;
                tmask |= nbm << sh;
                rank -= above;
                if (cntb == rank) {
                  whole = true;   // every key of the boundary bin is taken
                  break;
                }
              }
              need_eq = whole ? 0x7FFFFFFF : rank;   // else: equal keys, the first `rank` in slot order
            }
            for (int e = lane; e < n; e += 32) {
              const uint32_t mk = lk[e] & tmask;
              bool take = mk > tk;
              if (!take && mk == tk) {
                take = true;
                if (need_eq != 0x7FFFFFFF) {
                  const int t = ls[e];
                  int before = 0;
                  for (int f = 0; f < n; ++f) before += ((lk[f] & tmask) == tk && ls[f] < t) ? 1 : 0;
                  take = before < need_eq;
                }
              }
              if (take) {
                const int t = ls[e];
                red_shared_or(smem_u32(&bs[t >> 5]), 1u << (t & 31));
              }
            }
          }
        }
        if (mode == kMMiss && lane == 0) {
          S.mode = kMMiss;
          const int at = atomicAdd(p.miss_count, 1);
          if (at < p.miss_cap) p.miss_list[at] = make_int2(item, sw);
          else atomicOr(p.status, kStNoConverge);
        }
        __syncwarp();
      }
      sel_sync();

      // ---- rows: each member's taken candidates in ascending order
      auto my_bits = [&](const uint32_t* bm) -> uint32_t {
        if (nch == 0) return 0u;
        const int t0 = r * nch;
        const int w = t0 >> 5, o = t0 & 31;
        uint32_t x = bm[w] >> o;
        if (o != 0 && w + 1 < 128) x |= bm[w + 1] << (32 - o);
        return nch >= 32 ? x : (x & ((1u << nch) - 1u));
      };
      uint32_t selm[4];
      int mode4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * grp + i;
        mode4[i] = M->ms[m].mode;
        selm[i] = 0u;
        if (mode4[i] == kMAll) selm[i] = um[i];
        else if (mode4[i] == kMList || mode4[i] == kMBand) selm[i] = gt[i] | my_bits(hist + m * kBins + 256);
      }
      // group scan (thread order = candidate order) of the four members' counts
      int ex[4];
      {
        int incl[4], own[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) incl[i] = own[i] = __popc(selm[i]);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int y = __shfl_up_sync(0xffffffffu, incl[i], o);
            if (lane >= o) incl[i] += y;
          }
        }
        if (lane == 31) {
#pragma unroll
          for (int i = 0; i < 4; ++i) M->gscan[grp][quarter][i] = incl[i];
        }
        named_barrier(3 + grp, 128);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int off = 0;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) off += (qq < quarter) ? M->gscan[grp][qq][i] : 0;
          ex[i] = off + incl[i] - own[i];
        }
      }
      // the ranked lists' bytes become per-warp output staging (STGE entries
      // a warp); a warp's slice of a row goes out in STGE-entry parts
      constexpr int STGE = C::STGE;
      uint32_t* stg = lkeys + sw * STGE;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * grp + i;
        if (m >= nb || mode4[i] == kMMiss) continue;   // a miss is written by refine_fallback_kernel
        const int K = M->ms[m].K;
        const uint32_t sel = selm[i];
        const int slot = ex[i];
        const int wb = __shfl_sync(0xffffffffu, slot, 0);
        // (the selection takes exactly K; the bound only guards the row)
        const int wc = min(__shfl_sync(0xffffffffu, slot + __popc(sel), 31), K) - wb;
        const long long orow_off = ((it.qrow0 + it.mb + m) * p.H + it.h) * static_cast<long long>(p.top_k);
        int32_t* orow = p.out + orow_off;
        for (int part = 0; part * STGE < wc; ++part) {
          const int plo = part * STGE;
          // this lane's selected candidates that fall in the part [plo, plo + STGE)
          const int o0 = slot - wb - plo;
          uint32_t bits = sel;
          if (o0 < 0) {  // skip the ones staged by an earlier part
            for (int k = 0; k < -o0 && bits; ++k) bits &= bits - 1;
          }
          // two entries an iteration: their index loads overlap
          int o = max(o0, 0);
          while (bits != 0u && o < STGE) {
            const int c1 = __ffs(bits) - 1;
            bits &= bits - 1;
            const bool two = bits != 0u && o + 1 < STGE;
            const int c2 = two ? __ffs(bits) - 1 : c1;
            if (two) bits &= bits - 1;
            const uint32_t v1 = static_cast<uint32_t>(cx[cidx_pos(c1, r)]);
            const uint32_t v2 = static_cast<uint32_t>(cx[cidx_pos(c2, r)]);
            stg[o] = v1;
            if (two) stg[o + 1] = v2;
            o += two ? 2 : 1;
          }
          __syncwarp();
          const int n = min(wc - plo, STGE);
#pragma unroll 4
          for (int x = lane; x < n; x += 32) orow[wb + plo + x] = static_cast<int32_t>(stg[x]);
          __syncwarp();
        }
        if (p.out_scores) {
          float* srow = p.out_scores + orow_off;
          const uint32_t any = __reduce_or_sync(0xffffffffu, sel);
          for (int part = 0; part * STGE < wc; ++part) {
            const int plo = part * STGE;
            int o = slot - wb - plo;
            for (uint32_t a = any; a; a &= a - 1) {
              const int c = __ffs(a) - 1;
              uint32_t v;
              tmem_ld_32x32b_x1(tl + c * 16 + i, v);
              tmem_ld_wait();
              if ((sel >> c) & 1u) {
                if (o >= 0 && o < STGE) stg[o] = v;
                ++o;
              }
            }
            __syncwarp();
            const int n = min(wc - plo, STGE);
            for (int x = lane; x < n; x += 32) srow[wb + plo + x] = __uint_as_float(stg[x]);
            __syncwarp();
          }
          for (int x = K + r; x < p.top_k; x += 128) srow[x] = __int_as_float(0x7fc00000);
        }
        for (int x = K + r; x < p.top_k; x += 128) orow[x] = -1;
      }
      // Chunks past this item's list got their "scored" commit without MMAs.
      // Wait for those commits too before giving the chunks back: every
      // release then answers a commit of this item, and the MMA warp can never
      // find a chunk's "free" barrier two phases ahead of its wait.
      for (int c = nch; c < NCH; ++c)
        if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      // this item's TMEM columns and candidate list are free
      if (ok) release_upto(NCH);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&M->cfree[buf]));
      ++kk;
      if (named_barrier_or(2, C::NSEL, !ok)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

constexpr int kRfbNT = 512;

// Exact path for the members the one-pass select could not settle: re-score
// the member's usable candidates on CUDA cores (bf16 query times bf16 keys,
// fp32 accumulation) and select from all of them.  Dynamic shared memory:
// 2 * cand_row_words(Kc) + 2 * top_k words.
template <int D>
__global__ void __launch_bounds__(kRfbNT) refine_fallback_kernel(RefineParams p) {
  __shared__ SelectSmem<kRfbNT> sm;
  __shared__ float qv[D];
  __shared__ int nv_s;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int KW = cand_row_words(p.Kc);
  int32_t* cl = reinterpret_cast<int32_t*>(smem_raw);     // candidates, ascending
  uint32_t* sc = reinterpret_cast<uint32_t*>(cl + KW);     // their scores as order keys
  int32_t* sel = reinterpret_cast<int32_t*>(sc + KW);
  uint32_t* selk = reinterpret_cast<uint32_t*>(sel + p.top_k);
  const int total = min(*p.miss_count, p.miss_cap);
  if (blockIdx.x == 0 && threadIdx.x == 0 && total > 0) atomicOr(p.status, kStFallback);
  const long long rowstride = static_cast<long long>(p.H) * D;
  for (int w = blockIdx.x; w < total; w += gridDim.x) {
    const int2 e = p.miss_list[w];
    const RefineItem it = refine_item(p, e.x);
    const int m = it.mb + e.y;
    const int pos = it.pos0 + m;
    const int32_t* row = p.cand + (static_cast<long long>(it.h) * p.G + it.u) * KW;
    const long long qrow = (it.qrow0 + m) * p.H + it.h;
    __syncthreads();
    for (int t = threadIdx.x; t < it.nc; t += kRfbNT) cl[t] = row[cand_word(t, it.nch)];
    for (int c = threadIdx.x; c < D; c += kRfbNT) qv[c] = __uint_as_float(static_cast<uint32_t>(p.q[qrow * D + c]) << 16);
    __syncthreads();
    if (threadIdx.x == 0) {
      int lo = 0, hi = it.nc;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cl[mid] < pos) lo = mid + 1;
        else hi = mid;
      }
      nv_s = lo;
    }
    __syncthreads();
    const int nv = nv_s;
    const int K = min(p.top_k, nv);
    const uint16_t* kb = p.keys + (it.key_row0 * p.H + it.h) * static_cast<long long>(D);
    for (int t = threadIdx.x; t < nv; t += kRfbNT) {
      const int j = cl[t];
      float acc = 0.f;
      if (j >= 0 && j < it.jlim) {
        const uint4* kr = reinterpret_cast<const uint4*>(kb + j * rowstride);
#pragma unroll 4
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint4 u = kr[c8];
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            acc = fmaf(qv[c8 * 8 + 2 * k], __uint_as_float(w4[k] << 16), acc);
            acc = fmaf(qv[c8 * 8 + 2 * k + 1], __uint_as_float(w4[k] & 0xFFFF0000u), acc);
          }
        }
      }
      sc[t] = score_key(acc);
    }
    __syncthreads();
    block_select_emit<kRfbNT>(
        nv, K, [&](int x) { return sc[x]; },
        [&](int slot, int x) {
          sel[slot] = cl[x];
          selk[slot] = sc[x];
        },
        sm);
    __syncthreads();
    int32_t* orow = p.out + qrow * p.top_k;
    for (int t = threadIdx.x; t < p.top_k; t += kRfbNT) orow[t] = t < K ? sel[t] : -1;
    if (p.out_scores) {
      float* srow = p.out_scores + qrow * p.top_k;
      for (int t = threadIdx.x; t < p.top_k; t += kRfbNT)
        srow[t] = t < K ? key_score(selk[t]) : __int_as_float(0x7fc00000);
    }
  }
}

}  // namespace pivot
