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
// unit's scores (4096 x 16 fp32 = 256 KB) fill TMEM; the select warps give
// each chunk's columns back as soon as they no longer need them, and the MMA
// warp writes the next unit into them.
//
// Selection (exact, on 32-bit order keys, ties to the lower index):
//  * round 0 follows the MMAs chunk by chunk: chunk 0 is a 128-candidate
//    sample spread over the whole set; its score range sets a 512-bin
//    histogram linear in the score (monotone, clamped at both ends), and
//    every chunk is counted into it as soon as it is scored;
//  * select warp w finds the boundary bin of member w with a two-level scan
//    and inverts the bin function to key thresholds [kl, kh); one pass over
//    the scores marks each candidate "above" (key >= kh) or "boundary" and
//    collects the boundary keys in a shared list, after which the unit's TMEM
//    columns are given back;
//  * a list of up to kListCap keys is ranked exactly (the need-th largest key
//    tk, and how many of its copies are taken) and its decisions go to
//    per-member bitmaps; larger boundaries are narrowed by further key-linear
//    rounds, and a boundary of equal keys takes its first keys in order;
//  * one group scan gives every thread its output slot; each warp stages its
//    slice of an output row in shared memory and writes it coalesced.
#pragma once

#include "ptx.cuh"

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
  int* status;
};

// member selection modes
enum : int {
  kMNone = 0,    // takes nothing (no usable candidate)
  kMAll = 1,     // takes every usable candidate (top_k >= usable count)
  kMSel = 2,     // narrowing: the boundary bin of the current round is open
  kMWhole = 3,   // every key of the boundary bin is taken
  kMList = 4,    // boundary ranked from the shared list
  kMNarrow = 5,  // boundary too large for the list: another round
  kMTies = 6,    // boundary keys all equal: the first need_eq in order
};

constexpr int kRefBins = 512;
// 2^23: a float in [2^23, 2^24) is an integer, held in its low mantissa bits
constexpr float kMagic = 8388608.0f;
constexpr int kListCap = 256;
// Each key-linear round shrinks a boundary's key range by a factor of about
// 256, so 32-bit keys need at most five rounds after round 0.
constexpr int kMaxRounds = 8;

struct MemberSel {
  int nv;           // usable candidates: the ascending prefix with j < pos
  int K;            // min(top_k, nv)
  int mode;
  int active;       // takes part in the current round
  int need;         // keys still to take from the current candidate interval
  int cnt;          // keys in the boundary bin
  uint32_t lo;      // key-linear bins: origin; both: scale; score-linear: offset
  float scale, off;
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
  uint64_t full[4], empty[4], cready[2], cfree[2], drain;
  uint64_t tready[32], tfree[32];
  uint32_t tmem_slot;
  int abort_flag;
  int more;
};

template <int D>
struct RefineCfg {
  static constexpr int NPROD = 96;                      // producer threads (warps 0-2)
  static constexpr int MMA_WARP = 3;
  static constexpr int SEL_WARP0 = 4;                   // select warps 4-19
  static constexpr int NSEL = 512;
  static constexpr int NT = 640;
  static constexpr int NS = 4;                          // gather stages
  static constexpr int KATOMS = D / 64;
  static constexpr int ATOM_A = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int STAGE = KATOMS * ATOM_A;
  static constexpr int ATOM_B = 16 * 128;               // 16 member rows x 128 bytes
  static constexpr int B_BYTES = ((KATOMS * ATOM_B + 1023) / 1024) * 1024;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = NS * STAGE;              // two B buffers (item parity)
  static constexpr int OFF_C = OFF_B + 2 * B_BYTES;     // two candidate lists
  // histograms: 16 members x 512 bins of 32-bit counts; the same bytes later
  // hold the boundary lists, and together with the decision bitmaps that
  // follow them, the per-warp output staging
  static constexpr int HIST_BYTES = 16 * kRefBins * 4;
  static_assert(16 * 2 * kListCap * 4 <= HIST_BYTES, "lists alias the histograms");
  // output staging entries per select warp: the histogram and bitmap bytes
  __host__ __device__ static int stg_entries(int Kc) { return (HIST_BYTES / 4 + 16 * 2 * bm_words(Kc)) / 16; }
  __host__ __device__ static int nch_max(int Kc) { return (Kc + 127) / 128; }
  __host__ __device__ static int cidx_words(int Kc) { return nch_max(Kc) * 128; }
  // list decisions: per member, "above" and "equal" bitmaps over candidates
  __host__ __device__ static int bm_words(int Kc) { return nch_max(Kc) * 4; }
  static int smem_bytes(int Kc) {
    return OFF_C + 2 * cidx_words(Kc) * 4 + HIST_BYTES + 16 * 2 * bm_words(Kc) * 4 +
           static_cast<int>(sizeof(RefineMisc)) + 1024;
  }
};

// Linear bin of an order key over [lo, ...) with `scale` bins per key unit,
// clamped to [0, 511].  Every step is non-decreasing in the key.
__device__ __forceinline__ int key_bin(uint32_t key, uint32_t lo, float scale) {
  const uint32_t dl = key > lo ? key - lo : 0u;
  const uint32_t b = __float2uint_rz(__uint2float_rn(dl) * scale);
  return static_cast<int>(min(b, static_cast<uint32_t>(kRefBins - 1)));
}

// Linear bin of a score, round(s * scale + off) clamped to [0, 511], with
// offm = off + 2^23 (as a float): the fma rounds s*scale + offm to an integer
// in [2^23, 2^23 + 511] after the clamps, and the bin is its low mantissa
// bits.  One rounding of a function increasing in s, then monotone clamps, so
// the bins are ordered like the scores, and -0 and +0 share a bin.  Scores of
// real data spread evenly over such bins, while the order keys of scores on
// both sides of zero crowd into a few of the key-linear ones.
__device__ __forceinline__ int value_bin(float s, float scale, float offm) {
  const float t = fminf(fmaxf(__fmaf_rn(s, scale, offm), kMagic), kMagic + static_cast<float>(kRefBins - 1));
  return static_cast<int>(__float_as_uint(t) & static_cast<uint32_t>(kRefBins - 1));
}

// Bin of an order key under either bin function; key patterns beyond the
// infinities (no score has them) clamp to the infinities.
__device__ __forceinline__ int bin_of_key(uint32_t key, uint32_t lo, float scale, float off, bool vmode) {
  if (!vmode) return key_bin(key, lo, scale);
  const uint32_t kc = min(max(key, 0x007FFFFFu), 0xFF800000u);
  return value_bin(key_score(kc), scale, off);
}

// Smallest key whose bin is >= b (1 <= b <= 511), found by the whole warp;
// false when no key reaches bin b.  A 32-key probe around the bin's nominal
// edge usually brackets it; otherwise a 32-way search over all keys does.
__device__ __forceinline__ bool warp_first_key_of_bin(int b, uint32_t lo, float scale, float off, bool vmode,
                                                      int lane, uint32_t* out) {
  if (bin_of_key(0xFFFFFFFFu, lo, scale, off, vmode) < b) return false;
  uint32_t guess;
  if (vmode) {
    // the score where round(s * scale + offm) reaches 2^23 + b
    guess = score_key(static_cast<float>((static_cast<double>(kMagic) + b - 0.5 - static_cast<double>(off)) /
                                         static_cast<double>(scale)));
  } else {
    const float dk = __fdiv_rn(static_cast<float>(b), scale);
    guess = dk >= 4294967040.0f ? 0xFFFFFFFFu : lo + min(__float2uint_rz(dk), 0xFFFFFFFFu - lo);
  }
  const long long p0 = static_cast<long long>(guess) - 16;
  const long long pk = min(max(p0 + lane, 0ll), 4294967295ll);
  const unsigned ge =
      __ballot_sync(0xffffffffu, bin_of_key(static_cast<uint32_t>(pk), lo, scale, off, vmode) >= b);
  if ((ge & 1u) == 0u && (ge >> 31) != 0u && p0 >= 0 && p0 + 31 <= 4294967295ll) {
    *out = static_cast<uint32_t>(p0 + __ffs(ge) - 1);
    return true;
  }
  unsigned long long base = 0, span = 1ull << 32;
  while (span > 1) {
    const unsigned long long stride = (span + 31) / 32;
    const unsigned long long first = base + static_cast<unsigned long long>(lane) * stride;
    bool g = true;  // empty sub-ranges count as "beyond"
    if (first < base + span) {
      const unsigned long long last = min(first + stride, base + span) - 1;
      g = bin_of_key(static_cast<uint32_t>(last), lo, scale, off, vmode) >= b;
    }
    const int j = __ffs(__ballot_sync(0xffffffffu, g)) - 1;
    const unsigned long long nb = base + static_cast<unsigned long long>(j) * stride;
    span = min(stride, base + span - nb);
    base = nb;
  }
  *out = static_cast<uint32_t>(base);
  return true;
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
  const int BMW = C::bm_words(p.Kc);
  int32_t* cidx0 = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::OFF_C + 2 * CW * 4);
  uint32_t* bmap = hist + C::HIST_BYTES / 4;          // [16][2][BMW]
  RefineMisc* M = reinterpret_cast<RefineMisc*>(bmap + 16 * 2 * BMW);
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
        ok = mbar_wait(smem_u32(&M->cfree[buf]), ((kk >> 1) - 1) & 1, abort_flag, p.status, 256);
      ok = !named_barrier_or(1, C::NPROD, !ok);
      if (ok && pt == 0) {
        const uint32_t bytes = static_cast<uint32_t>(it.nch) * 128u * 4u;
        mbar_arrive_expect_tx(cbar, bytes);
        if (bytes) bulk_copy_g2s(smem_u32(cx), p.cand + (static_cast<long long>(it.h) * p.G + it.u) * CW, bytes, cbar);
      }
      if (ok) ok = mbar_wait(cbar, (kk >> 1) & 1, abort_flag, p.status, 128);
      const uint16_t* kbase = p.keys + (it.key_row0 * p.H + it.h) * static_cast<long long>(D) + p8 * 8;
      const uint32_t bB = sB + buf * C::B_BYTES;
      for (int c = 0; c < it.nch; ++c) {
        const int s = sseq % C::NS;
        // one warp watches the stage; the others sleep on the named barrier
        if (sseq >= C::NS && ok && warp == 0)
          ok = mbar_wait(smem_u32(&M->empty[s]), ((sseq / C::NS) - 1) & 1, abort_flag, p.status, 256);
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
        if (kk >= 1) ok = mbar_wait(smem_u32(&M->tfree[c]), (kk - 1) & 1, abort_flag, p.status, 128);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && c < it.nch) {
          const int s = sseq % C::NS;
          ok = mbar_wait(smem_u32(&M->full[s]), (sseq / C::NS) & 1, abort_flag, p.status, 64);
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
    const int sw = warp - C::SEL_WARP0;   // 0..15: also the member whose bins this warp scans
    const int grp = sw >> 2;              // member group: members 4grp..4grp+3
    const int quarter = warp & 3;         // TMEM lane quarter
    const int r = quarter * 32 + lane;    // this thread's candidate block
    const int stid = sw * 32 + lane;      // 0..511
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 4 * grp;
    auto sel_sync = [&]() { named_barrier(2, C::NSEL); };
    int kk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const RefineItem it = refine_item(p, item);
      if (it.nb <= 0) continue;
      const int buf = kk & 1;
      const int nch = it.nch, nb = it.nb;
      const int32_t* cx = cidx0 + buf * CW;
      if (ok) ok = mbar_wait(smem_u32(&M->cready[buf]), (kk >> 1) & 1, abort_flag, p.status, 256);
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
        S.off = 0.f;
      }
      for (int i = stid; i < C::HIST_BYTES / 16; i += C::NSEL) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
      for (int i = stid; i < 16 * 2 * BMW / 4; i += C::NSEL) reinterpret_cast<uint4*>(bmap)[i] = make_uint4(0, 0, 0, 0);
      if (named_barrier_or(2, C::NSEL, !ok)) break;

      // this thread's view of its four members (member 4*grp + i)
      uint32_t um[4];       // usable chunks of this thread's block (a low-bit prefix)
      uint32_t hm = 0;      // members counted in the round-0 histogram (uniform in the group)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const MemberSel& S = M->ms[4 * grp + i];
        const int nvt = min(max(S.nv - r * nch, 0), nch);
        um[i] = nvt >= 32 ? 0xFFFFFFFFu : ((1u << nvt) - 1u);
        hm |= (S.mode == kMSel ? 1u : 0u) << i;
      }
      uint32_t ob4[4];    // score-linear bins: the offset's bits; key-linear: the origin
      float sc4[4];
      uint32_t vm4 = 0;   // members whose round-0 bins are linear in the score

      auto sample_range = [&]() {
        uint32_t v[4];
        tmem_ld_32x32b_x4(tl, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          reg_fence(v[i]);
          const bool use = ((hm >> i) & um[i] & 1u) != 0u;
          const uint32_t key = score_key(__uint_as_float(v[i]));
          const uint32_t mn = __reduce_min_sync(0xffffffffu, use ? key : 0xFFFFFFFFu);
          const uint32_t mx = __reduce_max_sync(0xffffffffu, use ? key : 0u);
          if (lane == 0) {
            M->pmin[quarter][4 * grp + i] = mn;
            M->pmax[quarter][4 * grp + i] = mx;
          }
        }
      };
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
          const float voff = __fadd_rn(__fmul_rn(-vmin, vsc), kMagic);   // offset + 2^23
          const bool vm = mn < mx && isfinite(vmin) && isfinite(vmax) && isfinite(vsc) && vsc > 0.f && isfinite(voff);
          if (vm) {
            ob4[i] = __float_as_uint(voff);
            sc4[i] = vsc;
            vm4 |= 1u << i;
          } else if (mn > mx) {
            ob4[i] = 0u;
            sc4[i] = 0.f;
          } else {
            ob4[i] = mn;
            sc4[i] = static_cast<float>(kRefBins) / (__uint2float_rn(mx - mn) + 1.0f);
          }
          if (quarter == 0 && lane == 0) {
            M->ms[m].lo = vm ? 0u : ob4[i];
            M->ms[m].off = vm ? voff : 0.f;
            M->ms[m].scale = sc4[i];
            M->ms[m].vmode = vm ? 1 : 0;
          }
        }
      };
      // shared-memory address of this thread's members' histograms
      uint32_t hrow[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hrow[i] = smem_u32(hist + (4 * grp + i) * kRefBins);
      // chunks where all four members count every score of this thread's block
      uint32_t allc = 0;
      auto hist_chunk = [&](int c) {
        uint32_t v[4];
        tmem_ld_32x32b_x4(tl + c * 16, v);
        tmem_ld_wait();
        if ((allc >> c) & 1u) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reg_fence(v[i]);
            const int b = value_bin(__uint_as_float(v[i]), sc4[i], __uint_as_float(ob4[i]));
            red_shared_add(hrow[i] + 4u * b, 1u);
          }
        } else if (vm4 == hm) {  // every counted member has score-linear bins (the rule)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reg_fence(v[i]);
            const bool cnt = ((hm >> i) & (um[i] >> c) & 1u) != 0u;
            const int b = value_bin(__uint_as_float(v[i]), sc4[i], __uint_as_float(ob4[i]));
            if (cnt) red_shared_add(hrow[i] + 4u * b, 1u);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reg_fence(v[i]);
            if (((hm >> i) & (um[i] >> c) & 1u) != 0u) {
              const float f = __uint_as_float(v[i]);
              const int b = ((vm4 >> i) & 1u) ? value_bin(f, sc4[i], __uint_as_float(ob4[i]))
                                              : key_bin(score_key(f), ob4[i], sc4[i]);
              red_shared_add(hrow[i] + 4u * b, 1u);
            }
          }
        }
      };

      // ---- round 0, chunk by chunk as the MMAs finish
      for (int c = 0; c < nch; ++c) {
        if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status, 64);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && hm != 0) {
          tc_fence_after();
          if (c == 0) {
            sample_range();
          } else {
            if (c == 1) {
              set_range();
              allc = (hm == 0xFu && vm4 == 0xFu) ? (um[0] & um[1] & um[2] & um[3]) : 0u;
              hist_chunk(0);
            }
            hist_chunk(c);
          }
        }
        if (c == 0) sel_sync();  // the sample ranges are visible
      }
      if (ok && nch == 1 && hm != 0) {
        set_range();
        allc = (hm == 0xFu && vm4 == 0xFu) ? (um[0] & um[1] & um[2] & um[3]) : 0u;
        hist_chunk(0);
      }
      if (named_barrier_or(2, C::NSEL, !ok)) break;

      // ---- selection rounds
      uint32_t gt[4], bnd[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        gt[i] = M->ms[4 * grp + i].mode == kMAll ? um[i] : 0u;
        bnd[i] = 0u;
      }
      int released = 0;   // chunks whose TMEM columns this warp has given back
      auto release_upto = [&](int upto) {
        if (upto <= released) return;
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int c = released; c < upto; ++c) mbar_arrive(smem_u32(&M->tfree[c]));
        released = upto;
      };
#pragma unroll 1
      for (int round = 0;; ++round) {
        if (round == kMaxRounds) {
          if (stid == 0) atomicOr(p.status, kStNoConverge);
          break;
        }
        // (a) warp sw: boundary bin and key thresholds of member sw
        if (sw < nb && M->ms[sw].active) {
          MemberSel& S = M->ms[sw];
          const uint32_t* hw = hist + sw * kRefBins;
          const int need = S.need;
          // lane l owns bins [512 - 16(l+1), 512 - 16l), in descending order by lane
          const int b0 = kRefBins - 16 * (lane + 1);
          int s = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 x = reinterpret_cast<const uint4*>(hw + b0)[(i + lane) & 3];
            s += static_cast<int>(x.x + x.y + x.z + x.w);
          }
          int incl = s;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          // (the counts always reach need; the clamps only keep indices in range)
          const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
          const int L = hit ? __ffs(hit) - 1 : 31;
          const int exclL = __shfl_sync(0xffffffffu, incl - s, L);
          // lane i < 16: bin 512 - 16L - 1 - i
          const int cb = lane < 16 ? static_cast<int>(hw[kRefBins - 16 * L - 1 - lane]) : 0;
          int incl2 = cb;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl2, o);
            if (lane >= o) incl2 += y;
          }
          const unsigned hit2 = __ballot_sync(0xffffffffu, exclL + incl2 >= need);
          const int i2 = hit2 ? __ffs(hit2) - 1 : 15;
          const int above = __shfl_sync(0xffffffffu, exclL + incl2 - cb, i2);
          const int cntb = __shfl_sync(0xffffffffu, cb, i2);
          const int bstar = kRefBins - 16 * L - 1 - i2;
          const uint32_t lo = S.lo;
          const float sc = S.scale, off = S.off;
          const bool vm = S.vmode != 0;
          uint32_t kl = 0, kh = 0;
          bool has_kl = true, has_kh = false;
          if (bstar > 0) has_kl = warp_first_key_of_bin(bstar, lo, sc, off, vm, lane, &kl);
          if (bstar < kRefBins - 1) has_kh = warp_first_key_of_bin(bstar + 1, lo, sc, off, vm, lane, &kh);
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
          __syncwarp();
        }
        sel_sync();

        // (b) one pass over the scores: above / boundary, boundary lists.  In
        //     round 0 the columns are given back chunk by chunk unless a
        //     boundary needs more rounds or the scores are written out.
        //     key >= K  <=>  score >= key_score(K) (the key order is the score
        //     order, -0 folded onto +0), so the pass compares scores; no upper
        //     edge compares against NaN (never true), no lower edge against -inf.
        bool keep_tmem = p.out_scores != nullptr;
#pragma unroll
        for (int m = 0; m < 16; ++m) keep_tmem |= M->ms[m].active && M->ms[m].mode == kMNarrow;
        uint32_t lst = 0, nar = 0;
        float th4[4], tl4[4];
        uint32_t cand4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const MemberSel& S = M->ms[4 * grp + i];
          const bool a = S.active != 0;
          lst |= (a && S.mode == kMList ? 1u : 0u) << i;
          nar |= (a && S.mode == kMNarrow ? 1u : 0u) << i;
          th4[i] = S.kh_inf ? __int_as_float(0x7fc00000) : key_score(S.kh);
          tl4[i] = S.kl == 0u ? -__int_as_float(0x7f800000) : key_score(S.kl);
          cand4[i] = a ? (round == 0 ? um[i] : bnd[i]) : 0u;
          if (a) bnd[i] = 0u;
        }
        const uint32_t anyc = __reduce_or_sync(0xffffffffu, cand4[0] | cand4[1] | cand4[2] | cand4[3]);
        // common case: every candidate of every lane's block counts for all
        // four members, so the pass needs no per-key candidate test
        const uint32_t fullm = nch >= 32 ? 0xFFFFFFFFu : ((1u << nch) - 1u);
        const bool dense4 = __all_sync(0xffffffffu, (cand4[0] & cand4[1] & cand4[2] & cand4[3]) == fullm);
#pragma unroll 1
        for (int cb = 0; cb < nch; cb += 4) {
          if (((anyc >> cb) & 15u) != 0u) {
            uint32_t v[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (cb + j < nch) tmem_ld_32x32b_x4(tl + (cb + j) * 16, v[j]);
            tmem_ld_wait();
            if (dense4 && cb + 4 <= nch) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t bit = 1u << (cb + j);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  reg_fence(v[j][i]);
                  const float f = __uint_as_float(v[j][i]);
                  if (f >= th4[i]) gt[i] |= bit;
                  else if (f >= tl4[i]) bnd[i] |= bit;
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int c = cb + j;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  reg_fence(v[j][i]);
                  const float f = __uint_as_float(v[j][i]);
                  const uint32_t in = c < nch ? (cand4[i] >> c) & 1u : 0u;
                  const uint32_t hi = f >= th4[i] ? in : 0u;
                  const uint32_t lo = f >= tl4[i] ? in : 0u;
                  gt[i] |= hi << c;
                  bnd[i] |= (lo & ~hi) << c;
                }
              }
            }
            // this batch's boundary keys join their member's list, one
            // shared-memory atomic per warp and member (boundaries are small)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t mine = ((lst >> i) & 1u) ? (bnd[i] >> cb) & 15u : 0u;
              if (mine != 0u) {
                const int m = 4 * grp + i;
                int at = static_cast<int>(atom_shared_add(smem_u32(&M->ms[m].nlist), static_cast<uint32_t>(__popc(mine))));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  if ((mine >> j) & 1u) {
                    if (at < kListCap) {
                      hist[m * 2 * kListCap + at] = score_key(__uint_as_float(v[j][i]));
                      hist[m * 2 * kListCap + kListCap + at] = static_cast<uint32_t>(r * nch + cb + j);
                    }
                    ++at;
                  }
                }
              }
            }
          }
          if (round == 0 && !keep_tmem) release_upto(min(cb + 4, nch));
        }
        // key ranges of the boundaries that need another round (rare)
        if (nar != 0) {
#pragma unroll 1
          for (int c = 0; c < nch; ++c) {
            uint32_t v[4];
            tmem_ld_32x32b_x4(tl + c * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              reg_fence(v[i]);
              const bool in = ((nar >> i) & (bnd[i] >> c) & 1u) != 0u;
              const uint32_t key = score_key(__uint_as_float(v[i]));
              const uint32_t mn = __reduce_min_sync(0xffffffffu, in ? key : 0xFFFFFFFFu);
              const uint32_t mx = __reduce_max_sync(0xffffffffu, in ? key : 0u);
              if (lane == 0 && ((nar >> i) & 1u)) {
                red_shared_min(smem_u32(&M->ms[4 * grp + i].bmin), mn);
                red_shared_max(smem_u32(&M->ms[4 * grp + i].bmax), mx);
              }
            }
          }
        }
        if (stid == 0) M->more = 0;
        sel_sync();

        // (c) warp sw closes member sw's round: rank the list, or detect equal
        //     keys, or set up the next round over the boundary's key range
        if (sw < nb && M->ms[sw].active) {
          MemberSel& S = M->ms[sw];
          const int m = sw;
          const int mode = S.mode;
          const int need = S.need;
          if (mode == kMWhole) {
            if (lane == 0) {
              S.need_eq = 0x7FFFFFFF;
              S.active = 0;
            }
          } else if (mode == kMList) {
            const int n = min(S.nlist, kListCap);
            const uint32_t* lk = hist + m * 2 * kListCap;
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
            // the list's decisions, as bitmaps over candidates
            const uint32_t tk = S.tk;
            uint32_t* bgt = bmap + (m * 2) * BMW;
            uint32_t* beq = bgt + BMW;
            for (int e = lane; e < n; e += 32) {
              const uint32_t ke = lk[e];
              const uint32_t te = lk[kListCap + e];
              if (ke > tk) red_shared_or(smem_u32(&bgt[te >> 5]), 1u << (te & 31));
              else if (ke == tk) red_shared_or(smem_u32(&beq[te >> 5]), 1u << (te & 31));
            }
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
                S.off = 0.f;
                S.vmode = 0;
                S.mode = kMSel;
                M->more = 1;
              }
            }
          }
          __syncwarp();
        }
        sel_sync();
        if (!M->more) break;

        // (d) another histogram round over the open boundaries (rare: more
        //     than kListCap keys in one bin with distinct values)
        for (int i = stid; i < C::HIST_BYTES / 16; i += C::NSEL)
          reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
        sel_sync();
        {
          uint32_t c4[4], lo_[4];
          float sc_[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const MemberSel& S = M->ms[4 * grp + i];
            c4[i] = S.active ? bnd[i] : 0u;
            lo_[i] = S.lo;
            sc_[i] = S.scale;
          }
          const uint32_t anyb = __reduce_or_sync(0xffffffffu, c4[0] | c4[1] | c4[2] | c4[3]);
#pragma unroll 1
          for (int c = 0; c < nch; ++c) {
            if (((anyb >> c) & 1u) == 0u) continue;
            uint32_t v[4];
            tmem_ld_32x32b_x4(tl + c * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              reg_fence(v[i]);
              if ((c4[i] >> c) & 1u) {
                const int b = key_bin(score_key(__uint_as_float(v[i])), lo_[i], sc_[i]);
                red_shared_add(hrow[i] + 4u * b, 1u);
              }
            }
          }
        }
        sel_sync();
      }

      // ---- final rule per member: gt, plus the first need_eq of eq in order
      uint32_t eq[4];
      const int t0 = r * nch;
      auto my_bits = [&](const uint32_t* bm) -> uint32_t {
        if (nch == 0) return 0u;
        const int w = t0 >> 5, o = t0 & 31;
        uint32_t x = bm[w] >> o;
        if (o != 0 && w + 1 < BMW) x |= bm[w + 1] << (32 - o);
        return nch >= 32 ? x : (x & ((1u << nch) - 1u));
      };
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * grp + i;
        const int mode = M->ms[m].mode;
        eq[i] = 0u;
        if (mode == kMWhole || mode == kMTies) {
          eq[i] = bnd[i];
        } else if (mode == kMList) {
          gt[i] |= my_bits(bmap + (m * 2) * BMW);
          eq[i] = my_bits(bmap + (m * 2 + 1) * BMW);
        }
      }
      sel_sync();  // every warp has read its bitmaps: their bytes become staging
      // group scan (thread order = candidate order) of (|gt|, |eq|) for the four members
      int ex[8];
      {
        int incl[8], own[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          own[i] = __popc(gt[i]);
          own[4 + i] = __popc(eq[i]);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) incl[k] = own[k];
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
        named_barrier(3 + grp, 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          int off = 0;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) off += (qq < quarter) ? M->gscan[grp][qq][k] : 0;
          ex[k] = off + incl[k] - own[k];
        }
      }
      // the histogram and bitmap bytes become per-warp output staging (STGE
      // entries a warp); a warp's slice of a row goes out in STGE-entry parts
      const int STGE = C::stg_entries(p.Kc);
      uint32_t* stg = hist + sw * STGE;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * grp + i;
        if (m >= nb) continue;
        const int K = M->ms[m].K, need_eq = M->ms[m].need_eq;
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
        if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status, 64);
      ok = __all_sync(0xffffffffu, ok);
      // this item's TMEM columns and candidate list are free
      release_upto(NCH);
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

}  // namespace pivot
