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
//  * the select warps (4-19) select every member's exact top-k and write the
//    rows.
// Chunk c holds candidates c*128 .. c*128+127 (MMA row r = candidate
// c*128 + r), so TMEM lane quarter q of chunk c holds 32 consecutive
// candidates.  Chunks are scored in the order 0, 2, 4, ..., then 1, 3, 5, ...,
// so that the first ones spread over the whole candidate set.  With
// Kc <= 4096 a unit's scores (4096 x 16 fp32 = 256 KB) fill TMEM; the select
// warps read each chunk's columns once and give them back at once, so the
// MMA warp can write the next unit into them while this unit is still being
// selected.
//
// Selection (exact, on 32-bit order keys, ties to the lower index).  Select
// warp w = 4s + q reads TMEM lane quarter q of the chunks at scoring positions
// s, s+4, s+8, ... (all 16 members of 32 candidates per load) and later ranks
// member w's list and writes member w's bitmap:
//  * chunk 0's score range sets, per member, kBins bins linear in the score;
//    every usable score is counted into its member's histogram as soon as its
//    chunk's MMAs finish, so the counting overlaps the gather;
//  * the bin holding the member's k-th largest score is found exactly: keys
//    in higher bins are taken, the bin's own keys (a few on real scores) form
//    the member's list;
//  * one pass over all chunks classifies 32 candidates of a member with two
//    warp votes: the ">= hi" mask goes straight into the member's selection
//    bitmap (bit t = candidate t), the boundary-bin lanes append their scores
//    to the member's list; each chunk's TMEM columns are given back as soon
//    as they are loaded, so the next unit's MMAs follow this pass closely;
//  * the list is ranked exactly (pairwise when short, else by value bins or
//    a radix select; ties in candidate order) and its decisions are OR-ed into
//    the bitmap;
//  * the member's warp walks its bitmap in candidate order: each 32-bit word
//    gives one coalesced store of its selected key indices.
// A member whose chunk-0 range is empty, or whose boundary bin holds more than
// kCap keys (ties), is not written here: it is recorded in a miss list and
// refine_fallback_kernel redoes it exactly afterwards.
#pragma once

#include "decode_cache.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace pivot {

struct RefineParams {
  const uint16_t* q;      // prefill [L][H][d]; decode [B][g][H][d]
  const uint16_t* keys;   // prefill [L][H][d]; decode packed cache [rows][H][d]
  const int32_t* cand;    // [H][G][cand_row_words(Kc)] candidate rows in read order (ptx.cuh)
  int32_t* out;           // prefill [L][H][top_k]; decode [B][g][H][top_k]
  float* out_scores;      // same shape as out, or null
  CacheIndex ci;          // decode: where each sequence's keys live; all null for prefill
  int G, L, H, g, top_k, Kc, d;
  int max_seqlen;         // decode: sequences with more cache rows (or fewer than g) are skipped
  int n_items;            // H * G units x member batches
  int nbatch;             // member batches of up to 16 per unit
  uint32_t tmem_cols;
  int2* miss_list;        // (item, member within the item) for refine_fallback_kernel
  int* miss_count;        // zeroed before the launch
  int miss_cap;
  int* status;
  unsigned long long wait_ns;   // limit of every bounded wait
};

// member selection modes
enum : int {
  kMNone = 0,   // takes nothing (no usable candidate)
  kMAll = 1,    // takes every usable candidate (top_k >= usable count)
  kMBand = 3,   // a selection: >= hi taken, the boundary bin [lo, hi) ranked
  kMMiss = 4,   // redone by refine_fallback_kernel
};

constexpr int kBins = 1024;         // sample histogram bins per member
// 2^23: a float in [2^23, 2^24) is an integer, held in its low mantissa bits
constexpr float kMagic = 8388608.0f;
constexpr int kCap = 512;           // boundary list entries per member

struct MemberSel {
  int nv;           // usable candidates: the ascending prefix with j < pos
  int K;            // min(top_k, nv)
  int mode;
  int nlist;        // list entries appended (may exceed kCap: overflow)
  float lo, hi;     // list interval [lo, hi); hi = +inf: no "above" region
  float scale, offm;    // sample histogram bins: value_bin(s, scale, offm)
  uint32_t kmin, kmax;  // chunk 0's usable score range as order keys
  int need;             // keys of the list (the boundary bin) to take
};

struct RefineMisc {
  MemberSel ms[16];
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
  // selection bitmaps: one bit per candidate slot, word w of member m at
  // word 16w + m (the 16 members' words of a 32-candidate slice are adjacent)
  static constexpr int BMP_BYTES = 16 * 128 * 4;
  // per member 256 32-bit words: the list's radix histogram, and with the
  // scores written out the selection's per-word prefix counts
  static constexpr int HIST_BYTES = 16 * 256 * 4;
  static constexpr int LK_BYTES = 16 * kCap * 4;        // list scores (fp32 bits, then order keys)
  static constexpr int LT_BYTES = 16 * kCap * 2;        // list candidate slots
  // the sample histograms ([16][kBins] words) span the histogram and list
  // bytes, which are not in use before the pass that fills the lists
  static_assert(16 * kBins * 4 == HIST_BYTES + LK_BYTES + LT_BYTES, "sample histograms span hist + lists");
  __host__ __device__ static int nch_max(int Kc) { return (Kc + 127) / 128; }
  __host__ __device__ static int cidx_words(int Kc) { return nch_max(Kc) * 128; }
  __host__ __device__ static int off_bmp(int Kc) { return OFF_C + 2 * cidx_words(Kc) * 4; }
  static int smem_bytes(int Kc) {
    return off_bmp(Kc) + BMP_BYTES + HIST_BYTES + LK_BYTES + LT_BYTES + static_cast<int>(sizeof(RefineMisc)) +
           1024;
  }
};

// Linear bin of a score, round(s * scale + off) clamped to [0, kBins-1], with
// offm = off + 2^23 (as a float): the fma rounds s*scale + offm to an integer
// in [2^23, 2^23 + kBins-1] after the clamps, and the bin is its low mantissa
// bits.  One rounding of a function increasing in s, then monotone clamps, so
// the bins are ordered like the scores, and -0 and +0 share a bin.
template <int NB = kBins>
__device__ __forceinline__ int value_bin(float s, float scale, float offm) {
  const float t = fminf(fmaxf(__fmaf_rn(s, scale, offm), kMagic), kMagic + static_cast<float>(NB - 1));
  return static_cast<int>(__float_as_uint(t) & static_cast<uint32_t>(NB - 1));
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
  static_assert(PER % 4 == 0 && ((PER / 4) & (PER / 4 - 1)) == 0, "bins are read four at a time, 2^n reads per lane");
  const int b0 = NBINS - PER * (lane + 1);
  int s = 0;
  // lane l starts its 16-byte reads at a rotated offset: the lanes' groups lie
  // PER words apart, so unrotated reads would all hit the same banks
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) {
    const uint4 x = reinterpret_cast<const uint4*>(h + b0)[(i + lane) & (PER / 4 - 1)];
    s += static_cast<int>(x.x + x.y + x.z + x.w);
  }
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= r);
  const int L = hit ? __ffs(hit) - 1 : 31;
  const int cum = __shfl_sync(0xffffffffu, incl - s, L);   // counts above group L
  const int bL = NBINS - PER * (L + 1);
  // group L's bins, one per lane, summed from the top bin down: the answer is
  // the highest bin whose suffix (plus the counts above the group) reaches r
  const int c = lane < PER ? static_cast<int>(h[bL + lane]) : 0;
  int suf = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned ok = __ballot_sync(0xffffffffu, lane < PER && cum + suf >= r);
  const int i = ok ? 31 - __clz(ok) : 0;   // (the counts always reach r)
  *above = cum + __shfl_sync(0xffffffffu, suf - c, i);
  return bL + i;
}

// v[j] for a lane-varying j in [0, 16), by a tree of selects (no local memory).
__device__ __forceinline__ uint32_t pick16(const uint32_t (&v)[16], int j) {
  uint32_t w8[8], w4[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) w8[i] = (j & 1) ? v[2 * i + 1] : v[2 * i];
#pragma unroll
  for (int i = 0; i < 4; ++i) w4[i] = (j & 2) ? w8[2 * i + 1] : w8[2 * i];
  const uint32_t w0 = (j & 4) ? w4[1] : w4[0];
  const uint32_t w1 = (j & 4) ? w4[3] : w4[2];
  return (j & 8) ? w1 : w0;
}

// One work item: a unit's batch of up to 16 members.
struct RefineItem {
  int h, u, mb, nb, pos0, nc, nch;
  int jlim;             // candidate key indices lie in [0, jlim): the scan's bound
  long long key_row0;   // cache row of key index 0 (packed layouts)
  long long qrow0;      // row (before *H) of member 0's query and output
};

__device__ __forceinline__ RefineItem refine_item(const RefineParams& p, int item) {
  RefineItem it;
  const int ui = item / p.nbatch;
  it.mb = (item - ui * p.nbatch) * 16;
  it.h = ui / p.G;
  it.u = ui - it.h * p.G;
  int nm;
  if (!p.ci.decode()) {
    const int s = it.u * p.g;
    nm = min(s + p.g, p.L) - s;
    it.pos0 = s;
    it.key_row0 = 0;
    it.qrow0 = s;
  } else {
    nm = p.g;
    it.key_row0 = p.ci.row0(it.u);
    const int len = p.ci.len(it.u);
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

// The chunk scored at position i of a unit with nch chunks: even chunks
// first, then odd ones; positions past nch (chunks the unit does not use)
// map to themselves.
__device__ __forceinline__ int chunk_at(int i, int nch) {
  const int ne = (nch + 1) >> 1;
  return i < nch ? (i < ne ? 2 * i : 2 * (i - ne) + 1) : i;
}
// The scoring position of chunk c (the inverse of chunk_at).
__device__ __forceinline__ int chunk_pos(int c, int nch) {
  const int ne = (nch + 1) >> 1;
  return c < nch ? ((c & 1) ? ne + (c >> 1) : (c >> 1)) : c;
}

// PAGED: decode keys behind a block table (the key row of each candidate is
// looked up); else the rows of a sequence (or of the prefill) are contiguous.
template <int D, bool PAGED>
__global__ void __launch_bounds__(640, 1) refine_kernel(RefineParams p) {
  using C = RefineCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment by an offset from the shared array itself, so that
  // every pointer derived from it stays a shared-space pointer (plain shared
  // loads and stores rather than generic ones)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  const int NCH = C::nch_max(p.Kc);
  const int CW = C::cidx_words(p.Kc);
  int32_t* cidx0 = reinterpret_cast<int32_t*>(smem + C::OFF_C);
  uint32_t* bmp = reinterpret_cast<uint32_t*>(smem + C::off_bmp(p.Kc));       // [16][128]
  uint32_t* hist = bmp + C::BMP_BYTES / 4;                                      // [16][256]
  uint32_t* shist = hist;                                                       // [16][kBins], phase A only
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
      mbar_init(smem_u32(&M->tfree[c]), 4);   // the four lane-quarter warps that read chunk c
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
    // Thread 0 fetches each unit's candidate row with one bulk copy; then all
    // 96 producer threads gather the
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
        ok = mbar_wait(smem_u32(&M->cfree[buf]), ((kk >> 1) - 1) & 1, abort_flag, p.status, p.wait_ns);
      ok = !named_barrier_or(1, C::NPROD, !ok);
      if (ok && pt == 0) {
        const uint32_t bytes = static_cast<uint32_t>(it.nch) * 128u * 4u;
        mbar_arrive_expect_tx(cbar, bytes);
        if (bytes) bulk_copy_g2s(smem_u32(cx), p.cand + (static_cast<long long>(it.h) * p.G + it.u) * CW, bytes, cbar);
      }
      if (ok) ok = mbar_wait(cbar, (kk >> 1) & 1, abort_flag, p.status, p.wait_ns);
      const uint16_t* kbase = p.keys + (it.key_row0 * p.H + it.h) * static_cast<long long>(D) + p8 * 8;
      const uint32_t bB = sB + buf * C::B_BYTES;
      for (int ci = 0; ci < it.nch; ++ci) {
        const int c = chunk_at(ci, it.nch);
        const int s = sseq % C::NS;
        // one warp watches the stage; the others sleep on the named barrier
        if (sseq >= C::NS && ok && warp == 0)
          ok = mbar_wait(smem_u32(&M->empty[s]), ((sseq / C::NS) - 1) & 1, abort_flag, p.status, p.wait_ns);
        ok = !named_barrier_or(1, C::NPROD, !ok);
        if (ok) {
          const uint32_t dst0 = sA + s * C::STAGE;
          const int32_t* cxc = cx + c * 128;
          for (int rr = rr0; rr < 128; rr += RSTEP) {
            const int j = cxc[rr];
            // a missing candidate (-1 padding) reads as zeros; so would an
            // index outside the scan's bound, which no candidate row holds
            const bool in = j >= 0 && j < it.jlim;
            const long long row = PAGED ? p.ci.row(it.u, 0, in ? j : 0) : (in ? j : 0);
            const uint16_t* src = kbase + row * rowstride;
            const uint32_t dst = dst0 + rr * 128 + ((p8 ^ (rr & 7)) << 4);
            const uint32_t nbytes = in ? 16u : 0u;
#pragma unroll
            for (int a = 0; a < C::KATOMS; ++a) cp_async_16(dst + a * C::ATOM_A, src + a * 64, nbytes);
          }
          if (ci == 0) {
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
      for (int ci = 0; ci < NCH && ok; ++ci) {
        const int c = chunk_at(ci, it.nch);
        // the previous item's select warps are done with these columns
        if (kk >= 1) ok = mbar_wait(smem_u32(&M->tfree[c]), (kk - 1) & 1, abort_flag, p.status, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && c < it.nch) {
          const int s = sseq % C::NS;
          ok = mbar_wait(smem_u32(&M->full[s]), (sseq / C::NS) & 1, abort_flag, p.status, p.wait_ns);
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
    const int sw = warp - C::SEL_WARP0;   // 0..15: the member whose list and rows this warp handles
    const int q = warp & 3;               // TMEM lane quarter: candidates 32q .. 32q+31 of a chunk
    const int st = sw >> 2;               // chunk stream: the chunks at scoring positions st, st+4, ...
    const int stid = sw * 32 + lane;      // 0..511
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t ltmask = (1u << lane) - 1u;
    const float kInf = __int_as_float(0x7f800000);
    auto sel_sync = [&]() { named_barrier(2, C::NSEL); };
    // gives chunk c's columns back (this warp has its scores in registers)
    auto release = [&](int c) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&M->tfree[c]));
    };
    int kk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const RefineItem it = refine_item(p, item);
      if (it.nb <= 0) continue;
      const int buf = kk & 1;
      const int nch = it.nch, nb = it.nb;
      const int32_t* cx = cidx0 + buf * CW;
      if (ok) ok = mbar_wait(smem_u32(&M->cready[buf]), (kk >> 1) & 1, abort_flag, p.status, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      // ---- per-member usable counts (the candidate set is ascending) and modes
      if (sw == 0 && ok) {
        // member m (lane m) uses the candidates below its position.  The row
        // is ascending and its entries at or past member 0's position are the
        // group's own keys at its end, so when the last 32 entries hold them
        // all, one vote per member counts them; else a binary search does
        const int first = it.pos0 + it.mb;
        const int e = it.nc - 32 + lane;
        const int ce = e >= 0 ? cx[e] : -1;
        const bool covered = it.nc <= 32 || __shfl_sync(0xffffffffu, ce, 0) < first;
        int nv = 0;
        if (covered) {
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const int past = __popc(__ballot_sync(0xffffffffu, ce >= first + m));
            if (lane == m) nv = it.nc - past;
          }
        } else if (lane < 16) {
          const int pos = first + lane;
          int lo = 0, hi = it.nc;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (cx[mid] < pos) lo = mid + 1;
            else hi = mid;
          }
          nv = lo;
        }
        if (lane < 16) {
          if (lane >= nb) nv = 0;
          MemberSel& S = M->ms[lane];
          const int K = min(p.top_k, nv);
          S.nv = nv;
          S.K = K;
          S.mode = K == 0 ? kMNone : (K == nv ? kMAll : kMBand);
          S.nlist = 0;
          S.need = 0;
          S.lo = kInf;   // None and All take no list; Band is set below
          S.hi = kInf;
          S.kmin = 0xFFFFFFFFu;
          S.kmax = 0u;
        }
      }
      // bitmaps and histograms start at zero
      for (int i = stid; i < (C::BMP_BYTES + 16 * kBins * 4) / 16; i += C::NSEL)
        reinterpret_cast<uint4*>(bmp)[i] = make_uint4(0, 0, 0, 0);
      if (named_barrier_or(2, C::NSEL, !ok)) break;
      // the members that need a selection (bit m), and the fewest usable
      // candidates among them: one read per lane, one vote (uniform values)
      uint32_t bandm;
      int nvmin;
      {
        const MemberSel& S = M->ms[lane & 15];
        const bool band = S.mode == kMBand;
        bandm = __ballot_sync(0xffffffffu, band) & 0xFFFFu;
        nvmin = static_cast<int>(__reduce_min_sync(0xffffffffu, band ? static_cast<uint32_t>(S.nv) : 0x7FFFFFFFu));
      }
      const bool anyb = bandm != 0u;

      if (anyb) {
        // ---- chunk 0's score range sets each member's histogram bins
        if (st == 0) {
          if (ok) ok = mbar_wait(smem_u32(&M->tready[0]), kk & 1, abort_flag, p.status, p.wait_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (ok) {
            tc_fence_after();
            uint32_t v[16];
            tmem_ld_32x32b_x16(tq, v);
            tmem_ld_wait();
            const int t = q * 32 + lane;
            const bool all_use = 128 <= nvmin;   // chunk 0 lies inside every member's usable prefix
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              reg_fence(v[j]);
              if ((bandm >> j) & 1u) {
                const bool use = all_use || t < M->ms[j].nv;
                const uint32_t key = score_key(__uint_as_float(v[j]));
                const uint32_t mn = __reduce_min_sync(0xffffffffu, use ? key : 0xFFFFFFFFu);
                const uint32_t mx = __reduce_max_sync(0xffffffffu, use ? key : 0u);
                if (lane == 0) {
                  red_shared_min(smem_u32(&M->ms[j].kmin), mn);
                  red_shared_max(smem_u32(&M->ms[j].kmax), mx);
                }
              }
            }
          }
        }
        if (named_barrier_or(2, C::NSEL, !ok)) break;
        // bins linear in the score over chunk 0's range (scores outside it
        // clamp to the end bins); a member whose range is empty or not finite
        // goes to the exact fallback
        if (lane == 0 && M->ms[sw].mode == kMBand) {
          MemberSel& S = M->ms[sw];
          const float vmin = key_score(S.kmin), vmax = key_score(S.kmax);
          const float vsc = __fdiv_rn(static_cast<float>(kBins), __fsub_rn(vmax, vmin));
          const float voff = __fadd_rn(__fmul_rn(-vmin, vsc), kMagic);
          const bool good =
              S.kmin < S.kmax && isfinite(vmin) && isfinite(vmax) && isfinite(vsc) && vsc > 0.f && isfinite(voff);
          S.scale = vsc;
          S.offm = voff;
          if (!good) S.mode = kMMiss;
        }
        sel_sync();
        // ---- the histogram of every usable score, chunk by chunk as the MMAs
        //      finish (the columns stay in TMEM for the pass below).  A member
        //      without a selection counts into its own, unused, histogram,
        //      which keeps the loop free of branches
        float sc4[16], of4[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool band = M->ms[j].mode == kMBand;
          sc4[j] = band ? M->ms[j].scale : 0.f;
          of4[j] = band ? M->ms[j].offm : kMagic;
        }
        const uint32_t sh0 = smem_u32(shist);
        for (int i = st; i < nch; i += 4) {
          const int c = chunk_at(i, nch);
          if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status, p.wait_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          uint32_t v[16];
          tmem_ld_32x32b_x16(tq + 16 * c, v);
          tmem_ld_wait();
          const int t = c * 128 + q * 32 + lane;
          if (c * 128 + q * 32 + 32 <= nvmin) {   // every member can use every lane
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              reg_fence(v[j]);
              red_shared_add_nb(sh0 + 4u * (j * kBins + value_bin(__uint_as_float(v[j]), sc4[j], of4[j])), 1u);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              reg_fence(v[j]);
              if (t < M->ms[j].nv)
                red_shared_add_nb(sh0 + 4u * (j * kBins + value_bin(__uint_as_float(v[j]), sc4[j], of4[j])), 1u);
            }
          }
        }
        if (named_barrier_or(2, C::NSEL, !ok)) break;
        // ---- warp sw: member sw's boundary bin, the one that holds its k-th
        //      largest score: keys in higher bins are taken, the bin's own keys
        //      (its list) are ranked exactly
        if (sw < nb && M->ms[sw].mode == kMBand) {
          MemberSel& S = M->ms[sw];
          const uint32_t* hm = shist + sw * kBins;
          int above;
          const int b = warp_rank_bin<kBins>(hm, S.K, lane, &above);
          const int cnt = static_cast<int>(hm[b]);
          float hi = kInf, lo = -kInf;
          if (b < kBins - 1) hi = key_score(warp_first_key_of_bin(b + 1, S.scale, S.offm, lane));
          if (b > 0) lo = key_score(warp_first_key_of_bin(b, S.scale, S.offm, lane));
          if (lane == 0) {
            S.need = S.K - above;
            S.lo = lo;
            S.hi = hi;
            if (cnt > kCap) S.mode = kMMiss;   // a bin crowded by ties: the exact fallback
          }
          __syncwarp();
        }
        sel_sync();
      }

      // ---- one pass: per chunk, each member's ">= hi" lanes into its bitmap
      //      and its boundary-bin lanes onto its list; the chunk's TMEM columns
      //      go back as soon as they are loaded (unless the scores are
      //      written out, which reads them again)
      const bool keep_tmem = p.out_scores != nullptr;
      const uint32_t lk_s = smem_u32(lkeys), ls_s = smem_u32(lslot);
      float th[16], tl[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const MemberSel& S = M->ms[j];
        const bool cls = S.mode == kMBand;
        th[j] = cls ? S.hi : kInf;
        tl[j] = cls ? S.lo : kInf;
      }
#pragma unroll 1
      for (int i = st; i < nch; i += 4) {
        const int c = chunk_at(i, nch);
        if (ok && !anyb) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (!anyb) {   // nothing to classify
          if (!keep_tmem) release(c);
          continue;
        }
        tc_fence_after();
        uint32_t v[16];
        tmem_ld_32x32b_x16(tq + 16 * c, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) reg_fence(v[j]);
        if (!keep_tmem) release(c);
        const int base_t = c * 128 + q * 32;
        const int t = base_t + lane;
        // member j: the ">= hi" lanes by one vote (its bitmap word), the lanes
        // in [lo, hi) as bit j of this lane's band mask
        uint32_t a[16];
        uint32_t bm = 0u;
        if (base_t + 32 <= nvmin) {   // every classified member can use every lane
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float f = __uint_as_float(v[j]);
            const bool above = f >= th[j];
            a[j] = __ballot_sync(0xffffffffu, above);
            bm |= (!above && f >= tl[j]) ? (1u << j) : 0u;
          }
        } else {                      // a member's usable prefix ends in this slice
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float f = __uint_as_float(v[j]);
            const bool use = t < M->ms[j].nv;
            const bool above = use && f >= th[j];
            a[j] = __ballot_sync(0xffffffffu, above);
            bm |= (use && !above && f >= tl[j]) ? (1u << j) : 0u;
          }
        }
        if (lane == 0) {
          uint4* w = reinterpret_cast<uint4*>(bmp + (c * 4 + q) * 16);
          w[0] = make_uint4(a[0], a[1], a[2], a[3]);
          w[1] = make_uint4(a[4], a[5], a[6], a[7]);
          w[2] = make_uint4(a[8], a[9], a[10], a[11]);
          w[3] = make_uint4(a[12], a[13], a[14], a[15]);
        }
        // this lane's boundary keys onto their members' lists (a boundary bin
        // holds a few keys of the member's candidates, so few lanes loop)
        while (bm != 0u) {
          const int j = __ffs(bm) - 1;
          bm &= bm - 1u;
          const uint32_t at = min(atom_shared_add(smem_u32(&M->ms[j].nlist), 1u), static_cast<uint32_t>(kCap - 1));
          st_shared_u32_nb(lk_s + 4u * (j * kCap + at), pick16(v, j));
          st_shared_u16_nb(ls_s + 2u * (j * kCap + at), static_cast<uint16_t>(t));
        }
      }
      if (named_barrier_or(2, C::NSEL, !ok)) break;

      // ---- warp sw ranks member sw's list exactly: the need-th largest key
      //      (radix select from the highest bit that varies) and how many of
      //      its copies are taken; decisions OR-ed into the member's bitmap
      uint32_t* mb = bmp + sw;   // member sw's word w is mb[16 * w]
      if (sw < nb) {
        MemberSel& S = M->ms[sw];
        int mode = S.mode;
        if (mode == kMBand) {
          const int n = S.nlist, need = S.need;
          if (n > kCap || need < 1 || need > n) {
            mode = kMMiss;   // (cannot happen: the list is the boundary bin)
          } else {
            uint32_t* lk = lkeys + sw * kCap;
            const uint16_t* ls = lslot + sw * kCap;
            uint32_t* rh = hist + sw * 256;   // radix histogram
            for (int e = lane; e < n; e += 32) lk[e] = score_key(__uint_as_float(lk[e]));
            __syncwarp();
            uint32_t tk = 0u, tmask = 0u;
            int need_eq = 0x7FFFFFFF;   // the whole list, when need == n
            bool ranked = false;        // decisions already in the bitmap
            if (need < n && n <= 64) {
              // a short list: a key is taken when fewer than `need` keys beat
              // it (larger, or equal with a lower slot)
              for (int x = lane; x < n; x += 32) {
                const uint32_t kx = lk[x], sx = ls[x];
                int beat = 0;
                for (int y = 0; y < n; ++y) {
                  const uint32_t ky = lk[y], sy = ls[y];
                  beat += (ky > kx || (ky == kx && sy < sx)) ? 1 : 0;
                }
                if (beat < need) red_shared_or_nb(smem_u32(&mb[16 * (sx >> 5)]), 1u << (sx & 31));
              }
              __syncwarp();
              ranked = true;
            }
            if (need < n && !ranked) {
              // bins linear in the score over the list's own range spread its
              // keys evenly; the need-th largest lies in bin b, and the few
              // keys of bin b are ranked exactly against each other
              uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
              for (int e = lane; e < n; e += 32) {
                kmn = min(kmn, lk[e]);
                kmx = max(kmx, lk[e]);
              }
              kmn = __reduce_min_sync(0xffffffffu, kmn);
              kmx = __reduce_max_sync(0xffffffffu, kmx);
              const float vmin = key_score(kmn), vmax = key_score(kmx);
              const float lsc = __fdiv_rn(256.f, __fsub_rn(vmax, vmin));
              const float lof = __fadd_rn(__fmul_rn(-vmin, lsc), kMagic);
              if (kmn < kmx && isfinite(vmin) && isfinite(vmax) && isfinite(lsc) && lsc > 0.f && isfinite(lof)) {
                for (int b = lane; b < 256; b += 32) rh[b] = 0u;
                __syncwarp();
                for (int e = lane; e < n; e += 32)
                  red_shared_add_nb(smem_u32(&rh[value_bin<256>(key_score(lk[e]), lsc, lof)]), 1u);
                __syncwarp();
                int above;
                const int bb = warp_rank_bin<256>(rh, need, lane, &above);
                const int cntb = static_cast<int>(rh[bb]);
                const int r2 = need - above;   // keys of bin bb to take
                __syncwarp();
                if (cntb <= 64) {
                  // bin bb's keys and slots to rh[0..63] and rh[64..127]
                  int base = 0;
                  for (int e0 = 0; e0 < n; e0 += 32) {
                    const int e = e0 + lane;
                    const uint32_t key = e < n ? lk[e] : 0u;
                    const int bin = e < n ? value_bin<256>(key_score(key), lsc, lof) : -1;
                    const unsigned m = __ballot_sync(0xffffffffu, bin == bb);
                    if (bin == bb) {
                      const int at = base + __popc(m & ltmask);
                      rh[at] = key;
                      rh[64 + at] = ls[e];
                    }
                    if (bin > bb) red_shared_or_nb(smem_u32(&mb[16 * (ls[e] >> 5)]), 1u << (ls[e] & 31));
                    base += __popc(m);
                  }
                  __syncwarp();
                  // a key is taken when fewer than r2 keys of the bin beat it
                  // (larger, or equal with a lower slot)
                  for (int x = lane; x < cntb; x += 32) {
                    const uint32_t kx = rh[x], sx = rh[64 + x];
                    int beat = 0;
                    for (int y = 0; y < cntb; ++y) {
                      const uint32_t ky = rh[y], sy = rh[64 + y];
                      beat += (ky > kx || (ky == kx && sy < sx)) ? 1 : 0;
                    }
                    if (beat < r2) red_shared_or_nb(smem_u32(&mb[16 * (sx >> 5)]), 1u << (sx & 31));
                  }
                  __syncwarp();
                  ranked = true;
                }
              }
            }
            if (need < n && !ranked) {
              // many keys in one bin (ties, or a crowded bin): radix select on
              // the order keys from the highest bit that varies
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
                  if ((key & tmask) == tk) red_shared_add_nb(smem_u32(&rh[(key >> sh) & nbm]), 1u);
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
            for (int e = lane; e < n && !ranked; e += 32) {
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
                red_shared_or_nb(smem_u32(&mb[16 * (t >> 5)]), 1u << (t & 31));
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
      // ---- warp sw writes member sw's row: its bitmap in candidate order, one
      //      coalesced store per 32-candidate word (a miss's row is written by
      //      the fallback)
      if (sw < nb) {
        const MemberSel& S = M->ms[sw];
        const int mode = S.mode, K = S.K;
        const long long orow = (it.qrow0 + it.mb + sw) * p.H + it.h;
        int32_t* out_row = p.out + orow * p.top_k;
        if (mode == kMAll) {
          for (int t = lane; t < K; t += 32) out_row[t] = cx[t];
        } else if (mode == kMBand) {
          // eight 32-candidate words per round: their shared-memory reads go
          // out together, so a round waits for one read latency, not eight
          const int nw = nch * 4;
          int base = 0;
#pragma unroll 1
          for (int w0 = 0; w0 < nw; w0 += 8) {
            uint32_t wd[8];
            int32_t val[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const bool inw = w0 + x < nw;
              wd[x] = inw ? mb[16 * (w0 + x)] : 0u;
              val[x] = inw ? cx[(w0 + x) * 32 + lane] : 0;
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              if ((wd[x] >> lane) & 1u) out_row[base + __popc(wd[x] & ltmask)] = val[x];
              base += __popc(wd[x]);
            }
          }
        }
        if (mode != kMMiss)
          for (int t = K + lane; t < p.top_k; t += 32) out_row[t] = -1;
        uint32_t wds[4];
#pragma unroll
        for (int x = 0; x < 4 && keep_tmem; ++x) {
          const int w = 4 * lane + x;
          if (mode == kMAll) {
            const int u = K - 32 * w;
            wds[x] = u >= 32 ? 0xFFFFFFFFu : (u <= 0 ? 0u : ((1u << u) - 1u));
          } else if (mode == kMBand) {
            wds[x] = mb[16 * w];
          } else {
            wds[x] = 0u;
          }
        }
        if (keep_tmem) {
          // per-word prefix counts of the selection, for the scores' slots
          const int own = __popc(wds[0]) + __popc(wds[1]) + __popc(wds[2]) + __popc(wds[3]);
          int incl = own;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          uint32_t* pre = hist + sw * 256;
          int at = incl - own;
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            pre[4 * lane + x] = static_cast<uint32_t>(at);
            at += __popc(wds[x]);
          }
          if (mode != kMMiss)
            for (int t = K + lane; t < p.top_k; t += 32) p.out_scores[orow * p.top_k + t] = __int_as_float(0x7fc00000);
        }
      }
      if (keep_tmem) {
        // the selected scores, read again from TMEM, then the columns go back
        sel_sync();
        for (int i = st; i < nch; i += 4) {
          const int c = chunk_at(i, nch);
          tc_fence_after();
          uint32_t v[16];
          tmem_ld_32x32b_x16(tq + 16 * c, v);
          tmem_ld_wait();
          const int t = c * 128 + q * 32 + lane;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            reg_fence(v[j]);
            if (j < nb) {
              const int mode = M->ms[j].mode;
              float* srow = p.out_scores + ((it.qrow0 + it.mb + j) * p.H + it.h) * static_cast<long long>(p.top_k);
              if (mode == kMAll) {
                if (t < M->ms[j].K) srow[t] = __uint_as_float(v[j]);
              } else if (mode == kMBand) {
                const uint32_t word = bmp[(c * 4 + q) * 16 + j];
                if ((word >> lane) & 1u)
                  srow[hist[j * 256 + c * 4 + q] + __popc(word & ltmask)] = __uint_as_float(v[j]);
              }
            }
          }
          release(c);
        }
      }
      // Chunks past this item's list got their "scored" commit without MMAs;
      // this warp's stream owns those at positions st, st+4, ... past nch.
      // Wait for those commits too before giving the chunks back: every
      // release then answers a commit of this item, and the MMA warp can never
      // find a chunk's "free" barrier two phases ahead of its wait.
      for (int c = nch + ((st - nch) & 3); c < NCH; c += 4) {
        if (ok) ok = mbar_wait(smem_u32(&M->tready[c]), kk & 1, abort_flag, p.status, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) release(c);
      }
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
    for (int t = threadIdx.x; t < it.nc; t += kRfbNT) cl[t] = row[t];
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
        const uint4* kr = reinterpret_cast<const uint4*>(kb + p.ci.row(it.u, 0, j) * rowstride);
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
