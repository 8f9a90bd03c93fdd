// Prefix scan of proxies against keys on the 5th-generation tensor cores,
// with a fused streaming filter for the top-K select.
//
// Method ("PIVOT explained", section "How It Works"; paper abstract): one
// shared full-prefix scan per query group, scores s_j = p . k_j for the group's
// proxy p over its causal prefix, candidate set = the top-Kc of s.  Here the
// same kernel also serves the Reuse scan (prefix = keys before the group start,
// top-k) and the dense indexer (g = 1, proxy = the query itself).
//
// One CTA owns 128 proxy rows of one head (M = 128) and streams the head's
// keys in tiles of 128 (N = 128, K = d) through a TMA -> shared -> tcgen05.mma
// -> TMEM pipeline with four accumulators.  The proxy rows stay in shared
// memory as nterms bf16 tiles: the exact three-term split of the fp32 mean
// (hi + mid + lo), or one tile for the dense indexer (the query itself) and
// for the bf16-proxy variant.  Every key tile is multiplied by each term into
// the same accumulator, so a score is p . k with fp32 accumulation.
//   warp 0      TMA producer (keys, and the proxy tile once)
//   warp 1      TMEM allocator and MMA issuer (one elected thread)
//   warps 2..17 epilogue, four groups of four: thread (e, r) owns TMEM lane r
//               (proxy row r) of accumulator e, and in the main pass the
//               e-th quarter of the row's key tiles
// The score matrix is never written out.  Each epilogue thread compares its
// row's scores with a per-row threshold tau and appends the survivors
// (score bits, key index) to its run of the row's spill list in global
// memory, in ascending key order; an exact select over the four runs
// (finalize kernel) then gives the top-K.
//
// The threshold comes from a sample of the row's prefix: every S-th key tile is
// scanned twice before the main pass (two MSB radix histogram passes over the
// sample in shared memory), and tau is set at a sample rank a few standard
// deviations (four) above K * (sample size / prefix), so that nearly always
// at least K scores pass it.  Rows whose prefix fits half the
// spill capacity take every key (tau = -inf).  Rows where the guess is wrong
// (fewer than K survivors, or more than a spill region holds) are detected by
// the finalize kernel and redone exactly by the fallback kernel, so the result
// never depends on the guess.  Key tiles entirely beyond a CTA's longest
// prefix are skipped (causal skipping).
#pragma once

#include "ptx.cuh"

namespace pivot {

struct ScanParams {
  int G;           // proxy rows per head
  int L;           // keys per head
  int H;           // heads
  int g;           // group size (1 for the dense indexer)
  int bound_kind;  // 0: row i sees keys j < min(i*g+g, L) - 1; 1: keys j < i*g
  int K_sel;       // how many keys the finalize select keeps per row
  int cap;         // spill capacity per row (entries, even)
  int S;           // sample stride in key tiles (every S-th tile is sampled)
  int tiles_per_head;
  int nterms;      // bf16 proxy terms (1 or 3); term t's rows start at t*G in the proxy tensor map
  uint2* spill;    // [H*G][cap]: (score bits, key index); see cnt
  int4* cnt;       // [H*G]: survivors of the four runs (key quarters q = 0..3).
                   // Run q lives in region q/2 = [q/2 * cap/2, (q/2+1) * cap/2):
                   // even runs fill it upward from its first slot, odd runs
                   // downward from its last; a region whose two runs sum to
                   // more than cap/2 has overflowed
  int* status;     // device status word
  unsigned long long wait_ns;   // limit of every bounded wait
};

__device__ __forceinline__ int row_bound(const ScanParams& p, int i) {
  if (p.bound_kind == 0) return min(i * p.g + p.g, p.L) - 1;
  return i * p.g;
}

template <int D>
struct ScanCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;                      // keys per tile (MMA N)
  static constexpr int NACC = 4;                      // TMEM accumulators = epilogue groups
  static constexpr int KATOMS = D / 64;               // 64-element (128-byte) K slices
  static constexpr int NTERMS = 3;                    // proxy tiles held (the most any call uses)
  static constexpr int NST = (D == 128) ? 2 : 6;      // key-tile stages in shared memory
  static constexpr int A_BYTES = BM * D * 2;          // one proxy term
  static constexpr int B_BYTES = BN * D * 2;
  static constexpr int HIST_BYTES = 128 * BM * 4;     // [128 bin pairs][128 rows], two u16 counts per word
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NTERMS * A_BYTES;
  static constexpr int OFF_HIST = OFF_B + NST * B_BYTES;
  static constexpr int OFF_MISC = OFF_HIST + HIST_BYTES;  // per-row sample counts
  static constexpr int OFF_BAR = OFF_MISC + BM * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;   // barriers + alignment slack
  static constexpr int NEPI = NACC * 128;             // epilogue threads
  static constexpr int THREADS = 64 + NEPI;
  static constexpr uint32_t TMEM_COLS = NACC * BN;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int CW = 16;                       // columns per TMEM load (one chunk)
  static_assert(NACC * (2 * CW / 4) * BM * 16 <= HIST_BYTES, "main-pass staging (a chunk pair) aliases the histograms");
};

// The CTA's work, in one order shared by the producer, the MMA issuer and the
// epilogue: two sample passes over every S-th key tile (sample step s belongs
// to epilogue group s % 4), then the main pass, in which group q takes the
// q-th quarter of the key tiles, [q*nQ, min(q*nQ + nQ, nkt)), in ascending
// order, and the groups' tiles are interleaved round by round.
template <class F>
__device__ __forceinline__ void for_each_step(int ns, int S, int nkt, F f) {
  for (int pass = 0; pass < 2; ++pass)
    for (int s = 0; s < ns; ++s) f(s & 3, (s + 1) * S - 1, pass);
  const int nQ = (nkt + 3) / 4;
  for (int k = 0; k < nQ; ++k)
    for (int q = 0; q < 4; ++q)
      if (q * nQ + k < nkt) f(q, q * nQ + k, 2);
}

template <int D>
__global__ void __launch_bounds__(ScanCfg<D>::THREADS, 1)
scan_filter_kernel(const __grid_constant__ CUtensorMap tm_proxy, const __grid_constant__ CUtensorMap tm_keys,
                   ScanParams p) {
  using C = ScanCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment by an offset from the shared array itself, so that
  // every pointer derived from it stays a shared-space pointer (plain shared
  // loads and stores rather than generic ones)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  int* nsamp = reinterpret_cast<int*>(smem + C::OFF_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // barrier slots: [0,NST) full, [NST,2NST) empty, 2NST a_full,
  // 2NST+1+q tmem_full of accumulator q, 2NST+1+NACC+q tmem_empty of accumulator q
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::NST + s); };
  const uint32_t a_full = bar0 + 8u * (2 * C::NST);
  auto tfull_bar = [&](int q) { return bar0 + 8u * (2 * C::NST + 1 + q); };
  auto tempty_bar = [&](int q) { return bar0 + 8u * (2 * C::NST + 1 + C::NACC + q); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 192);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 200);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bid = blockIdx.x;
  const int h = bid / p.tiles_per_head;
  const int t = p.tiles_per_head - 1 - (bid % p.tiles_per_head);  // longest tiles first
  const int i0 = t * C::BM;
  const int i_last = min(i0 + C::BM, p.G) - 1;
  const int max_bound = row_bound(p, i_last);
  const int nkt = (max_bound + C::BN - 1) / C::BN;                // key tiles needed
  const int capH = p.cap / 2;                                      // entries per spill region
  const bool sampling = max_bound > capH;
  const int ns = sampling ? nkt / p.S : 0;                         // sampled tiles

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(a_full, 1);
    for (int q = 0; q < C::NACC; ++q) {
      mbar_init(tfull_bar(q), 1);
      mbar_init(tempty_bar(q), 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && 2 * ns + nkt > 0) {
      tma_prefetch_desc(&tm_proxy);
      tma_prefetch_desc(&tm_keys);
      mbar_arrive_expect_tx(a_full, p.nterms * C::A_BYTES);
      for (int tt = 0; tt < p.nterms; ++tt)
        for (int a = 0; a < C::KATOMS; ++a)
          tma_load_3d(sA + tt * C::A_BYTES + a * (C::BM * 128), &tm_proxy, a_full, a * 64, h, tt * p.G + i0);
      int step = 0, issued = 0;
      bool ok = true;
      for_each_step(ns, p.S, nkt, [&](int, int jt, int) {
        if (!ok) return;
        const int s = step % C::NST;
        const int use = step / C::NST;
        if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status, p.wait_ns)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(full_bar(s), C::B_BYTES);
        for (int a = 0; a < C::KATOMS; ++a)
          tma_load_3d(sB + s * C::B_BYTES + a * (C::BN * 128), &tm_keys, full_bar(s), a * 64, h, jt * C::BN);
        issued = ++step;
      });
      // Never leave the CTA with a copy still landing in its shared memory.
      mbar_wait_cleanup(a_full, 0);
      for (int q = max(0, issued - C::NST); q < issued; ++q) mbar_wait_cleanup(full_bar(q % C::NST), (q / C::NST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && 2 * ns + nkt > 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BM, C::BN);
      int use[C::NACC] = {0, 0, 0, 0};
      int step = 0;
      bool ok = mbar_wait(a_full, 0, abort_flag, p.status, p.wait_ns);
      for_each_step(ns, p.S, nkt, [&](int q, int, int) {
        if (!ok) return;
        const int s = step % C::NST;
        if (!mbar_wait(full_bar(s), (step / C::NST) & 1, abort_flag, p.status, p.wait_ns)) {
          ok = false;
          return;
        }
        int uq = 0;
#pragma unroll
        for (int x = 0; x < C::NACC; ++x) uq = (x == q) ? use[x] : uq;
        if (uq > 0 && !mbar_wait(tempty_bar(q), (uq - 1) & 1, abort_flag, p.status, p.wait_ns)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + q * C::BN;
        for (int tt = 0; tt < p.nterms; ++tt) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int a = kk >> 2, k4 = kk & 3;
            const uint64_t adesc = sw128_kmajor_desc(sA + tt * C::A_BYTES + a * (C::BM * 128) + k4 * 32);
            const uint64_t bdesc = sw128_kmajor_desc(sB + s * C::B_BYTES + a * (C::BN * 128) + k4 * 32);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (tt > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(empty_bar(s));
        umma_commit(tfull_bar(q));
#pragma unroll
        for (int x = 0; x < C::NACC; ++x) use[x] += (x == q) ? 1 : 0;
        ++step;
      });
      // All issued MMAs must be complete before the accumulators are released.
#pragma unroll
      for (int x = 0; x < C::NACC; ++x)
        if (use[x] > 0) mbar_wait_cleanup(tfull_bar(x), (use[x] - 1) & 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Four groups of four warps; group e owns accumulator e and the steps
    // for_each_step gives it.  Thread (e, r) handles proxy row r of the tile:
    // in the main pass, the e-th quarter of the row's key tiles.
    const int e = (warp - 2) >> 2;
    const int quarter = warp & 3;               // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;          // proxy row within the tile
    const int i = i0 + r;
    const bool row_ok = i < p.G;
    const int bound = row_ok ? row_bound(p, i) : 0;
    const long long row_id = static_cast<long long>(h) * p.G + i;
    // this thread's run: region e/2, upward (even e) or downward (odd e)
    uint2* run = p.spill + row_id * p.cap + (e >> 1) * capH + ((e & 1) ? capH - 1 : 0);
    const int dir = (e & 1) ? -1 : 1;
    int cnt = 0;
    float tau = -__int_as_float(0x7f800000);    // -inf: keep everything
    // the largest float below tau: for finite scores, v >= tau <=> v > tau_below
    float tau_below = tau;
    int n_sample = 0;
    int b1 = -1, rem = 0;
    const bool row_samples = sampling && bound > capH;

    auto bin_count = [&](int b) -> int { return (hist[(b >> 1) * C::BM + r] >> ((b & 1) << 4)) & 0xFFFF; };
    auto bin_add = [&](int b) { red_shared_add(smem_u32(&hist[(b >> 1) * C::BM + r]), 1u << ((b & 1) << 4)); };
    auto zero_quarter_row = [&]() {
      for (int w = 0; w < 32; ++w) hist[(e * 32 + w) * C::BM + r] = 0;
    };
    // Phase changes (sample pass 1 -> 2 -> main); every epilogue thread takes
    // the same barriers, in the same order.
    int done = sampling ? 0 : 2;
    if (sampling) {
      zero_quarter_row();
      if (e == 0) nsamp[r] = 0;
      named_barrier(1, C::NEPI);
    }
    auto advance = [&](int target) {
      while (done < target) {
        if (done == 0) {
          // end of sample pass 1: choose the top digit of tau
          if (n_sample) atomicAdd(&nsamp[r], n_sample);
          named_barrier(1, C::NEPI);
          const int total = nsamp[r];
          if (row_samples && total > 0) {
            const float expect = static_cast<float>(p.K_sel) * static_cast<float>(total) / static_cast<float>(bound);
            const int target_rank = static_cast<int>(ceilf(expect + 4.0f * sqrtf(expect) + 4.0f));
            if (target_rank <= total) {
              int cum = 0;
              for (int b = 255; b >= 0; --b) {
                const int cb = bin_count(b);
                if (cum + cb >= target_rank) {
                  b1 = b;
                  rem = target_rank - cum;
                  break;
                }
                cum += cb;
              }
            }
          }
          named_barrier(1, C::NEPI);
          zero_quarter_row();
          named_barrier(1, C::NEPI);
        } else {
          // end of sample pass 2: the second digit, then tau
          named_barrier(1, C::NEPI);
          if (b1 >= 0) {
            int cum = 0, b2 = 0;
            for (int b = 255; b >= 0; --b) {
              const int cb = bin_count(b);
              if (cum + cb >= rem) {
                b2 = b;
                break;
              }
              cum += cb;
            }
            tau = key_lower_edge_value((static_cast<uint32_t>(b1) << 24) | (static_cast<uint32_t>(b2) << 16));
            const uint32_t u = __float_as_uint(tau);
            if (tau == -__int_as_float(0x7f800000)) tau_below = tau;
            else if ((u & 0x7FFFFFFFu) == 0u) tau_below = __uint_as_float(0x80000001u);  // below +-0
            else tau_below = __uint_as_float((u >> 31) ? u + 1u : u - 1u);
          }
          // the main pass reuses the histogram space for staging
          named_barrier(1, C::NEPI);
        }
        ++done;
      }
    };

    // Main-pass staging for survivor lookups: this thread's values of a pair
    // of chunks (2*CW of them) as 2*CW/4 float4 at [((e*Q4 + i)*128 + r)*4].
    // The survivors of both chunks of a pair go out in one loop, which halves
    // how often a warp waits for its lane with the most survivors.
    constexpr int Q4 = 2 * C::CW / 4;
    float* stage = reinterpret_cast<float*>(hist);
    const float* st_r = stage + (static_cast<long long>(e) * Q4 * C::BM + r) * 4;
    uint32_t pend = 0;   // survivors of the pair's first chunk (bits 0..CW-1)
    // bit x = (v[x] >= tau) = the sign of tau_below - v[x] (an fadd, on the
    // FMA pipe), shifted into the mask by one funnel shift; four chains of
    // four consecutive keys, taken from the top so each bit lands in place
    auto chunk_mask = [&](const uint32_t (&v)[C::CW], uint32_t live) -> uint32_t {
      uint32_t c4[C::CW / 4];
#pragma unroll
      for (int k = 0; k < C::CW / 4; ++k) {
        uint32_t c = 0;
#pragma unroll
        for (int x = 4 * k + 3; x >= 4 * k; --x)
          c = __funnelshift_l(__float_as_uint(__fsub_rn(tau_below, __uint_as_float(v[x]))), c, 1);
        c4[k] = c;
      }
      uint32_t m = 0;
#pragma unroll
      for (int k = 0; k < C::CW / 4; ++k) m |= c4[k] << (4 * k);
      return m & live;
    };
    // survivors of a pair (bit x: key j0 + x) in ascending order, two per
    // step: (score bits, key index)
    auto flush = [&](uint32_t m, int j0) {
      if (cnt + __popc(m) > capH) {
        // the region is full: only count (the row goes to the exact fallback)
        cnt += __popc(m);
        return;
      }
      while (m) {
        const int x1 = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t s1 = __float_as_uint(st_r[(x1 >> 2) * (C::BM * 4) + (x1 & 3)]);
        run[dir * cnt] = make_uint2(s1, static_cast<uint32_t>(j0 + x1));
        ++cnt;
        if (m) {
          const int x2 = __ffs(m) - 1;
          m &= m - 1;
          const uint32_t s2 = __float_as_uint(st_r[(x2 >> 2) * (C::BM * 4) + (x2 & 3)]);
          run[dir * cnt] = make_uint2(s2, static_cast<uint32_t>(j0 + x2));
          ++cnt;
        }
      }
    };
    // half: 0 for the first chunk of a pair, 1 for the second (keys j0 - CW ...)
    auto process = [&](const uint32_t (&v)[C::CW], int j0, int phase, int half) {
      if (phase == 2) {
        const uint32_t live =
            j0 >= bound ? 0u : ((j0 + C::CW <= bound) ? (0xFFFFFFFFu >> (32 - C::CW)) : ((1u << (bound - j0)) - 1u));
        const uint32_t m = live ? chunk_mask(v, live) : 0u;
        if (m) {
#pragma unroll
          for (int q4 = 0; q4 < C::CW / 4; ++q4)
            reinterpret_cast<uint4*>(stage)[(e * Q4 + half * (C::CW / 4) + q4) * C::BM + r] =
                make_uint4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        }
        if (half == 0) {
          pend = m;
        } else {
          const uint32_t mm = pend | (m << C::CW);
          if (mm) flush(mm, j0 - C::CW);
        }
        return;
      }
      if (j0 >= bound) return;
      const uint32_t live = (j0 + C::CW <= bound) ? (0xFFFFFFFFu >> (32 - C::CW)) : ((1u << (bound - j0)) - 1u);
      if (phase == 0) {
#pragma unroll
        for (int x = 0; x < C::CW; ++x)
          if ((live >> x) & 1u) bin_add(static_cast<int>(score_key(__uint_as_float(v[x])) >> 24));
        n_sample += __popc(live);
      } else if (b1 >= 0) {
#pragma unroll
        for (int x = 0; x < C::CW; ++x) {
          if ((live >> x) & 1u) {
            const uint32_t key = score_key(__uint_as_float(v[x]));
            if (static_cast<int>(key >> 24) == b1) bin_add(static_cast<int>((key >> 16) & 255));
          }
        }
      }
    };

    // An aborted warp keeps stepping (without waits or TMEM loads) so that it
    // still takes every phase barrier.
    bool alive = true;
    int use = 0;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + e * C::BN;
    for_each_step(ns, p.S, nkt, [&](int q, int jt, int phase) {
      if (q != e) return;
      advance(phase);
      // the whole warp decides together: tcgen05.ld below is warp-collective
      if (alive) alive = __all_sync(0xffffffffu, mbar_wait(tfull_bar(e), use & 1, abort_flag, p.status, p.wait_ns));
      ++use;
      if (!alive) return;
      tc_fence_after();
      // two register buffers: the TMEM load of chunk c+1 overlaps the work on chunk c
      constexpr int NCK = C::BN / C::CW;
      uint32_t va[C::CW], vb[C::CW];
      tmem_ld_32x32b_x16(taddr, va);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < C::CW; ++x) reg_fence(va[x]);
#pragma unroll 1
      for (int c = 0; c < NCK; c += 2) {
        tmem_ld_32x32b_x16(taddr + (c + 1) * C::CW, vb);
        process(va, jt * C::BN + c * C::CW, phase, 0);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < C::CW; ++x) reg_fence(vb[x]);
        if (c + 2 < NCK) {
          tmem_ld_32x32b_x16(taddr + (c + 2) * C::CW, va);
        } else {
          // every column of this accumulator is in registers now
          tc_fence_before();
          mbar_arrive(tempty_bar(e));
        }
        process(vb, jt * C::BN + (c + 1) * C::CW, phase, 1);
        if (c + 2 < NCK) {
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < C::CW; ++x) reg_fence(va[x]);
        }
      }
    });
    advance(2);
    if (row_ok) reinterpret_cast<int*>(p.cnt)[4 * row_id + e] = cnt;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace pivot
