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
// keys in tiles of 256 (N = 256, K = d) through a TMA -> shared -> tcgen05.mma
// -> TMEM pipeline:
//   warp 0      TMA producer (keys, and the proxy tile once)
//   warp 1      TMEM allocator and MMA issuer (one elected thread)
//   warps 2..9  epilogue, two groups of four: thread (e, r) owns TMEM lane r
//               (proxy row r) of accumulator buffer e
// The score matrix is never written out.  Each epilogue thread compares its
// row's scores with a per-row threshold tau and appends the survivors
// (order key, key index) to that row's spill list in global memory; an exact
// select over the spill list (finalize kernel) then gives the top-K.
//
// The threshold comes from a sample of the row's prefix: every S-th key tile is
// scanned twice before the main pass (two MSB radix histogram passes over the
// sample in shared memory), and tau is set at a sample rank a few standard
// deviations above K * (sample size / prefix), so that with overwhelming
// probability at least K scores pass it.  Rows whose prefix fits the spill
// capacity take every key (tau = -inf).  Rows where the guess is wrong (fewer
// than K or more than `cap` survivors) are detected by the finalize kernel and
// redone exactly by the fallback kernel, so the result never depends on the
// guess.  Key tiles entirely beyond a CTA's longest prefix are skipped (causal
// skipping).
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
  int cap;         // spill capacity per row (entries)
  int S;           // sample stride in key tiles (every S-th tile is sampled)
  int tiles_per_head;
  uint2* spill;    // [H*G][cap]: (order key, key index); see cnt
  int2* cnt;       // [H*G]: survivors from the first half of the row's key
                   // tiles (stored upward from slot 0) and from the second half
                   // (stored downward from slot cap-1); a sum above cap means
                   // the list overflowed
  int* status;     // device status word
};

__device__ __forceinline__ int row_bound(const ScanParams& p, int i) {
  if (p.bound_kind == 0) return min(i * p.g + p.g, p.L) - 1;
  return i * p.g;
}

template <int D>
struct ScanCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 256;
  static constexpr int KATOMS = D / 64;               // 64-element (128-byte) K slices
  static constexpr int NST = (D == 128) ? 2 : 4;      // key-tile stages in shared memory
  static constexpr int A_BYTES = BM * D * 2;
  static constexpr int B_BYTES = BN * D * 2;
  static constexpr int HIST_BYTES = 128 * BM * 4;     // [128 bin pairs][128 rows], two u16 counts per word
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + A_BYTES;
  static constexpr int OFF_HIST = OFF_B + NST * B_BYTES;
  static constexpr int OFF_MISC = OFF_HIST + HIST_BYTES;  // per-row sample counts of the two groups
  static constexpr int OFF_BAR = OFF_MISC + 2 * BM * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;   // barriers + alignment slack
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 2 * BN;       // double-buffered accumulator
};

template <int D>
__global__ void __launch_bounds__(320, 1)
scan_filter_kernel(const __grid_constant__ CUtensorMap tm_proxy, const __grid_constant__ CUtensorMap tm_keys,
                   ScanParams p) {
  using C = ScanCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A;
  const uint32_t sB = sbase + C::OFF_B;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  int* nsamp = reinterpret_cast<int*>(smem + C::OFF_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // barrier slots: [0,NST) full, [NST,2NST) empty, 2NST a_full, 2NST+1..2 tmem_full, 2NST+3..4 tmem_empty
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::NST + s); };
  const uint32_t a_full = bar0 + 8u * (2 * C::NST);
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::NST + 1 + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::NST + 3 + b); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 136);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bid = blockIdx.x;
  const int h = bid / p.tiles_per_head;
  const int t = p.tiles_per_head - 1 - (bid % p.tiles_per_head);  // longest tiles first
  const int i0 = t * C::BM;
  const int i_last = min(i0 + C::BM, p.G) - 1;
  const int max_bound = row_bound(p, i_last);
  const int nkt = (max_bound + C::BN - 1) / C::BN;                // key tiles needed
  const int nA = (nkt + 1) / 2;                                    // first-half tiles
  const bool sampling = max_bound > p.cap;
  const int ns = sampling ? nkt / p.S : 0;                         // sampled tiles
  const int nsteps = 2 * ns + nkt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(a_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 128);
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

  // Step order: the two sample passes, then the main pass with even steps on
  // the first half of the key tiles and odd steps on the second half, so that
  // accumulator buffer b = step & 1 always belongs to epilogue group b.
  auto step_tile = [&](int step) -> int {
    if (step < ns) return (step + 1) * p.S - 1;
    if (step < 2 * ns) return (step - ns + 1) * p.S - 1;
    const int m = step - 2 * ns;
    return (m & 1) ? nA + (m >> 1) : (m >> 1);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_desc(&tm_proxy);
      tma_prefetch_desc(&tm_keys);
      mbar_arrive_expect_tx(a_full, C::A_BYTES);
      for (int a = 0; a < C::KATOMS; ++a)
        tma_load_3d(sA + a * (C::BM * 128), &tm_proxy, a_full, a * 64, h, i0);
      int issued = 0;
      for (int step = 0; step < nsteps; ++step) {
        const int s = step % C::NST;
        const int use = step / C::NST;
        if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status)) break;
        const int jt = step_tile(step);
        mbar_arrive_expect_tx(full_bar(s), C::B_BYTES);
        for (int a = 0; a < C::KATOMS; ++a)
          tma_load_3d(sB + s * C::B_BYTES + a * (C::BN * 128), &tm_keys, full_bar(s), a * 64, h, jt * C::BN);
        issued = step + 1;
      }
      // Never leave the CTA with a copy still landing in its shared memory.
      mbar_wait_cleanup(a_full, 0);
      for (int step = max(0, issued - C::NST); step < issued; ++step)
        mbar_wait_cleanup(full_bar(step % C::NST), (step / C::NST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BM, C::BN);
      int issued = 0;
      if (mbar_wait(a_full, 0, abort_flag, p.status)) {
        for (int step = 0; step < nsteps; ++step) {
          const int s = step % C::NST;
          const int ab = step & 1;
          if (!mbar_wait(full_bar(s), (step / C::NST) & 1, abort_flag, p.status)) break;
          if (step >= 2 && !mbar_wait(tempty_bar(ab), ((step >> 1) - 1) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + ab * C::BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int a = kk >> 2, k4 = kk & 3;
            const uint64_t adesc = sw128_kmajor_desc(sA + a * (C::BM * 128) + k4 * 32);
            const uint64_t bdesc = sw128_kmajor_desc(sB + s * C::B_BYTES + a * (C::BN * 128) + k4 * 32);
            umma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
          umma_commit(tfull_bar(ab));
          issued = step + 1;
        }
      }
      // All issued MMAs must be complete before the accumulator is released.
      if (issued > 0) mbar_wait_cleanup(tfull_bar((issued - 1) & 1), ((issued - 1) >> 1) & 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two groups of four warps; group e owns accumulator buffer e (steps of
    // parity e).  Thread (e, r) handles row r: group 0 the first half of its
    // key tiles, group 1 the second half.
    const int e = (warp - 2) >> 2;
    const int quarter = warp & 3;               // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;          // proxy row within the tile
    const int i = i0 + r;
    const bool row_ok = i < p.G;
    const int bound = row_ok ? row_bound(p, i) : 0;
    const long long row_id = static_cast<long long>(h) * p.G + i;
    uint2* spill = p.spill + row_id * p.cap;
    int cnt = 0;
    float tau = -__int_as_float(0x7f800000);    // -inf: keep everything
    int n_sample = 0;
    int b1 = -1, rem = 0;
    const bool row_samples = sampling && bound > p.cap;

    auto bin_count = [&](int b) -> int { return (hist[(b >> 1) * C::BM + r] >> ((b & 1) << 4)) & 0xFFFF; };
    auto bin_add = [&](int b) { red_shared_add(smem_u32(&hist[(b >> 1) * C::BM + r]), 1u << ((b & 1) << 4)); };
    auto zero_half_row = [&]() {
      for (int w = 0; w < 64; ++w) hist[(e * 64 + w) * C::BM + r] = 0;
    };
    // Phase changes (sample pass 1 -> 2 -> main); every epilogue thread of both
    // groups takes the same barriers, in the same order.
    int done = sampling ? 0 : 2;
    if (sampling) {
      zero_half_row();
      named_barrier(1, 256);
    }
    auto advance = [&](int target) {
      while (done < target) {
        if (done == 0) {
          // end of sample pass 1: choose the top digit of tau
          nsamp[e * C::BM + r] = n_sample;
          named_barrier(1, 256);
          const int total = nsamp[r] + nsamp[C::BM + r];
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
          named_barrier(1, 256);
          zero_half_row();
          named_barrier(1, 256);
        } else {
          // end of sample pass 2: the second digit, then tau
          named_barrier(1, 256);
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
          }
          // the main pass reuses the histogram space for staging
          named_barrier(1, 256);
        }
        ++done;
      }
    };

    // Main-pass staging for survivor lookups: this thread's 32 values of the
    // current chunk as 8 float4 at [((e*8 + i)*128 + r)*4].
    float* stage = reinterpret_cast<float*>(hist);
    const int stage_base = e * 8 * C::BM;
    auto process = [&](const uint32_t (&v)[32], int j0, int phase) {
      if (j0 >= bound) return;
      const uint32_t live = (j0 + 32 <= bound) ? 0xFFFFFFFFu : ((1u << (bound - j0)) - 1u);
      if (phase == 2) {
        uint32_t m0 = 0, m1 = 0;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          if (__uint_as_float(v[x]) >= tau) m0 |= 1u << x;
          if (__uint_as_float(v[x + 1]) >= tau) m1 |= 2u << x;
        }
        uint32_t m = (m0 | m1) & live;
        if (m == 0) return;
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          reinterpret_cast<uint4*>(stage)[stage_base + q4 * C::BM + r] =
              make_uint4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        while (m) {
          const int x = __ffs(m) - 1;
          m &= m - 1;
          const float sc = stage[((stage_base + (x >> 2) * C::BM) + r) * 4 + (x & 3)];
          if (cnt < p.cap) {
            const uint2 ent = make_uint2(score_key(sc), static_cast<uint32_t>(j0 + x));
            spill[e == 0 ? cnt : p.cap - 1 - cnt] = ent;
          }
          ++cnt;
        }
      } else if (phase == 0) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if ((live >> x) & 1u) bin_add(static_cast<int>(score_key(__uint_as_float(v[x])) >> 24));
        n_sample += __popc(live);
      } else if (b1 >= 0) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
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
    for (int step = e; step < nsteps; step += 2) {
      const int phase = step < ns ? 0 : (step < 2 * ns ? 1 : 2);
      advance(phase);
      // the whole warp decides together: tcgen05.ld below is warp-collective
      if (alive) alive = __all_sync(0xffffffffu, mbar_wait(tfull_bar(e), (step >> 1) & 1, abort_flag, p.status, 256));
      if (!alive) continue;
      tc_fence_after();
      const int jt = step_tile(step);
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + e * C::BN;
      // two register buffers: the TMEM load of chunk c+1 overlaps the work on chunk c
      uint32_t va[32], vb[32];
      tmem_ld_32x32b_x32(taddr, va);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) reg_fence(va[x]);
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; c += 2) {
        tmem_ld_32x32b_x32(taddr + (c + 1) * 32, vb);
        process(va, jt * C::BN + c * 32, phase);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(vb[x]);
        if (c + 2 < C::BN / 32) {
          tmem_ld_32x32b_x32(taddr + (c + 2) * 32, va);
        } else {
          // every column of this accumulator buffer is in registers now
          tc_fence_before();
          mbar_arrive(tempty_bar(e));
        }
        process(vb, jt * C::BN + (c + 1) * 32, phase);
        if (c + 2 < C::BN / 32) {
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) reg_fence(va[x]);
        }
      }
    }
    advance(2);
    if (row_ok) reinterpret_cast<int*>(p.cnt)[2 * row_id + e] = cnt;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace pivot
