"""Statistics of a one-pass refine select with a predicted boundary interval.

The refine kernel's select reads every member score twice (a histogram pass
and a classifying pass), so the next unit's MMAs wait for the second pass to
give TMEM back.  A one-pass alternative predicts, from a sample of the
candidate set, an interval [lo, hi) that holds the K-th largest member score,
then classifies every score once (>= hi: taken; in [lo, hi): kept in a list
that is ranked exactly).  This script measures, on seeded samples of the
L=131072 workload, what that needs: how many keys per member land in the list
(shared memory) and how often the interval misses the K-th score (a miss
redoes the unit).

The sample is what the kernel sees first: chunks 0..s-1, i.e. candidates t
with t mod nch < s (candidate t = r*nch + c sits in chunk c).  Scores are
exact (fp64) dot products of bf16 values, from the oracle's candidate sets.

    python -m oracle.one_pass_select_sim
"""
from __future__ import annotations

import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import synthetic  # noqa: E402


def f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def main(name="C3", units=48, seed=9, sample_chunks=(4, 8), zs=(3.0, 3.5, 4.0)):
    c = synthetic.CONFIGS[name]
    q, k = synthetic.make_prefill(name)
    L, H = c["L"], c["H"]
    g, top_k, Kc = c["g"], c["top_k"], c["Kc"]
    G = (L + g - 1) // g
    rng = np.random.default_rng(seed)
    gi = rng.integers(G // 8, G, size=units).astype(np.int32)
    hi_ = rng.integers(0, H, size=units).astype(np.int32)
    r = oracle.prefill_units(q, k, g, top_k, Kc, oracle.REFINE, gi, hi_, want_cand=True)
    stats = {(s, z): {"list": [], "miss": 0, "n": 0} for s in sample_chunks for z in zs}
    for u in range(units):
        i, h = int(gi[u]), int(hi_[u])
        C = r["cand"][u]
        C = C[C >= 0]
        nch = (len(C) + 127) // 128
        kc = f64(k[C, h])                                  # [nC, d]
        for m in range(min(g, L - i * g)):
            pos = i * g + m
            usable = C < pos
            nv = int(usable.sum())
            K = min(top_k, nv)
            if K == 0 or K == nv:
                continue
            scores = kc @ f64(q[pos, h])
            t = np.arange(len(C))
            kth = np.sort(scores[usable])[::-1][K - 1]     # the K-th largest usable score
            for s in sample_chunks:
                samp = np.sort(scores[usable & ((t % nch) < s)])[::-1]
                ns = samp.size
                p = K / nv
                for z in zs:
                    st = stats[(s, z)]
                    st["n"] += 1
                    mid = p * ns
                    half = z * np.sqrt(ns * p * (1 - p)) + 1
                    r_hi = int(np.floor(mid - half))          # sample rank of the upper edge
                    r_lo = int(np.ceil(mid + half))           # sample rank of the lower edge
                    hi_v = samp[r_hi] if 0 <= r_hi < ns else np.inf
                    lo_v = samp[r_lo] if 0 <= r_lo < ns else -np.inf
                    st["list"].append(int(((scores >= lo_v) & (scores < hi_v) & usable).sum()))
                    if not (lo_v <= kth < hi_v):
                        st["miss"] += 1
    for (s, z), st in stats.items():
        lst = np.array(st["list"])
        print(f"{name}: sample {s} chunks, {z:.1f} sigma: {st['n']} member selections, "
              f"list keys mean {lst.mean():.0f} p99 {np.percentile(lst, 99):.0f} max {lst.max()}, "
              f"misses {st['miss']}")


if __name__ == "__main__":
    main()
