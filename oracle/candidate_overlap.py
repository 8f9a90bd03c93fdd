"""Overlap of the candidate sets of consecutive groups (oracle only).

Refine gathers the key rows of each group's candidate set C (Kc rows of d
bf16 values).  Consecutive groups of one head have similar proxies, so their
candidate sets overlap, and a refine that gathered the union of T consecutive
groups' sets once would read |C_i u ... u C_{i+T-1}| rows instead of the sum
of the |C|.  This script measures that ratio on seeded samples of the
L=131072 workload (whole runs of T consecutive groups, random heads), with the
oracle's candidate sets.

    python -m oracle.candidate_overlap
"""
from __future__ import annotations

import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import synthetic  # noqa: E402


def main(name="C3", runs=6, T_max=8, seed=5):
    c = synthetic.CONFIGS[name]
    q, k = synthetic.make_prefill(name)
    g, top_k, Kc = c["g"], c["top_k"], c["Kc"]
    G = (c["L"] + g - 1) // g
    rng = np.random.default_rng(seed)
    ratios = {T: [] for T in (2, 4, 8) if T <= T_max}
    for _ in range(runs):
        i0 = int(rng.integers(G // 4, G - T_max))   # long prefixes: |C| = Kc
        h = int(rng.integers(0, c["H"]))
        gi = np.arange(i0, i0 + T_max, dtype=np.int32)
        r = oracle.prefill_units(q, k, g, top_k, Kc, oracle.REFINE, gi, np.full(T_max, h, np.int32),
                                 want_cand=True)
        sets = [set(row[row >= 0].tolist()) for row in r["cand"]]
        for T in ratios:
            for a in range(0, T_max, T):
                part = sets[a:a + T]
                ratios[T].append(len(set().union(*part)) / sum(len(s) for s in part))
    for T, v in ratios.items():
        print(f"{name}: union of {T} consecutive groups' candidates / sum of their sizes = "
              f"{np.mean(v):.3f} (min {np.min(v):.3f}, max {np.max(v):.3f}, {len(v)} runs)")


if __name__ == "__main__":
    main()
