"""How much the single-scan reading of PIVOT-Refine changes the result.

The pages' listing re-runs the proxy scan for every member over that member's
own prefix (keys j < pos); the method's prose describes one shared scan per
group.  The library implements the one scan over the group's largest prefix
(keys j < last) with j >= pos masked per member.  This script runs both
readings in the oracle (modes REFINE and REFINE_PER_MEMBER) on seeded
workloads and prints, per workload:

* the fraction of output rows that are identical between the two readings;
* Recall@k of each reading against the dense indexer (rows with pos >= 1).

Oracle only (test infrastructure); it reads nothing from the CUDA library.

    python -m oracle.compare_readings
"""
from __future__ import annotations

import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import synthetic  # noqa: E402


def recall(rows, dense_rows):
    hits = []
    for a, b in zip(rows, dense_rows):
        bb = b[b >= 0]
        if bb.size:
            hits.append(np.intersect1d(a[a >= 0], bb).size / bb.size)
    return float(np.mean(hits))


def compare_units(name, q, k, g, top_k, Kc, groups, heads):
    L = q.shape[0]
    one = oracle.prefill_units(q, k, g, top_k, Kc, oracle.REFINE, groups, heads)["out"]
    per = oracle.prefill_units(q, k, g, top_k, Kc, oracle.REFINE_PER_MEMBER, groups, heads)["out"]
    rows_one, rows_per, rows_dense = [], [], []
    for u, (i, h) in enumerate(zip(groups, heads)):
        pos = np.arange(i * g, min(i * g + g, L))
        keep = pos >= 1
        if not keep.any():
            continue
        d = oracle.dense_units(q, k, top_k, pos[keep].astype(np.int32),
                               np.full(int(keep.sum()), h, np.int32))["out"]
        rows_one.extend(one[u, : len(pos)][keep])
        rows_per.extend(per[u, : len(pos)][keep])
        rows_dense.extend(d)
    same = float(np.mean([np.array_equal(a, b) for a, b in zip(rows_one, rows_per)]))
    print(f"{name}: rows {len(rows_one)}, identical {same:.4f}, "
          f"recall vs dense: one scan {recall(rows_one, rows_dense):.4f}, "
          f"per member {recall(rows_per, rows_dense):.4f}")


def main():
    c = synthetic.CONFIGS["C0"]
    q, k = synthetic.make_prefill("C0")
    G = (c["L"] + c["g"] - 1) // c["g"]
    gi, hi = np.meshgrid(np.arange(G, dtype=np.int32), np.arange(c["H"], dtype=np.int32), indexing="ij")
    compare_units("C0 (all rows)", q, k, c["g"], c["top_k"], c["Kc"], gi.ravel(), hi.ravel())

    c = synthetic.CONFIGS["C1"]
    q, k = synthetic.make_prefill("C1")
    G = (c["L"] + c["g"] - 1) // c["g"]
    rng = np.random.default_rng(11)
    n = 64
    compare_units(f"C1 ({n} random groups)", q, k, c["g"], c["top_k"], c["Kc"],
                  rng.integers(0, G, size=n).astype(np.int32), rng.integers(0, c["H"], size=n).astype(np.int32))


if __name__ == "__main__":
    main()
