"""How much two readings of PIVOT-Refine change the result.

1. Scan extent.  The pages' listing re-runs the proxy scan for every member
   over that member's own prefix (keys j < pos); the method's prose describes
   one shared scan per group.  The library implements the one scan over the
   group's largest prefix (keys j < last) with j >= pos masked per member
   (oracle modes REFINE and REFINE_PER_MEMBER).
2. Proxy precision.  The library rounds the fp32 mean to bf16, the tensor
   cores' operand type; REFINE_FP32_PROXY scans with the fp32 mean instead.

For each, on seeded workloads, the script prints the fraction of output rows
that are identical between the two readings and Recall@k of each against the
dense indexer (rows with pos >= 1).

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


def compare_units(name, q, k, g, top_k, Kc, groups, heads, other=oracle.REFINE_PER_MEMBER, label="per member"):
    L = q.shape[0]
    one = oracle.prefill_units(q, k, g, top_k, Kc, oracle.REFINE, groups, heads)["out"]
    per = oracle.prefill_units(q, k, g, top_k, Kc, other, groups, heads)["out"]
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
          f"recall vs dense: library reading {recall(rows_one, rows_dense):.4f}, "
          f"{label} {recall(rows_per, rows_dense):.4f}")


def main():
    c0 = synthetic.CONFIGS["C0"]
    q0, k0 = synthetic.make_prefill("C0")
    G = (c0["L"] + c0["g"] - 1) // c0["g"]
    gi, hi = np.meshgrid(np.arange(G, dtype=np.int32), np.arange(c0["H"], dtype=np.int32), indexing="ij")
    c1 = synthetic.CONFIGS["C1"]
    q1, k1 = synthetic.make_prefill("C1")
    G1 = (c1["L"] + c1["g"] - 1) // c1["g"]
    rng = np.random.default_rng(11)
    n = 64
    g1 = rng.integers(0, G1, size=n).astype(np.int32)
    h1 = rng.integers(0, c1["H"], size=n).astype(np.int32)
    for other, label in ((oracle.REFINE_PER_MEMBER, "per-member scan"), (oracle.REFINE_FP32_PROXY, "fp32 proxy")):
        print(f"-- library reading vs {label}")
        compare_units("C0 (all rows)", q0, k0, c0["g"], c0["top_k"], c0["Kc"], gi.ravel(), hi.ravel(), other, label)
        compare_units(f"C1 ({n} random groups)", q1, k1, c1["g"], c1["top_k"], c1["Kc"], g1, h1, other, label)


if __name__ == "__main__":
    main()
