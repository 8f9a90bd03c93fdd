"""Brute-force restatement of the PIVOT indexer for tiny inputs (pins the oracle).

Written independently of ``oracle/pivot_oracle.c``: numpy float64 arithmetic,
a full ``np.lexsort`` ranking per row, torch's own fp32->bf16 conversion for
the proxy rounding.  Only for small sizes.
"""
import numpy as np
import torch


def decode_bf16(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_proxy(mean64):
    """fp64 -> fp32 -> bf16 (torch's round-to-nearest-even) -> float64 (the bf16 proxy variant)."""
    t = torch.from_numpy(np.asarray(mean64, dtype=np.float64).astype(np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def top_set(scores, idx, K):
    """Indices of the K best (score desc, index asc), returned ascending."""
    if K <= 0 or len(idx) == 0:
        return np.zeros(0, np.int64)
    order = np.lexsort((idx, -scores))
    return np.sort(idx[order[:K]])


def pad(sel, width):
    r = -np.ones(width, np.int64)
    r[:len(sel)] = sel
    return r


def dense(qb, kb, top_k):
    q = decode_bf16(qb)
    k = decode_bf16(kb)
    L, H, _ = q.shape
    out = -np.ones((L, H, top_k), np.int64)
    for h in range(H):
        S = q[:, h] @ k[:, h].T          # S[pos, j]
        for pos in range(L):
            j = np.arange(pos)
            out[pos, h] = pad(top_set(S[pos, :pos], j, min(top_k, pos)), top_k)
    return out


def _group_rows(q, k, members, positions, s, last, top_k, Kc, mode, proxy_prec="fp32"):
    mean = q[members].mean(axis=0)
    if proxy_prec == "fp32":
        proxy = mean.astype(np.float32).astype(np.float64)
    else:   # the bf16 variant: the fp32 mean rounded once more, to bf16
        proxy = round_proxy(mean)
    rows = []
    if mode == 1:
        j = np.arange(s)
        sel = top_set(k[:s] @ proxy, j, min(top_k, s))
        rows = [pad(sel, top_k) for _ in members]
    elif mode == 2:
        # the listing's Refine: each member scans its own prefix j < pos
        for m, pos in zip(members, positions):
            C = top_set(k[:pos] @ proxy, np.arange(pos), min(Kc, pos))
            r = k[C] @ q[m]
            rows.append(pad(top_set(r, C, min(top_k, len(C))), top_k))
    else:
        j = np.arange(last)
        C = top_set(k[:last] @ proxy, j, min(Kc, last))
        for m, pos in zip(members, positions):
            V = C[C < pos]
            r = k[V] @ q[m]
            rows.append(pad(top_set(r, V, min(top_k, len(V))), top_k))
    return proxy, rows


def prefill(qb, kb, g, top_k, Kc, mode, proxy_prec="fp32"):
    q = decode_bf16(qb)
    k = decode_bf16(kb)
    L, H, _ = q.shape
    out = -np.ones((L, H, top_k), np.int64)
    for h in range(H):
        for s in range(0, L, g):
            e = min(s + g, L)
            mem = list(range(s, e))
            _, rows = _group_rows(q[:, h], k[:, h], mem, mem, s, e - 1, top_k, Kc, mode, proxy_prec)
            for pos, r in zip(mem, rows):
                out[pos, h] = r
    return out


def decode(qb, kcb, cu, g, top_k, Kc, mode, proxy_prec="fp32"):
    q = decode_bf16(qb)          # [B, g, H, d]
    kc = decode_bf16(kcb)        # [rows, H, d]
    B, _, H, _ = q.shape
    out = -np.ones((B, g, H, top_k), np.int64)
    for b in range(B):
        n_b = int(cu[b + 1] - cu[b] - g)
        keys = kc[cu[b]:cu[b + 1]]
        for h in range(H):
            pos = [n_b + i for i in range(g)]
            _, rows = _group_rows(q[b, :, h], keys[:, h], list(range(g)), pos, n_b, n_b + g - 1,
                                  top_k, Kc, mode, proxy_prec)
            for i, r in enumerate(rows):
                out[b, i, h] = r
    return out
