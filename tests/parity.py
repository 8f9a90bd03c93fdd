"""Comparison of GPU index rows with the oracle's, under the parity rules.

A row must equal the oracle's row exactly, unless it is a near tie: the
oracle's k-th and (k+1)-th scores of that row's final select (or, for Refine,
its group's Kc-th and (Kc+1)-th proxy scores) differ by less than 1e-4
relative.  Exempt rows must still be valid rows (ascending, unique, causal).
Reported scores must agree within 1e-3 relative (floor 1).
"""
import numpy as np

REL_TIE = 1e-4
REL_SCORE = 1e-3


def near_tie(edge, rel=REL_TIE):
    e0, e1 = edge[..., 0], edge[..., 1]
    ok = np.isfinite(e0) & np.isfinite(e1)
    gap = np.abs(e0 - e1)
    return ok & (gap < rel * np.maximum(np.abs(e0), np.abs(e1)))


def valid_rows(rows, pos):
    """rows [..., k] int, pos [...] int: ascending valid prefix, -1 padding, all < pos."""
    v = rows >= 0
    ok = np.all(np.diff(v.astype(np.int8), axis=-1) <= 0, axis=-1)
    big = np.where(v, rows, np.iinfo(np.int32).max)
    ok &= np.all((np.diff(big, axis=-1) > 0) | ~v[..., 1:], axis=-1)
    ok &= np.all(~v | (rows < pos[..., None]), axis=-1)
    return ok


def compare(got, want, edge, pos, cand_edge=None, got_scores=None, want_scores=None):
    """Returns dict(exact, exempt, mismatch, bad_rows, score_bad)."""
    got = np.asarray(got)
    eq = np.all(got == want, axis=-1)
    ex = near_tie(edge)
    if cand_edge is not None:
        ex = ex | near_tie(cand_edge)
    mism = ~eq & ~ex
    res = dict(exact=int(eq.sum()), exempt=int((~eq & ex).sum()), mismatch=int(mism.sum()),
               invalid=int((~valid_rows(got, np.asarray(pos))).sum()))
    if mism.any():
        idx = np.argwhere(mism)[:3]
        res["examples"] = [(tuple(i), got[tuple(i)][:8].tolist(), want[tuple(i)][:8].tolist()) for i in idx]
    if got_scores is not None:
        m = eq[..., None] & (want >= 0)
        a = np.asarray(got_scores, dtype=np.float64)[m]
        b = want_scores[m]
        res["score_bad"] = int((np.abs(a - b) > REL_SCORE * np.maximum(np.abs(b), 1.0)).sum())
    return res


def assert_parity(res, what=""):
    assert res["mismatch"] == 0, f"{what}: {res}"
    assert res["invalid"] == 0, f"{what}: {res}"
    assert res.get("score_bad", 0) == 0, f"{what}: {res}"


def oracle_threads(fn, q, k, g, top_k, Kc, mode, units_a, units_b, threads=None, **kw):
    """Runs an oracle *_units function over its units on several host threads
    (the oracle is plain C called through ctypes, which releases the GIL, and
    keeps no global state) and joins the per-unit results in unit order."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    n = len(units_a)
    threads = threads or max(1, min(len(os.sched_getaffinity(0)), 32, n))
    cuts = np.linspace(0, n, threads + 1).astype(int)
    parts = [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
    with ThreadPoolExecutor(len(parts)) as ex:
        res = list(ex.map(lambda ab: fn(q, k, g, top_k, Kc, mode, units_a[ab[0]:ab[1]], units_b[ab[0]:ab[1]], **kw),
                          parts))
    out = {}
    for key in res[0]:
        vals = [r[key] for r in res]
        out[key] = None if vals[0] is None else np.concatenate(vals, axis=0)
    return out
