"""CPU oracle of the PIVOT query-group indexer -- TEST INFRASTRUCTURE ONLY.

A ctypes front end to ``pivot_oracle.c`` (plain single-threaded C, fp64
arithmetic, full sorts).  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package.  It shares
no code with the CUDA library (``query_group_top_b200``) and neither imports
the other.

Functions work on "units": (group, head) for PIVOT, (position, head) for the
dense indexer, (sequence, head) for decode.  Inputs are bfloat16 bit patterns
(numpy uint16) as produced by :mod:`synthetic`.

Parity status: every function here is pinned by the CPU tests (brute force on
tiny inputs, closed forms, hand-worked fixtures, invariants); see
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pivot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

REFINE, REUSE = 0, 1
# The listing's own Refine ("Show Me The Code", pivot_refine): a proxy scan over
# each member's own prefix.
REFINE_PER_MEMBER = 2
# Proxy precision: the scan operand is the fp32 mean of the group ("fp32") --
# the method -- or that mean rounded once more to bf16 ("bf16"), a variant.
PROXY_PRECISIONS = ("fp32", "bf16")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/liboracle.so`` (if stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_prefill_units.argtypes = [P, P, i, i, i, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_dense_units.argtypes = [P, P, i, i, i, i, i, P, P, P, P, P]
        lib.oracle_decode_units.argtypes = [P, P, P, i, i, i, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P]
        lib.oracle_sparse_attention.argtypes = [P, P, P, P, P, i, i, i, i, i, P]
        for f in (lib.oracle_prefill_units, lib.oracle_dense_units, lib.oracle_decode_units,
                  lib.oracle_sparse_attention):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def _proxy_flag(proxy):
    if proxy not in PROXY_PRECISIONS:
        raise ValueError(f"proxy must be one of {PROXY_PRECISIONS}")
    return 1 if proxy == "bf16" else 0


def prefill_units(q, k, g, top_k, Kc, mode, groups, heads, want_cand=False, proxy="fp32"):
    """PIVOT (Refine mode=0, Reuse mode=1, per-member-scan Refine mode=2) on the
    listed (group, head) units; `proxy` is the scan operand's precision.

    Returns dict: out [n,g,top_k] int32, score [n,g,top_k] f64, edge [n,g,2] f64,
    cand [n,Kc] int32 and cand_edge [n,2] (Refine), member_cand_edge [n,g,2]
    (mode 2: each member's own Kc-th and (Kc+1)-th proxy scores), proxy [n,d]
    float32 (the fp32 mean) and proxy_bf16 [n,d] uint16 (its bf16 rounding).
    """
    lib = _load()
    pb = _proxy_flag(proxy)
    q = _u16(q)
    k = _u16(k)
    L, H, d = q.shape
    groups = np.ascontiguousarray(groups, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    n = groups.size
    out = np.empty((n, g, top_k), np.int32)
    sc = np.empty((n, g, top_k), np.float64)
    edge = np.empty((n, g, 2), np.float64)
    cand = np.empty((n, Kc), np.int32) if want_cand else None
    cedge = np.empty((n, 2), np.float64)
    p32 = np.empty((n, d), np.float32)
    p16 = np.empty((n, d), np.uint16)
    medge = np.empty((n, g, 2), np.float64)
    rc = lib.oracle_prefill_units(_p(q), _p(k), L, H, d, g, top_k, Kc, mode, pb, n, _p(groups), _p(heads),
                                  _p(out), _p(sc), _p(edge), _p(cand), _p(cedge), _p(p32), _p(p16), _p(medge))
    if rc != 0:
        raise ValueError("oracle_prefill_units rejected its arguments")
    return dict(out=out, score=sc, edge=edge, cand=cand, cand_edge=cedge, member_cand_edge=medge, proxy=p32,
                proxy_bf16=p16)


def prefill(q, k, g, top_k, Kc, mode, want_cand=False, proxy="fp32"):
    """Full prefill PIVOT: out [L,H,top_k] int32 plus per-row scores/edges."""
    L, H, _ = q.shape
    G = (L + g - 1) // g
    gi, hi = np.meshgrid(np.arange(G, dtype=np.int32), np.arange(H, dtype=np.int32), indexing="ij")
    r = prefill_units(q, k, g, top_k, Kc, mode, gi.ravel(), hi.ravel(), want_cand, proxy)
    # [G*H, g, k] -> [G, H, g, k] -> [G, g, H, k] -> [G*g, H, k] -> [:L]
    def fold(a):
        a = a.reshape(G, H, g, *a.shape[2:])
        a = np.swapaxes(a, 1, 2).reshape(G * g, H, *a.shape[3:])
        return np.ascontiguousarray(a[:L])
    res = dict(out=fold(r["out"]), score=fold(r["score"]), edge=fold(r["edge"]),
               member_cand_edge=fold(r["member_cand_edge"]),
               cand_edge=r["cand_edge"].reshape(G, H, 2), proxy=r["proxy"].reshape(G, H, -1),
               proxy_bf16=r["proxy_bf16"].reshape(G, H, -1))
    if want_cand:
        res["cand"] = r["cand"].reshape(G, H, Kc)
    return res


def dense_units(q, k, top_k, positions, heads):
    """Dense indexer on (position, head) units: out [n,top_k], score, edge [n,2]."""
    lib = _load()
    q = _u16(q)
    k = _u16(k)
    L, H, d = q.shape
    positions = np.ascontiguousarray(positions, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    n = positions.size
    out = np.empty((n, top_k), np.int32)
    sc = np.empty((n, top_k), np.float64)
    edge = np.empty((n, 2), np.float64)
    rc = lib.oracle_dense_units(_p(q), _p(k), L, H, d, top_k, n, _p(positions), _p(heads),
                                _p(out), _p(sc), _p(edge))
    if rc != 0:
        raise ValueError("oracle_dense_units rejected its arguments")
    return dict(out=out, score=sc, edge=edge)


def dense(q, k, top_k):
    """Full dense indexer: out [L,H,top_k]."""
    L, H, _ = q.shape
    pi, hi = np.meshgrid(np.arange(L, dtype=np.int32), np.arange(H, dtype=np.int32), indexing="ij")
    r = dense_units(q, k, top_k, pi.ravel(), hi.ravel())
    return dict(out=r["out"].reshape(L, H, top_k), score=r["score"].reshape(L, H, top_k),
                edge=r["edge"].reshape(L, H, 2))


def decode_units(q, kcache, cu_seqlens, g, top_k, Kc, mode, seqs, heads, want_cand=False, proxy="fp32"):
    """Decode PIVOT on (sequence, head) units; q [B,g,H,d], kcache [rows,H,d]."""
    lib = _load()
    pb = _proxy_flag(proxy)
    q = _u16(q)
    kcache = _u16(kcache)
    B, gq, H, d = q.shape
    if gq != g:
        raise ValueError("q's second axis must be the group size g")
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    seqs = np.ascontiguousarray(seqs, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    n = seqs.size
    out = np.empty((n, g, top_k), np.int32)
    sc = np.empty((n, g, top_k), np.float64)
    edge = np.empty((n, g, 2), np.float64)
    cand = np.empty((n, Kc), np.int32) if want_cand else None
    cedge = np.empty((n, 2), np.float64)
    p32 = np.empty((n, d), np.float32)
    p16 = np.empty((n, d), np.uint16)
    rc = lib.oracle_decode_units(_p(q), _p(kcache), _p(cu), B, H, d, g, top_k, Kc, mode, pb, n,
                                 _p(seqs), _p(heads), _p(out), _p(sc), _p(edge), _p(cand),
                                 _p(cedge), _p(p32), _p(p16))
    if rc != 0:
        raise ValueError("oracle_decode_units rejected its arguments")
    return dict(out=out, score=sc, edge=edge, cand=cand, cand_edge=cedge, proxy=p32, proxy_bf16=p16)


def sparse_attention(q, k, v, idx, cu_seqlens=None, g=1):
    """The attention that consumes the index rows: out[r, h] = softmax over the
    row's valid indices of (q . k_j) * d^-1/2, applied to v_j (fp64); rows
    without a valid index give zeros.  Prefill: q, k, v bf16 bits [R, H, d].
    Decode: q [B, g, H, d] or [B*g, H, d], k and v the packed cache, index j of
    sequence b at cache row cu_seqlens[b] + j.  idx int32 [..., H, top_k].
    Returns float64 [R, H, d] (R = query rows)."""
    lib = _load()
    q = _u16(q)
    k = _u16(k)
    v = _u16(v)
    H, d = q.shape[-2], q.shape[-1]
    R = q.size // (H * d)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    top_k = idx.shape[-1]
    if idx.size != R * H * top_k or k.shape != v.shape:
        raise ValueError("sparse_attention: shapes do not agree")
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    out = np.empty((R, H, d), np.float64)
    rc = lib.oracle_sparse_attention(_p(q), _p(k), _p(v), _p(idx), _p(cu), R, H, d, g, top_k, _p(out))
    if rc != 0:
        raise ValueError("oracle_sparse_attention rejected its arguments")
    return out
