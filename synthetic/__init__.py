"""Seeded synthetic inputs for the PIVOT indexer (shared by the tests, the bench and the oracle runs).

This module holds no arithmetic of the indexer itself: it only draws random
numbers, shapes them into the workloads' query/key tensors and rounds them to
bfloat16 once, at the boundary. Every tensor it returns is a numpy array of
bfloat16 *bit patterns* (dtype uint16), so that the CUDA path and the oracle
consume exactly the same values.

Workload recipes (stand-ins for the model activations that the pages measure on
and that are not available here):

* ``iid``      -- q then k drawn i.i.d. N(0,1) in fp32 (the pages' demo shape,
                  "PIVOT explained", section "Show Me The Code").
* ``prefill``  -- keys N(0,1) with a random fraction of positions scaled by a
                  constant (long-tailed scores, the pages' Observation 2); queries
                  an AR(1) sequence along positions per head and channel,
                  q_0 ~ N(0,1), q_t = rho*q_{t-1} + sqrt(1-rho^2)*eps_t (high
                  neighbour overlap, Observation 1).
* ``decode``   -- a batch of sequences with context lengths drawn uniformly in
                  [lo, hi]; each sequence's cache holds its n_b context keys plus
                  the g keys of the step being decoded (prefill key generator per
                  sequence); the g step queries are an AR(1) chain.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "bf16_from_f32", "bf16_to_f32", "gen_iid", "gen_prefill", "gen_decode",
    "DecodeInputs", "CONFIGS",
]


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (round to nearest, ties to even); returns uint16 bits.

    Inputs must be finite (the generators never produce NaN or Inf).
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to fp32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _ar1(eps: np.ndarray, rho: float) -> np.ndarray:
    """AR(1) along axis 0 in fp32 via scipy's IIR filter: y_0 = eps_0, y_t = rho*y_{t-1} + sqrt(1-rho^2)*eps_t."""
    from scipy.signal import lfilter
    b = np.float32(math.sqrt(1.0 - rho * rho))
    x = eps.astype(np.float32, copy=True)
    x[0] = x[0] / b          # so that y_0 = b * (eps_0 / b) = eps_0
    y = lfilter(np.array([b], dtype=np.float32), np.array([1.0, -rho], dtype=np.float32), x, axis=0)
    return y.astype(np.float32, copy=False)


def gen_iid(L: int, H: int, d: int, seed: int = 0):
    """q then k, both i.i.d. N(0,1) fp32 [L,H,d] from ``default_rng(seed)``, rounded to bf16."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, H, d), dtype=np.float32)
    k = rng.standard_normal((L, H, d), dtype=np.float32)
    return bf16_from_f32(q), bf16_from_f32(k)


def _keys(rng, L, H, d, heavy_frac, heavy_scale):
    k = rng.standard_normal((L, H, d), dtype=np.float32)
    n_heavy = int(round(heavy_frac * L))
    if n_heavy > 0:
        pos = rng.choice(L, size=n_heavy, replace=False)
        k[pos] *= np.float32(heavy_scale)
    return k


def gen_prefill(L: int, H: int, d: int, seed: int, rho: float = 0.95,
                heavy_frac: float = 0.01, heavy_scale: float = 4.0):
    """Prefill inputs: heavy-tailed keys, AR(1) queries; returns (q_bits, k_bits) [L,H,d] uint16."""
    rng = np.random.default_rng(seed)
    k = _keys(rng, L, H, d, heavy_frac, heavy_scale)
    eps = rng.standard_normal((L, H, d), dtype=np.float32)
    q = _ar1(eps, rho)
    return bf16_from_f32(q), bf16_from_f32(k)


@dataclass
class DecodeInputs:
    q: np.ndarray           # [B, g, H, d] uint16 (bf16 bits)
    kcache: np.ndarray      # [sum_b (n_b + g), H, d] uint16 (bf16 bits)
    cu_seqlens: np.ndarray  # [B+1] int32, cache row offsets
    n_ctx: np.ndarray       # [B] int32, context lengths n_b


def gen_decode(B: int, H: int, d: int, g: int, seed: int, lo: int, hi: int,
               rho: float = 0.95, heavy_frac: float = 0.01, heavy_scale: float = 4.0,
               key_fn=None) -> DecodeInputs:
    """Decode inputs for one multi-token-prediction step of g queries per sequence.

    n_b ~ U{lo..hi} (inclusive) from ``default_rng(seed)``; sequence b's keys
    come from ``default_rng([seed, b])`` with the prefill key generator
    (n_b + g rows); its g queries from ``default_rng([seed, b, 1])`` as an AR(1)
    chain.  ``key_fn(b, rows_bits)`` may be given to receive each sequence's
    key rows instead of materialising the whole cache on the host.
    """
    rng = np.random.default_rng(seed)
    n_ctx = rng.integers(lo, hi, size=B, endpoint=True).astype(np.int32)
    lens = n_ctx.astype(np.int64) + g
    cu = np.zeros(B + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    q = np.empty((B, g, H, d), dtype=np.uint16)
    kc = None if key_fn is not None else np.empty((int(cu[-1]), H, d), dtype=np.uint16)
    a = np.float32(rho)
    b_ = np.float32(math.sqrt(1.0 - rho * rho))
    for b in range(B):
        r = np.random.default_rng([seed, b])
        kb = bf16_from_f32(_keys(r, int(lens[b]), H, d, heavy_frac, heavy_scale))
        if key_fn is not None:
            key_fn(b, kb)
        else:
            kc[cu[b]:cu[b + 1]] = kb
        rq = np.random.default_rng([seed, b, 1])
        eps = rq.standard_normal((g, H, d), dtype=np.float32)
        qq = np.empty_like(eps)
        qq[0] = eps[0]
        for i in range(1, g):
            qq[i] = a * qq[i - 1] + b_ * eps[i]
        q[b] = bf16_from_f32(qq)
    if cu[-1] >= 2**31:
        raise ValueError("decode cache too large for int32 offsets")
    return DecodeInputs(q=q, kcache=kc, cu_seqlens=cu.astype(np.int32), n_ctx=n_ctx)


# The five workloads (sizes, selection parameters and generator settings).
CONFIGS = {
    "C0": dict(kind="iid", L=1024, H=8, d=64, top_k=64, g=8, Kc=128, seed=0),
    "C1": dict(kind="prefill", L=8192, H=16, d=128, top_k=256, g=8, Kc=512, seed=1,
               rho=0.95, heavy_frac=0.01, heavy_scale=4.0),
    "C2": dict(kind="prefill", L=32768, H=32, d=128, top_k=2048, g=8, Kc=4096, seed=2,
               rho=0.95, heavy_frac=0.01, heavy_scale=4.0),
    "C3": dict(kind="prefill", L=131072, H=16, d=128, top_k=2048, g=16, Kc=4096, seed=3,
               rho=0.9, heavy_frac=0.005, heavy_scale=5.0),
    "C4": dict(kind="decode", B=64, H=16, d=128, g=2, top_k=2048, Kc=4096, seed=4,
               lo=16384, hi=131072, rho=0.95, heavy_frac=0.01, heavy_scale=4.0),
}


def make_prefill(name: str):
    """Generate the (q, k) bf16-bit tensors of a prefill workload by name."""
    c = CONFIGS[name]
    if c["kind"] == "iid":
        return gen_iid(c["L"], c["H"], c["d"], c["seed"])
    return gen_prefill(c["L"], c["H"], c["d"], c["seed"], c["rho"], c["heavy_frac"], c["heavy_scale"])


def gen_decode_device(B: int, H: int, d: int, g: int, seed: int, lo: int, hi: int,
                      rho: float = 0.95, heavy_frac: float = 0.01, heavy_scale: float = 4.0,
                      device="cuda", first: int = 0, count=None):
    """Large decode batches drawn on the GPU (same recipe as ``gen_decode``).

    Context lengths, heavy-key positions and the step queries come from numpy
    exactly as in ``gen_decode``; the key rows themselves are drawn with
    torch's device generator seeded per sequence (seed * 1000003 + b), in fp32,
    then rounded to bf16 (round to nearest even).  Returns torch tensors
    (q [B,g,H,d] bf16, kcache [rows,H,d] bf16, cu_seqlens [B+1] int32) on the
    device and the numpy context lengths.  Use ``kcache[cu[b]:cu[b+1]]`` to
    read a sequence back for a CPU check.  ``first`` and ``count`` draw only
    sequences [first, first+count) of the B-sequence batch (the same values
    as in the whole batch), packed from cache row 0.
    """
    import torch
    rng = np.random.default_rng(seed)
    n_all = rng.integers(lo, hi, size=B, endpoint=True).astype(np.int32)
    count = B - first if count is None else count
    if not 0 <= first <= first + count <= B:
        raise ValueError("gen_decode_device: sequences out of range")
    n_ctx = n_all[first:first + count]
    seqs = range(first, first + count)
    lens = n_ctx.astype(np.int64) + g
    cu = np.zeros(count + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    if cu[-1] >= 2**31:
        raise ValueError("decode cache too large for int32 offsets")
    kc = torch.empty((int(cu[-1]), H, d), dtype=torch.bfloat16, device=device)
    q = np.empty((count, g, H, d), dtype=np.uint16)
    a = np.float32(rho)
    b_ = np.float32(math.sqrt(1.0 - rho * rho))
    gen = torch.Generator(device=device)
    for i_b, b in enumerate(seqs):
        n = int(lens[i_b])
        gen.manual_seed(seed * 1000003 + b)
        kb = torch.randn((n, H, d), generator=gen, device=device, dtype=torch.float32)
        n_heavy = int(round(heavy_frac * n))
        if n_heavy > 0:
            pos = np.random.default_rng([seed, b]).choice(n, size=n_heavy, replace=False)
            kb[torch.from_numpy(pos).to(device)] *= heavy_scale
        kc[int(cu[i_b]):int(cu[i_b + 1])] = kb.to(torch.bfloat16)
        del kb
        rq = np.random.default_rng([seed, b, 1])
        eps = rq.standard_normal((g, H, d), dtype=np.float32)
        qq = np.empty_like(eps)
        qq[0] = eps[0]
        for i in range(1, g):
            qq[i] = a * qq[i - 1] + b_ * eps[i]
        q[i_b] = bf16_from_f32(qq)
    qd = torch.from_numpy(q.view(np.int16)).to(device).view(torch.bfloat16)
    cud = torch.from_numpy(cu.astype(np.int32)).to(device)
    return qd, kc, cud, n_ctx
