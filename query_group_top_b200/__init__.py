"""B200 (sm_100a) PIVOT query-group indexer -- Python binding.

Argument marshalling only: every step runs in the CUDA kernels of the in-tree
``libpivot.so`` (C ABI declared in ``include/pivot.h``).  PyTorch supplies
device memory and streams.  There is no CPU fallback: without the built
library or an sm_100 device every call raises.

    idx = pivot_index(q, k, g=16, top_k=2048, Kc=4096, mode=REFINE)   # [L, H, top_k] int32
    idx = pivot_index(q, k, 16, 2048, 4096, REFINE, proxy="bf16")      # the bf16-proxy variant
    idx = dense_index(q, k, top_k=2048)
    idx = pivot_decode_index(q, kcache, cu_seqlens, g=2, top_k=2048, Kc=4096, max_seqlen=...)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["REFINE", "REUSE", "PROXY_BF16", "PER_MEMBER_SCAN", "PivotError", "pivot_index", "dense_index", "pivot_decode_index",
           "pivot_decode_index_paged", "sparse_attention",
           "sync_status", "trace_enable", "trace_collect", "library_path", "load_library", "EXPORTED",
           "head_range"]

REFINE, REUSE = 0, 1
PROXY_BF16 = 0x100          # option bit of `mode`: scan with the bf16-rounded mean
PER_MEMBER_SCAN = 0x200     # option bit of REFINE: each member's own-prefix candidate set
FLAG_TIMEOUT, FLAG_BADLEN, FLAG_FALLBACK, FLAG_NOCONVERGE = 1, 2, 4, 8

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libpivot.so")
_lib = None

# Every symbol declared in include/pivot.h.
EXPORTED = (
    "pivot_index", "dense_index", "pivot_decode_index",
    "pivot_workspace_size", "pivot_index_ws", "dense_workspace_size", "dense_index_ws",
    "pivot_decode_workspace_size", "pivot_decode_index_ws", "pivot_sync_status", "pivot_last_error",
    "pivot_trace_enable", "pivot_trace_collect", "pivot_decode_index_noalloc",
    "pivot_index_ex", "pivot_decode_index_ex", "pivot_set_wait_limit", "pivot_decode_index_paged",
    "pivot_sparse_attention",
)


class PivotError(RuntimeError):
    pass


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libpivot.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise PivotError(f"{_LIB_PATH} is missing: build it with `python -m query_group_top_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "pivot_index": ([P, P, I, I, I, I, I, I, I, P, P], I),
        "dense_index": ([P, P, I, I, I, I, P, P], I),
        "pivot_decode_index": ([P, P, P, I, I, I, I, I, I, I, I, P, P], I),
        "pivot_workspace_size": ([I, I, I, I, I, I, I], Z),
        "pivot_index_ws": ([P, P, I, I, I, I, I, I, I, P, P, P, Z, P], I),
        "dense_workspace_size": ([I, I, I, I], Z),
        "dense_index_ws": ([P, P, I, I, I, I, P, P, P, Z, P], I),
        "pivot_decode_workspace_size": ([I, I, I, I, I, I, I, I], Z),
        "pivot_decode_index_ws": ([P, P, P, I, I, I, I, I, I, I, I, P, P, P, Z, P], I),
        "pivot_sync_status": ([P, ctypes.POINTER(I)], I),
        "pivot_last_error": ([], ctypes.c_char_p),
        "pivot_trace_enable": ([I], I),
        "pivot_trace_collect": ([ctypes.c_char_p, Z, P, P, I], I),
        "pivot_decode_index_noalloc": ([P, P, P, I, I, I, I, I, I, I, I, P, P, P], I),
        "pivot_index_ex": ([P, P, I, I, I, I, I, I, I, P, P, P, P, P, Z, P], I),
        "pivot_decode_index_ex": ([P, P, P, I, I, I, I, I, I, I, I, P, P, P, P, P, Z, P], I),
        "pivot_decode_index_paged": ([P, P, P, P, I, I, I, I, I, I, I, I, I, I, P, P, P, Z, P], I),
        "pivot_sparse_attention": ([P, P, P, P, P, I, I, I, I, I, P, P], I),
        "pivot_set_wait_limit": ([ctypes.c_ulonglong], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _err(lib, rc: int):
    if rc != 0:
        raise PivotError(f"pivot error {rc}: {lib.pivot_last_error().decode(errors='replace')}")


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check_bf16(name, t, ndim):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise PivotError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise PivotError(f"{name} must be bfloat16 (got {t.dtype})")
    if t.dim() != ndim or not t.is_contiguous():
        raise PivotError(f"{name} must be a contiguous {ndim}-d tensor")


_ws = {}


def _workspace(nbytes: int, device, stream_ptr: int) -> torch.Tensor:
    """Per (device, stream) cached workspace, grown on demand."""
    key = (device, stream_ptr)
    t = _ws.get(key)
    if t is None or t.numel() < nbytes:
        _ws.pop(key, None)
        t = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
        _ws[key] = t
    return t


def _out(out, shape, dtype, device, name):
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype or not out.is_contiguous() or out.device != device:
        raise PivotError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}")
    return out


def _mode_bits(mode, proxy, scan="group"):
    if mode not in (REFINE, REUSE):
        raise PivotError("mode must be REFINE or REUSE")
    if proxy not in ("fp32", "bf16"):
        raise PivotError('proxy must be "fp32" (the method) or "bf16" (the variant)')
    if scan not in ("group", "member") or (scan == "member" and mode != REFINE):
        raise PivotError('scan must be "group" (the method) or, with REFINE, "member" (the listing\'s variant)')
    return mode | (PROXY_BF16 if proxy == "bf16" else 0) | (PER_MEMBER_SCAN if scan == "member" else 0)


def _ptr(t):
    return None if t is None else t.data_ptr()


def pivot_index(q, k, g, top_k, Kc, mode=REFINE, out=None, out_scores=None, stream=None, proxy="fp32",
                out_proxy=None, out_cand=None, scan="group"):
    """PIVOT prefill indexer: q, k bf16 [L, H, d] -> int32 [L, H, top_k] (ascending, -1 padded).

    proxy: "fp32" scans with the fp32 group mean (the method), "bf16" with its
    bf16 rounding (a variant).  scan: "group" takes one candidate set per
    group (the method), "member" (Refine only) each member's own top-Kc over
    its prefix (the listing's variant).  out_proxy (float32 [G, H, d]) and
    out_cand (int32 [G, H, Kc], Refine only; [L, H, Kc] with scan="member")
    receive the groups' proxies and candidate sets when given (G = ceil(L / g)).
    """
    lib = load_library()
    bits = _mode_bits(mode, proxy, scan)
    _check_bf16("q", q, 3)
    _check_bf16("k", k, 3)
    if q.shape != k.shape:
        raise PivotError("q and k must have the same shape [L, H, d]")
    L, H, d = q.shape
    out = _out(out, (L, H, top_k), torch.int32, q.device, "out")
    if out_scores is not None:
        out_scores = _out(out_scores, (L, H, top_k), torch.float32, q.device, "out_scores")
    G = (L + g - 1) // g if g >= 1 else 0
    if out_proxy is not None:
        out_proxy = _out(out_proxy, (G, H, d), torch.float32, q.device, "out_proxy")
    if out_cand is not None:
        out_cand = _out(out_cand, (L if scan == "member" else G, H, Kc), torch.int32, q.device, "out_cand")
    sp = _stream_ptr(stream)
    n = lib.pivot_workspace_size(L, H, d, g, top_k, Kc, bits)
    ws = _workspace(n, q.device, sp)
    if out_proxy is None and out_cand is None:
        rc = lib.pivot_index_ws(q.data_ptr(), k.data_ptr(), L, H, d, g, top_k, Kc, bits, out.data_ptr(),
                                _ptr(out_scores), ws.data_ptr(), ws.numel(), sp)
    else:
        rc = lib.pivot_index_ex(q.data_ptr(), k.data_ptr(), L, H, d, g, top_k, Kc, bits, out.data_ptr(),
                                _ptr(out_scores), _ptr(out_proxy), _ptr(out_cand), ws.data_ptr(), ws.numel(), sp)
    _err(lib, rc)
    return out


def dense_index(q, k, top_k, out=None, out_scores=None, stream=None):
    """Dense per-query indexer: q, k bf16 [L, H, d] -> int32 [L, H, top_k]."""
    lib = load_library()
    _check_bf16("q", q, 3)
    _check_bf16("k", k, 3)
    if q.shape != k.shape:
        raise PivotError("q and k must have the same shape [L, H, d]")
    L, H, d = q.shape
    out = _out(out, (L, H, top_k), torch.int32, q.device, "out")
    if out_scores is not None:
        out_scores = _out(out_scores, (L, H, top_k), torch.float32, q.device, "out_scores")
    sp = _stream_ptr(stream)
    n = lib.dense_workspace_size(L, H, d, top_k)
    ws = _workspace(n, q.device, sp)
    rc = lib.dense_index_ws(q.data_ptr(), k.data_ptr(), L, H, d, top_k, out.data_ptr(),
                            None if out_scores is None else out_scores.data_ptr(), ws.data_ptr(), ws.numel(), sp)
    _err(lib, rc)
    return out


def pivot_decode_index(q, kcache, cu_seqlens, g, top_k, Kc, mode=REFINE, max_seqlen=None, out=None,
                       out_scores=None, stream=None, proxy="fp32", out_proxy=None, out_cand=None):
    """PIVOT decode indexer: q bf16 [B, g, H, d], kcache bf16 [rows, H, d], cu_seqlens int32 [B+1]
    (device) -> int32 [B, g, H, top_k].  max_seqlen bounds every sequence's cache rows.
    out_proxy (float32 [B, H, d]) and out_cand (int32 [B, H, Kc], Refine only) as in pivot_index."""
    lib = load_library()
    bits = _mode_bits(mode, proxy)
    _check_bf16("q", q, 4)
    _check_bf16("kcache", kcache, 3)
    B, gq, H, d = q.shape
    if gq != g:
        raise PivotError("q's second axis must equal g")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.numel() != B + 1:
        raise PivotError("cu_seqlens must be an int32 CUDA tensor of B+1 offsets")
    if max_seqlen is None:
        raise PivotError("max_seqlen (an upper bound on cache rows per sequence) is required")
    out = _out(out, (B, g, H, top_k), torch.int32, q.device, "out")
    if out_scores is not None:
        out_scores = _out(out_scores, (B, g, H, top_k), torch.float32, q.device, "out_scores")
    if out_proxy is not None:
        out_proxy = _out(out_proxy, (B, H, d), torch.float32, q.device, "out_proxy")
    if out_cand is not None:
        out_cand = _out(out_cand, (B, H, Kc), torch.int32, q.device, "out_cand")
    sp = _stream_ptr(stream)
    n = lib.pivot_decode_workspace_size(B, H, d, g, top_k, Kc, bits, int(max_seqlen))
    ws = _workspace(n, q.device, sp)
    if out_proxy is None and out_cand is None:
        rc = lib.pivot_decode_index_ws(q.data_ptr(), kcache.data_ptr(), cu_seqlens.data_ptr(), B, H, d, g, top_k,
                                       Kc, bits, int(max_seqlen), out.data_ptr(), _ptr(out_scores), ws.data_ptr(),
                                       ws.numel(), sp)
    else:
        rc = lib.pivot_decode_index_ex(q.data_ptr(), kcache.data_ptr(), cu_seqlens.data_ptr(), B, H, d, g, top_k,
                                       Kc, bits, int(max_seqlen), out.data_ptr(), _ptr(out_scores),
                                       _ptr(out_proxy), _ptr(out_cand), ws.data_ptr(), ws.numel(), sp)
    _err(lib, rc)
    return out


def pivot_decode_index_paged(q, kpages, block_table, seqlens, g, top_k, Kc, mode=REFINE, max_seqlen=None,
                             out=None, out_scores=None, stream=None, proxy="fp32"):
    """PIVOT decode over a paged key cache: q bf16 [B, g, H, d], kpages bf16
    [num_pages, page_size, H, d] (page_size a power of two), block_table int32
    [B, max_pages] and seqlens int32 [B] on the device (sequence b's key j is
    row j % page_size of page block_table[b, j // page_size]; it holds
    seqlens[b] = n_b + g keys) -> int32 [B, g, H, top_k], as pivot_decode_index."""
    lib = load_library()
    bits = _mode_bits(mode, proxy)
    _check_bf16("q", q, 4)
    _check_bf16("kpages", kpages, 4)
    B, gq, H, d = q.shape
    if gq != g:
        raise PivotError("q's second axis must equal g")
    _, page_size, Hk, dk = kpages.shape
    if (Hk, dk) != (H, d):
        raise PivotError("kpages must be [num_pages, page_size, H, d] with q's H and d")
    if (block_table.dtype != torch.int32 or not block_table.is_cuda or block_table.dim() != 2
            or block_table.shape[0] != B or not block_table.is_contiguous()):
        raise PivotError("block_table must be a contiguous int32 CUDA tensor [B, max_pages]")
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda or seqlens.numel() != B:
        raise PivotError("seqlens must be an int32 CUDA tensor of B lengths")
    if max_seqlen is None:
        raise PivotError("max_seqlen (an upper bound on cache rows per sequence) is required")
    out = _out(out, (B, g, H, top_k), torch.int32, q.device, "out")
    if out_scores is not None:
        out_scores = _out(out_scores, (B, g, H, top_k), torch.float32, q.device, "out_scores")
    sp = _stream_ptr(stream)
    n = lib.pivot_decode_workspace_size(B, H, d, g, top_k, Kc, bits, int(max_seqlen))
    ws = _workspace(n, q.device, sp)
    rc = lib.pivot_decode_index_paged(q.data_ptr(), kpages.data_ptr(), block_table.data_ptr(), seqlens.data_ptr(), B,
                                      H, d, g, int(page_size), int(block_table.shape[1]), top_k, Kc, bits,
                                      int(max_seqlen), out.data_ptr(), _ptr(out_scores), ws.data_ptr(), ws.numel(),
                                      sp)
    _err(lib, rc)
    return out


def sparse_attention(q, k, v, idx, cu_seqlens=None, g=1, out=None, stream=None):
    """The attention that consumes the index rows: for each query row and head,
    softmax over the row's valid indices of (q . k_j) * d^-1/2, applied to v_j
    (fp32; rows without indices give zeros).  Prefill: q, k, v bf16 [L, H, d],
    idx int32 [L, H, top_k].  Decode: q bf16 [B, g, H, d], k and v the packed
    cache [rows, H, d] with cu_seqlens int32 [B+1] (device), idx [B, g, H,
    top_k].  Returns float32 with q's shape."""
    lib = load_library()
    _check_bf16("q", q, q.dim())
    _check_bf16("k", k, 3)
    _check_bf16("v", v, 3)
    if k.shape != v.shape or k.shape[1:] != q.shape[-2:]:
        raise PivotError("k and v must be [rows, H, d] with q's H and d")
    H, d = q.shape[-2], q.shape[-1]
    R = q.numel() // (H * d)
    if (idx.dtype != torch.int32 or not idx.is_cuda or not idx.is_contiguous() or tuple(idx.shape[:-1]) != tuple(q.shape[:-1])):
        raise PivotError("idx must be a contiguous int32 CUDA tensor [..., H, top_k] matching q")
    top_k = idx.shape[-1]
    cu_ptr = None
    if cu_seqlens is not None:
        if q.dim() != 4 or q.shape[1] != g:
            raise PivotError("with cu_seqlens, q must be [B, g, H, d]")
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.numel() != q.shape[0] + 1:
            raise PivotError("cu_seqlens must be an int32 CUDA tensor of B+1 offsets")
        cu_ptr = cu_seqlens.data_ptr()
    elif q.dim() != 3:
        raise PivotError("prefill q must be [L, H, d]")
    out = _out(out, tuple(q.shape), torch.float32, q.device, "out")
    rc = lib.pivot_sparse_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), cu_ptr, R, H, d, g,
                                    top_k, out.data_ptr(), _stream_ptr(stream))
    _err(lib, rc)
    return out


def trace_enable(on: bool = True) -> None:
    """Turns the library's per-launch CUDA-event trace on or off (calling thread)."""
    _err(load_library(), load_library().pivot_trace_enable(1 if on else 0))


def trace_collect() -> dict:
    """Waits for the traced launches and returns {kernel: (total_ms, launches)}; clears the trace."""
    lib = load_library()
    names = ctypes.create_string_buffer(4096)
    ms = (ctypes.c_float * 64)()
    cnt = (ctypes.c_int * 64)()
    n = lib.pivot_trace_collect(names, 4096, ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p), 64)
    if n < 0:
        _err(lib, -n)
    keys = names.value.decode().split(",") if n > 0 else []
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(keys)}


def sync_status(stream=None) -> int:
    """Synchronises the stream and returns the kernels' status bits; raises on a kernel error."""
    lib = load_library()
    flags = ctypes.c_int(0)
    rc = lib.pivot_sync_status(_stream_ptr(stream), ctypes.byref(flags))
    _err(lib, rc)
    return flags.value


def head_range(H: int, rank: int, world: int) -> tuple:
    """Heads [h0, h1) of an H-head layer that rank `rank` of `world` indexes
    when the indexer is split across GPUs by head.  Every head's proxy, scan,
    candidate set and refine read only that head's queries and keys ("PIVOT
    explained", "Show Me The Code": the loop over heads), so the ranks exchange
    nothing; each indexes its heads as an [L, h1-h0, d] layer of its own.  The
    ranges are contiguous, in rank order, cover every head once and differ in
    size by at most one head."""
    if H < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"head_range: need H >= 1 and 0 <= rank < world (H={H}, rank={rank}, world={world})")
    return rank * H // world, (rank + 1) * H // world
