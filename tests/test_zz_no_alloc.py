"""The decode entry point that allocates nothing.

Some callers cannot allocate device memory in the middle of a decode step. One
example is an inference engine that has already given every free byte of HBM to
its KV-cache pool. Another is host code that owns no device allocator.
``pivot_decode_index_noalloc`` serves them from a fixed scratch array built into
the library. This test calls it through the C ABI, twice in a row, on two
different batches. Both calls must give the same rows and scores as the
workspace-taking entry point, and a call too large for the fixed scratch must
be refused with a clear error.

This file is collected last, so a run that stops at the first failure has
already run every other test.  It also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import query_group_top_b200 as qg
import synthetic
from tests.parity import REL_SCORE

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _batch(seed, B, lo, hi):
    dec = synthetic.gen_decode(B, 4, 128, 2, seed=seed, lo=lo, hi=hi)
    q, kc = _dev(dec.q), _dev(dec.kcache)
    cu = torch.from_numpy(dec.cu_seqlens).cuda()
    return q, kc, cu, int(np.diff(dec.cu_seqlens).max())


def _noalloc(lib, q, kc, cu, g, top_k, Kc, mode, max_seqlen):
    B, _, H, d = q.shape
    out = torch.full((B, g, H, top_k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, g, H, top_k), 7.0, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.pivot_decode_index_noalloc(q.data_ptr(), kc.data_ptr(), cu.data_ptr(), B, H, d, g, top_k, Kc, mode,
                                        max_seqlen, out.data_ptr(), sc.data_ptr(), stream)
    assert rc == 0, lib.pivot_last_error()
    qg.sync_status()
    return out, sc


@pytest.mark.parametrize("mode", [qg.REFINE, qg.REUSE])
def test_noalloc_decode_matches_workspace_entry_point(mode):
    lib = qg.load_library()
    g, top_k, Kc = 2, 256, 512
    # two different batches back to back: the second is shorter, so any
    # stale scratch from the first call would show up in its rows
    for seed, B, lo, hi in ((21, 3, 6000, 20000), (22, 2, 100, 3000)):
        q, kc, cu, max_seqlen = _batch(seed, B, lo, hi)
        want_sc = torch.empty((B, g, 4, top_k), dtype=torch.float32, device="cuda")
        want = qg.pivot_decode_index(q, kc, cu, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=want_sc)
        qg.sync_status()
        got, got_sc = _noalloc(lib, q, kc, cu, g, top_k, Kc, mode, max_seqlen)
        assert torch.equal(got, want)
        valid = want >= 0
        a = got_sc[valid].double()
        b = want_sc[valid].double()
        assert torch.all((a - b).abs() <= REL_SCORE * torch.clamp(b.abs(), min=1.0))
        assert torch.all(torch.isnan(got_sc[~valid]))


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    lib = qg.load_library()
    q, kc, cu, _ = _batch(23, 2, 100, 200)
    B, g, H, d = q.shape
    out = torch.empty((B, g, H, 8), dtype=torch.int32, device="cuda")
    big = 3_000_000  # H*B*max_seqlen*4 bytes of order keys alone is far above 32 MiB
    rc = lib.pivot_decode_index_noalloc(q.data_ptr(), kc.data_ptr(), cu.data_ptr(), B, H, d, g, 8, 16, qg.REFINE,
                                        big, out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert rc == 5
    assert b"static maximum" in lib.pivot_last_error()
