"""GPU path vs the CPU oracle, element by element, through the C ABI.

Small shapes are checked in full (several 128-row tiles, ragged tails, partial
groups, d = 64 and 128, g up to 24); the workload sizes are checked on a
seeded sample of (group, head) units that the oracle computes one by one, plus
properties that hold on every row (ascending, unique, causal, row sizes).
"""
import numpy as np
import pytest
import torch

import oracle
import query_group_top_b200 as qg
import synthetic
from tests.parity import assert_parity, compare, near_tie, oracle_threads, valid_rows

pytestmark = pytest.mark.gpu


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_prefill(q, k, g, top_k, Kc, mode, dense=False, proxy="fp32"):
    qd, kd = to_dev(q), to_dev(k)
    L, H, _ = q.shape
    sc = torch.empty((L, H, top_k), dtype=torch.float32, device="cuda")
    if dense:
        out = qg.dense_index(qd, kd, top_k, out_scores=sc)
    else:
        out = qg.pivot_index(qd, kd, g, top_k, Kc, mode, out_scores=sc, proxy=proxy)
    flags = qg.sync_status()
    return out.cpu().numpy(), sc.cpu().numpy(), flags


def check_full(q, k, g, top_k, Kc, mode, dense=False, proxy="fp32"):
    got, gs, flags = run_prefill(q, k, g, top_k, Kc, mode, dense, proxy)
    L, H, _ = q.shape
    pos = np.broadcast_to(np.arange(L)[:, None], (L, H))
    if dense:
        ref = oracle.dense(q, k, top_k)
        cedge = None
    else:
        ref = oracle.prefill(q, k, g, top_k, Kc, mode, proxy=proxy)
        cedge = ref["cand_edge"][np.arange(L) // g] if mode == oracle.REFINE else None
    res = compare(got, ref["out"], ref["edge"], pos, cedge, gs, ref["score"])
    assert_parity(res, f"L={L} H={H} d={q.shape[2]} g={g} k={top_k} Kc={Kc} mode={mode} dense={dense} {proxy}")
    return res, flags


@pytest.mark.parametrize("mode", ["refine", "reuse", "dense", "refine-bf16", "reuse-bf16"])
def test_c0_full(mode):
    c = synthetic.CONFIGS["C0"]
    q, k = synthetic.make_prefill("C0")
    m = oracle.REUSE if mode.startswith("reuse") else oracle.REFINE
    proxy = "bf16" if mode.endswith("bf16") else "fp32"
    res, _ = check_full(q, k, c["g"], c["top_k"], c["Kc"], m, dense=(mode == "dense"), proxy=proxy)
    assert res["exact"] + res["exempt"] == 1024 * 8


SMALL = [
    # L, H, d, g, top_k, Kc
    (1, 1, 64, 1, 1, 1),
    (2, 1, 128, 2, 1, 2),
    (5, 2, 64, 3, 4, 9),
    (64, 1, 128, 8, 8, 16),
    (129, 2, 64, 5, 10, 20),
    (300, 3, 128, 16, 24, 48),
    (511, 1, 64, 17, 7, 33),
    (1000, 2, 128, 8, 37, 80),
    (1500, 1, 64, 24, 64, 128),
    (2049, 2, 128, 2, 100, 300),
    (700, 1, 128, 1, 50, 50),
    (3000, 1, 64, 8, 300, 600),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_small_shapes_all_modes(shape):
    L, H, d, g, top_k, Kc = shape
    q, k = synthetic.gen_prefill(L, H, d, seed=L + 7 * g, rho=0.9)
    check_full(q, k, g, top_k, Kc, oracle.REFINE)
    check_full(q, k, g, top_k, Kc, oracle.REUSE)
    check_full(q, k, g, top_k, Kc, oracle.REUSE, dense=True)
    check_full(q, k, g, top_k, Kc, oracle.REFINE, proxy="bf16")
    check_full(q, k, g, top_k, Kc, oracle.REUSE, proxy="bf16")


@pytest.mark.parametrize("proxy", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(1024, 2, 128, 8, 64, 128), (3000, 3, 64, 5, 100, 300), (700, 1, 128, 16, 30, 64),
                                   (2500, 2, 128, 3, 200, 2000)], ids=lambda s: "x".join(map(str, s)))
def test_proxies_bit_exact_and_candidate_sets(shape, proxy):
    """The proxy kernel's output equals the oracle's proxy bit for bit (the fp32
    mean, or its bf16 rounding); every group's candidate set equals the
    oracle's exactly unless its Kc-th and (Kc+1)-th proxy scores are a near tie."""
    L, H, d, g, top_k, Kc = shape
    q, k = synthetic.gen_prefill(L, H, d, seed=3 * L + g, rho=0.9)
    G = (L + g - 1) // g
    qd, kd = to_dev(q), to_dev(k)
    P = torch.empty((G, H, d), dtype=torch.float32, device="cuda")
    C = torch.empty((G, H, Kc), dtype=torch.int32, device="cuda")
    qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE, proxy=proxy, out_proxy=P, out_cand=C)
    qg.sync_status()
    ref = oracle.prefill(q, k, g, top_k, Kc, oracle.REFINE, want_cand=True, proxy=proxy)
    want_p = ref["proxy"] if proxy == "fp32" else synthetic.bf16_to_f32(ref["proxy_bf16"])
    np.testing.assert_array_equal(P.cpu().numpy().view(np.uint32), want_p.view(np.uint32))
    cand = C.cpu().numpy()
    eq = np.all(cand == ref["cand"], axis=-1)
    assert np.all(eq | near_tie(ref["cand_edge"])), np.argwhere(~eq)[:5]
    assert eq.mean() > 0.99


PER_MEMBER_SHAPES = [
    # L, H, d, g, top_k, Kc
    (5, 2, 64, 3, 2, 4),
    (300, 3, 128, 16, 24, 48),
    (1000, 2, 64, 8, 37, 80),
    (2049, 2, 128, 4, 100, 300),
    (1500, 1, 128, 1, 40, 80),
]


@pytest.mark.parametrize("shape", PER_MEMBER_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_per_member_scan_refine(shape):
    """The listing's reading of Refine ("Show Me The Code", pivot_refine: a
    proxy scan over k[:pos] for each member): every member's candidate set is
    the group proxy's top-Kc over its own prefix.  Checked in full against the
    oracle's per-member mode; a row is exempt when its final select or its own
    candidate select is a near tie."""
    L, H, d, g, top_k, Kc = shape
    q, k = synthetic.gen_prefill(L, H, d, seed=5 * L + g, rho=0.9)
    qd, kd = to_dev(q), to_dev(k)
    sc = torch.empty((L, H, top_k), dtype=torch.float32, device="cuda")
    C = torch.empty((L, H, Kc), dtype=torch.int32, device="cuda")
    out = qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE, out_scores=sc, out_cand=C, scan="member")
    assert qg.sync_status() & ~qg.FLAG_FALLBACK == 0
    ref = oracle.prefill(q, k, g, top_k, Kc, oracle.REFINE_PER_MEMBER)
    pos = np.broadcast_to(np.arange(L)[:, None], (L, H))
    res = compare(out.cpu().numpy(), ref["out"], ref["edge"], pos, ref["member_cand_edge"], sc.cpu().numpy(),
                  ref["score"])
    assert_parity(res, f"per-member L={L} H={H} d={d} g={g} k={top_k} Kc={Kc}")
    # every member's candidate row: min(Kc, pos) ascending indices below pos
    device_rows_valid(C, 0, lambda p: torch.clamp(p, max=Kc))
    # a group's last member scans the shared prefix j < last: same rows as the method
    shared = qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE)
    last = torch.from_numpy(np.minimum(np.arange(0, L, g) + g, L) - 1).cuda()
    ref_shared = oracle.prefill(q, k, g, top_k, Kc, oracle.REFINE)
    lc = last.cpu().numpy()
    ok = np.all(out[last].cpu().numpy() == shared[last].cpu().numpy(), axis=-1)
    assert np.all(ok | near_tie(ref_shared["cand_edge"]) | near_tie(ref["edge"][lc]) |
                  near_tie(ref_shared["edge"][lc]))


def test_per_member_scan_c1_sampled():
    """The per-member scan on the C1 workload (L=8192, H=16, g=8, k=256,
    Kc=512): the whole layer on the GPU, 96 sampled groups by the oracle."""
    c = synthetic.CONFIGS["C1"]
    q, k = synthetic.make_prefill("C1")
    L, H, _ = q.shape
    g, top_k, Kc = c["g"], c["top_k"], c["Kc"]
    G = (L + g - 1) // g
    qd, kd = to_dev(q), to_dev(k)
    sc = torch.empty((L, H, top_k), dtype=torch.float32, device="cuda")
    out = qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE, out_scores=sc, scan="member")
    qg.sync_status()
    device_rows_valid(out, 0, lambda p: torch.clamp(p, max=top_k))
    gi, hi = sampled_units(G, H, 96, seed=L + 17)
    r = oracle_threads(oracle.prefill_units, q, k, g, top_k, Kc, oracle.REFINE_PER_MEMBER, gi, hi)
    for u, (i, h) in enumerate(zip(gi, hi)):
        rows = np.arange(i * g, min(i * g + g, L))
        nm = len(rows)
        o = out[rows[0]:rows[-1] + 1, h].cpu().numpy()
        s = sc[rows[0]:rows[-1] + 1, h].cpu().numpy()
        res = compare(o, r["out"][u, :nm], r["edge"][u, :nm], rows, r["member_cand_edge"][u, :nm], s,
                      r["score"][u, :nm])
        assert_parity(res, f"C1 per-member group={i} head={h}")


def test_exact_ties_and_fallback_rows():
    """Constant keys: every score of a row ties, the lowest indices win; the
    sampled threshold cannot separate them, so long rows go to the exact
    fallback path (flag bit 4) and must still be exact."""
    L, H, d, top_k = 3000, 2, 64, 8
    rng = np.random.default_rng(5)
    q = synthetic.bf16_from_f32(rng.standard_normal((L, H, d)).astype(np.float32))
    k = synthetic.bf16_from_f32(np.ones((L, H, d), np.float32))
    res, flags = check_full(q, k, 1, top_k, top_k, oracle.REUSE, dense=True)
    assert flags & qg.FLAG_FALLBACK
    assert res["exempt"] == 0
    res, flags = check_full(q, k, 4, top_k, 2 * top_k, oracle.REFINE)
    assert res["exempt"] == 0


def test_g1_pivot_equals_dense_on_gpu():
    """g = 1: the proxy is the query itself, so Reuse runs the dense computation
    (bit-identical) and Refine must agree with the dense oracle."""
    q, k = synthetic.gen_prefill(1200, 2, 128, seed=9)
    b, _, _ = run_prefill(q, k, 1, 40, 40, oracle.REUSE, dense=True)
    c, _, _ = run_prefill(q, k, 1, 40, 40, oracle.REUSE)
    np.testing.assert_array_equal(b, c)
    a, sa, _ = run_prefill(q, k, 1, 40, 80, oracle.REFINE)
    ref = oracle.dense(q, k, 40)
    pos = np.broadcast_to(np.arange(1200)[:, None], (1200, 2))
    assert_parity(compare(a, ref["out"], ref["edge"], pos, None, sa, ref["score"]), "g=1 refine vs dense")


# ------------------------------------------------------------ workload sizes
def sampled_units(G, H, n, seed):
    rng = np.random.default_rng(seed)
    gi = rng.integers(0, G, size=n)
    gi[:2] = [G - 1, max(0, G // 2)]           # the longest prefix and a ragged middle
    hi = rng.integers(0, H, size=n)
    return gi.astype(np.int32), hi.astype(np.int32)


def device_rows_valid(out, pos0, want_n=None):
    """Properties of every row, checked on the device: an ascending prefix of
    valid indices, -1 padding after it, every index < its position, and (when
    want_n is given) want_n(pos) valid entries.  out [P, H, k] covers positions
    pos0 .. pos0+P-1."""
    P = out.shape[0]
    for a in range(0, P, 2048):
        o = out[a:a + 2048]
        pos = torch.arange(pos0 + a, pos0 + a + o.shape[0], device=o.device, dtype=torch.int64)[:, None, None]
        v = o >= 0
        assert not bool((v[..., 1:] & ~v[..., :-1]).any()), "valid entry after padding"
        assert bool(((o[..., 1:] > o[..., :-1]) | ~v[..., 1:]).all()), "not strictly ascending"
        assert bool(((o < pos) | ~v).all()), "index not causal"
        assert bool(((o == -1) | v).all()), "padding other than -1"
        if want_n is not None:
            assert bool((v.sum(-1) == want_n(pos[:, :, 0])).all()), "row size"


def check_sampled(name, modes, n_units):
    c = synthetic.CONFIGS[name]
    q, k = synthetic.make_prefill(name)
    L, H, _ = q.shape
    g, top_k, Kc = c["g"], c["top_k"], c["Kc"]
    G = (L + g - 1) // g
    qd, kd = to_dev(q), to_dev(k)
    for mode in modes:
        sc = torch.empty((L, H, top_k), dtype=torch.float32, device="cuda")
        out = qg.pivot_index(qd, kd, g, top_k, Kc, mode, out_scores=sc)
        qg.sync_status()
        device_rows_valid(out, 0, (lambda p: torch.clamp(p, max=top_k)) if mode == oracle.REFINE else None)
        gi, hi = sampled_units(G, H, n_units, seed=L + mode)
        r = oracle_threads(oracle.prefill_units, q, k, g, top_k, Kc, mode, gi, hi)
        rows_all = np.concatenate([np.arange(i * g, min(i * g + g, L)) for i in gi])
        head_all = np.concatenate([np.full(min(i * g + g, L) - i * g, h) for i, h in zip(gi, hi)])
        ri = torch.from_numpy(rows_all).cuda()
        hh = torch.from_numpy(head_all).cuda()
        o = out[ri, hh].cpu().numpy()
        s = sc[ri, hh].cpu().numpy()
        at = 0
        for u, (i, h) in enumerate(zip(gi, hi)):
            rows = np.arange(i * g, min(i * g + g, L))
            nm = len(rows)
            res = compare(o[at:at + nm], r["out"][u, :nm], r["edge"][u, :nm], rows,
                          np.broadcast_to(r["cand_edge"][u], (nm, 2)) if mode == oracle.REFINE else None,
                          s[at:at + nm], r["score"][u, :nm])
            assert_parity(res, f"{name} mode={mode} group={i} head={h}")
            at += nm
        del out, sc
    torch.cuda.empty_cache()


def test_c1_sampled():
    check_sampled("C1", (oracle.REFINE, oracle.REUSE), 256)


def test_c2_sampled():
    check_sampled("C2", (oracle.REFINE, oracle.REUSE), 128)


def test_c3_sampled():
    check_sampled("C3", (oracle.REFINE, oracle.REUSE), 256)


def test_c1_dense_sampled():
    c = synthetic.CONFIGS["C1"]
    q, k = synthetic.make_prefill("C1")
    L, H, _ = q.shape
    got, gs, _ = run_prefill(q, k, 1, c["top_k"], c["top_k"], oracle.REUSE, dense=True)
    rng = np.random.default_rng(17)
    pi = rng.integers(0, L, size=64).astype(np.int32)
    pi[0] = L - 1
    hi = rng.integers(0, H, size=64).astype(np.int32)
    r = oracle.dense_units(q, k, c["top_k"], pi, hi)
    res = compare(got[pi, hi], r["out"], r["edge"], pi, None, gs[pi, hi], r["score"])
    assert_parity(res, "C1 dense")


# ------------------------------------------------------------------- decode
def run_decode(dec, g, top_k, Kc, mode, max_seqlen, proxy="fp32"):
    qd = to_dev(dec.q)
    kd = to_dev(dec.kcache)
    cu = torch.from_numpy(dec.cu_seqlens).cuda()
    B, _, H, _ = dec.q.shape
    sc = torch.empty((B, g, H, top_k), dtype=torch.float32, device="cuda")
    out = qg.pivot_decode_index(qd, kd, cu, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=sc, proxy=proxy)
    qg.sync_status()
    return out.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("proxy", ["fp32", "bf16"])
def test_decode_proxies_and_candidate_sets(proxy):
    """Decode: the fp32 proxies bit for bit, and the candidate sets, against
    the oracle (one sequence shorter than Kc, the others longer)."""
    B, H, d, g, top_k, Kc = 4, 2, 128, 2, 64, 700
    dec = synthetic.gen_decode(B, H, d, g, seed=91, lo=300, hi=6000)
    max_seqlen = int(np.diff(dec.cu_seqlens).max())
    qd, kd, cu = to_dev(dec.q), to_dev(dec.kcache), torch.from_numpy(dec.cu_seqlens).cuda()
    P = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    C = torch.empty((B, H, Kc), dtype=torch.int32, device="cuda")
    qg.pivot_decode_index(qd, kd, cu, g, top_k, Kc, qg.REFINE, max_seqlen=max_seqlen, proxy=proxy, out_proxy=P,
                          out_cand=C)
    qg.sync_status()
    bi, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    r = oracle.decode_units(dec.q, dec.kcache, dec.cu_seqlens, g, top_k, Kc, oracle.REFINE, bi.ravel(), hh.ravel(),
                            want_cand=True, proxy=proxy)
    want_p = r["proxy"] if proxy == "fp32" else synthetic.bf16_to_f32(r["proxy_bf16"])
    np.testing.assert_array_equal(P.cpu().numpy().reshape(B * H, d).view(np.uint32), want_p.view(np.uint32))
    cand = C.cpu().numpy().reshape(B * H, Kc)
    eq = np.all(cand == r["cand"], axis=-1)
    assert np.all(eq | near_tie(r["cand_edge"])), np.argwhere(~eq)[:5]


@pytest.mark.parametrize("proxy", ["fp32", "bf16"])
@pytest.mark.parametrize("case", [
    # B, H, d, g, lo, hi, top_k, Kc
    (1, 1, 128, 1, 0, 0, 4, 8),
    (3, 2, 64, 2, 0, 300, 16, 32),
    (4, 2, 128, 2, 1000, 5000, 64, 128),
    (2, 1, 128, 3, 200, 9000, 300, 700),
    (5, 2, 64, 4, 50, 2500, 100, 200),
])
def test_decode_small(case, proxy):
    B, H, d, g, lo, hi, top_k, Kc = case
    dec = synthetic.gen_decode(B, H, d, g, seed=B * 31 + g, lo=lo, hi=hi)
    max_seqlen = int(np.diff(dec.cu_seqlens).max())
    bi, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    for mode in (oracle.REFINE, oracle.REUSE):
        got, gs = run_decode(dec, g, top_k, Kc, mode, max_seqlen, proxy)
        r = oracle.decode_units(dec.q, dec.kcache, dec.cu_seqlens, g, top_k, Kc, mode, bi.ravel(), hh.ravel(),
                                proxy=proxy)
        want = r["out"].reshape(B, H, g, top_k).transpose(0, 2, 1, 3)
        edge = r["edge"].reshape(B, H, g, 2).transpose(0, 2, 1, 3)
        wsc = r["score"].reshape(B, H, g, top_k).transpose(0, 2, 1, 3)
        cedge = None
        if mode == oracle.REFINE:
            cedge = np.broadcast_to(r["cand_edge"].reshape(B, H, 1, 2).transpose(0, 2, 1, 3), (B, g, H, 2))
        pos = np.broadcast_to((dec.n_ctx[:, None] + np.arange(g)[None, :])[:, :, None], (B, g, H))
        res = compare(got, want, edge, pos, cedge, gs, wsc)
        assert_parity(res, f"decode {case} mode={mode}")


def paged_cache(dec, page_size, seed):
    """The packed cache of `dec` laid out in pages: every sequence's rows cut
    into pages of page_size rows, the pages placed in a random order (with a
    few unused pages between them) and reached through a block table."""
    rng = np.random.default_rng(seed)
    cu = dec.cu_seqlens.astype(np.int64)
    B = len(cu) - 1
    lens = np.diff(cu)
    npages = (lens + page_size - 1) // page_size
    total = int(npages.sum()) + 5
    order = rng.permutation(total)
    _, H, d = dec.kcache.shape
    kpages = np.zeros((total, page_size, H, d), np.uint16)
    table = np.zeros((B, int(npages.max())), np.int32)
    at = 0
    for b in range(B):
        for pg in range(int(npages[b])):
            phys = int(order[at])
            at += 1
            rows = dec.kcache[cu[b] + pg * page_size:min(cu[b] + (pg + 1) * page_size, cu[b + 1])]
            kpages[phys, :len(rows)] = rows
            table[b, pg] = phys
    return kpages, table, lens.astype(np.int32)


@pytest.mark.parametrize("page_size", [16, 128])
def test_paged_decode_equals_packed_and_oracle(page_size):
    """A paged key cache (the serving layout): the keys of a packed cache cut
    into pages in a random order behind a block table.  Refine and Reuse must
    give the packed cache's rows and scores bit for bit, and match the oracle."""
    B, H, d, g, top_k, Kc = 5, 2, 128, 3, 48, 96
    dec = synthetic.gen_decode(B, H, d, g, seed=page_size + 3, lo=20, hi=2600)
    max_seqlen = int(np.diff(dec.cu_seqlens).max())
    kpages, table, lens = paged_cache(dec, page_size, seed=page_size)
    qd, kp = to_dev(dec.q), to_dev(kpages)
    bt, sl = torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda()
    bi, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    for mode in (oracle.REFINE, oracle.REUSE):
        want_rows, want_sc = run_decode(dec, g, top_k, Kc, mode, max_seqlen)
        sc = torch.empty((B, g, H, top_k), dtype=torch.float32, device="cuda")
        out = qg.pivot_decode_index_paged(qd, kp, bt, sl, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=sc)
        assert qg.sync_status() & ~qg.FLAG_FALLBACK == 0
        got, gs = out.cpu().numpy(), sc.cpu().numpy()
        np.testing.assert_array_equal(got, want_rows)
        np.testing.assert_array_equal(gs.view(np.uint32), want_sc.view(np.uint32))
        r = oracle.decode_units(dec.q, dec.kcache, dec.cu_seqlens, g, top_k, Kc, mode, bi.ravel(), hh.ravel())
        want = r["out"].reshape(B, H, g, top_k).transpose(0, 2, 1, 3)
        edge = r["edge"].reshape(B, H, g, 2).transpose(0, 2, 1, 3)
        wsc = r["score"].reshape(B, H, g, top_k).transpose(0, 2, 1, 3)
        cedge = None
        if mode == oracle.REFINE:
            cedge = np.broadcast_to(r["cand_edge"].reshape(B, H, 1, 2).transpose(0, 2, 1, 3), (B, g, H, 2))
        pos = np.broadcast_to((dec.n_ctx[:, None] + np.arange(g)[None, :])[:, :, None], (B, g, H))
        assert_parity(compare(got, want, edge, pos, cedge, gs, wsc), f"paged decode ps={page_size} mode={mode}")


def test_c4_decode_sampled():
    """The MTP decode workload at full size (64 sequences, contexts up to 131072,
    19 GB of keys) in the launch configuration the bench times; the oracle
    checks whole sequences, all heads, the longest included."""
    c = synthetic.CONFIGS["C4"]
    g, top_k, Kc, H = c["g"], c["top_k"], c["Kc"], c["H"]
    q, kc, cu, n_ctx = synthetic.gen_decode_device(c["B"], H, c["d"], g, c["seed"], c["lo"], c["hi"],
                                                   c["rho"], c["heavy_frac"], c["heavy_scale"])
    max_seqlen = int((n_ctx + g).max())
    cu_h = cu.cpu().numpy()
    rng = np.random.default_rng(44)
    seqs = [int(np.argmax(n_ctx)), int(np.argmin(n_ctx))] + list(rng.integers(0, c["B"], size=1))
    for mode in (oracle.REFINE, oracle.REUSE):
        sc = torch.empty((c["B"], g, H, top_k), dtype=torch.float32, device="cuda")
        out = qg.pivot_decode_index(q, kc, cu, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=sc)
        qg.sync_status()
        o = out.cpu().numpy()
        pos = np.broadcast_to((n_ctx[:, None] + np.arange(g)[None, :])[:, :, None], o.shape[:3])
        assert valid_rows(o, pos).all()
        s = sc.cpu().numpy()
        for b in seqs:
            kb = kc[int(cu_h[b]):int(cu_h[b + 1])].cpu().view(torch.int16).numpy().view(np.uint16)
            qb = q[b:b + 1].cpu().view(torch.int16).numpy().view(np.uint16)
            cub = np.array([0, kb.shape[0]], np.int32)
            r = oracle.decode_units(qb, kb, cub, g, top_k, Kc, mode, np.zeros(H, np.int32), np.arange(H, dtype=np.int32))
            want = r["out"].transpose(1, 0, 2)            # [g, H, k]
            edge = r["edge"].transpose(1, 0, 2)
            cedge = None
            if mode == oracle.REFINE:
                cedge = np.broadcast_to(r["cand_edge"][None], (g, H, 2))
            res = compare(o[b], want, edge, pos[b], cedge, s[b], r["score"].transpose(1, 0, 2))
            assert_parity(res, f"C4 mode={mode} seq={b} n_ctx={n_ctx[b]}")
        del out, sc
    del kc
    torch.cuda.empty_cache()


def _bad_length_batch(g, H, d):
    """Three sequences: 0 is valid, 1 holds fewer cache rows than one step,
    2 is longer than the max_seqlen the call declares."""
    dec = synthetic.gen_decode(3, H, d, g, seed=77, lo=300, hi=2000)
    lens = np.diff(dec.cu_seqlens).astype(np.int64)
    if lens[2] <= lens[0]:
        lens[[0, 2]] = lens[[2, 0]]
        rows = [dec.kcache[dec.cu_seqlens[2]:dec.cu_seqlens[3]], dec.kcache[dec.cu_seqlens[1]:dec.cu_seqlens[2]],
                dec.kcache[dec.cu_seqlens[0]:dec.cu_seqlens[1]]]
        q = dec.q[[2, 1, 0]]
    else:
        rows = [dec.kcache[dec.cu_seqlens[b]:dec.cu_seqlens[b + 1]] for b in range(3)]
        q = dec.q
    rows[1] = rows[1][:g - 1]
    kc = np.ascontiguousarray(np.concatenate(rows, axis=0))
    cu = np.zeros(4, np.int32)
    cu[1:] = np.cumsum([r.shape[0] for r in rows])
    max_seqlen = int(rows[0].shape[0])
    assert rows[2].shape[0] > max_seqlen >= g > rows[1].shape[0]
    return np.ascontiguousarray(q), kc, cu, max_seqlen


@pytest.mark.parametrize("entry", ["ws", "noalloc"])
@pytest.mark.parametrize("mode", ["reuse", "refine"])
def test_decode_bad_lengths_are_skipped_and_reported(mode, entry):
    """A sequence longer than max_seqlen, or with fewer cache rows than one
    MTP step, is skipped on the device: its rows come back empty (-1), the
    status reads PIVOT_ERR_INVALID_ARG, and the valid sequence is exact."""
    import ctypes
    g, top_k, Kc, H, d = 3, 16, 40, 2, 64
    m = oracle.REFINE if mode == "refine" else oracle.REUSE
    q, kc, cu, max_seqlen = _bad_length_batch(g, H, d)
    qd, kd, cud = to_dev(q), to_dev(kc), torch.from_numpy(cu).cuda()
    lib = qg.load_library()
    qg.sync_status()  # start from a clear status word
    out = torch.full((3, g, H, top_k), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty((3, g, H, top_k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    if entry == "ws":
        qg.pivot_decode_index(qd, kd, cud, g, top_k, Kc, m, max_seqlen=max_seqlen, out=out, out_scores=sc)
    else:
        rc = lib.pivot_decode_index_noalloc(qd.data_ptr(), kd.data_ptr(), cud.data_ptr(), 3, H, d, g, top_k, Kc, m,
                                            max_seqlen, out.data_ptr(), sc.data_ptr(), stream)
        assert rc == 0, lib.pivot_last_error()
    flags = ctypes.c_int(0)
    rc = lib.pivot_sync_status(stream, ctypes.byref(flags))
    assert rc == 1 and flags.value & qg.FLAG_BADLEN, (rc, flags.value)
    assert qg.sync_status() == 0  # the status word was cleared
    o = out.cpu().numpy()
    assert np.all(o[1:] == -1)
    cub = np.array([0, cu[1]], np.int32)
    r = oracle.decode_units(q[:1], kc[:cu[1]], cub, g, top_k, Kc, m, np.zeros(H, np.int32),
                            np.arange(H, dtype=np.int32))
    n0 = cu[1] - g
    pos = np.broadcast_to((n0 + np.arange(g))[:, None], (g, H))
    cedge = np.broadcast_to(r["cand_edge"][None], (g, H, 2)) if m == oracle.REFINE else None
    res = compare(o[0], r["out"].transpose(1, 0, 2), r["edge"].transpose(1, 0, 2), pos, cedge,
                  sc.cpu().numpy()[0], r["score"].transpose(1, 0, 2))
    assert_parity(res, f"bad-length batch, valid sequence, {mode} {entry}")


def test_refine_select_ties_and_misses():
    """Refine members with more than 512 usable candidates take the sampled
    interval path.  Constant keys make every score of a member equal, so the
    sample has no score range: the member goes to the exact refine fallback
    (flag bit 4) and must still take the lowest indices.  Keys and queries of
    small integers give many exact ties inside the ranked list, resolved in
    candidate (index) order."""
    L, H, d, g, top_k, Kc = 6000, 1, 64, 4, 700, 1500
    rng = np.random.default_rng(31)
    q = synthetic.bf16_from_f32(rng.standard_normal((L, H, d)).astype(np.float32))
    k = synthetic.bf16_from_f32(np.ones((L, H, d), np.float32))
    res, flags = check_full(q, k, g, top_k, Kc, oracle.REFINE)
    assert flags & qg.FLAG_FALLBACK
    assert res["exempt"] == 0
    qi = synthetic.bf16_from_f32(rng.integers(-1, 2, size=(L, 2, d)).astype(np.float32))
    ki = synthetic.bf16_from_f32(rng.integers(-1, 2, size=(L, 2, d)).astype(np.float32))
    res, _ = check_full(qi, ki, g, top_k, Kc, oracle.REFINE)
    assert res["exempt"] == 0
    res, _ = check_full(qi, ki, 8, 300, 2000, oracle.REFINE)
    assert res["exempt"] == 0


def test_bounded_waits_time_out_and_the_next_call_is_exact():
    """Every kernel wait on another role gives up after a limit.  With the
    limit set to 1 ns a call's waits run out: the kernels drain what they
    issued, return, and pivot_sync_status reports PIVOT_ERR_TIMEOUT; with the
    default limit restored the next call is exact."""
    import ctypes
    lib = qg.load_library()
    L, H, d, g, top_k, Kc = 300, 1, 64, 4, 8, 16
    q, k = synthetic.gen_prefill(L, H, d, seed=5, rho=0.9)
    qd, kd = to_dev(q), to_dev(k)
    qg.sync_status()
    stream = torch.cuda.current_stream().cuda_stream
    try:
        lib.pivot_set_wait_limit(1)
        qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE)
        flags = ctypes.c_int(0)
        rc = lib.pivot_sync_status(stream, ctypes.byref(flags))
        assert rc == 4 and flags.value & qg.FLAG_TIMEOUT, (rc, flags.value)
    finally:
        lib.pivot_set_wait_limit(0)
    assert qg.sync_status() == 0
    check_full(q, k, g, top_k, Kc, oracle.REFINE)


def test_bare_entry_points_allocate_their_own_workspace():
    """pivot_index, dense_index and pivot_decode_index take their scratch with
    cudaMallocAsync on the stream; their rows equal the oracle's."""
    lib = qg.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    L, H, d, g, top_k, Kc = 700, 2, 128, 8, 30, 64
    q, k = synthetic.gen_prefill(L, H, d, seed=41, rho=0.9)
    qd, kd = to_dev(q), to_dev(k)
    pos = np.broadcast_to(np.arange(L)[:, None], (L, H))
    for mode in (oracle.REFINE, oracle.REUSE):
        out = torch.full((L, H, top_k), -7, dtype=torch.int32, device="cuda")
        assert lib.pivot_index(qd.data_ptr(), kd.data_ptr(), L, H, d, g, top_k, Kc, mode, out.data_ptr(), stream) == 0
        qg.sync_status()
        ref = oracle.prefill(q, k, g, top_k, Kc, mode)
        cedge = ref["cand_edge"][np.arange(L) // g] if mode == oracle.REFINE else None
        assert_parity(compare(out.cpu().numpy(), ref["out"], ref["edge"], pos, cedge), f"bare pivot_index {mode}")
    out = torch.full((L, H, top_k), -7, dtype=torch.int32, device="cuda")
    assert lib.dense_index(qd.data_ptr(), kd.data_ptr(), L, H, d, top_k, out.data_ptr(), stream) == 0
    qg.sync_status()
    ref = oracle.dense(q, k, top_k)
    assert_parity(compare(out.cpu().numpy(), ref["out"], ref["edge"], pos), "bare dense_index")
    dec = synthetic.gen_decode(3, H, d, 2, seed=43, lo=100, hi=3000)
    dq, dk, cu = to_dev(dec.q), to_dev(dec.kcache), torch.from_numpy(dec.cu_seqlens).cuda()
    max_seqlen = int(np.diff(dec.cu_seqlens).max())
    bi, hh = np.meshgrid(np.arange(3), np.arange(H), indexing="ij")
    for mode in (oracle.REFINE, oracle.REUSE):
        out = torch.full((3, 2, H, top_k), -7, dtype=torch.int32, device="cuda")
        assert lib.pivot_decode_index(dq.data_ptr(), dk.data_ptr(), cu.data_ptr(), 3, H, d, 2, top_k, Kc, mode,
                                      max_seqlen, out.data_ptr(), stream) == 0
        qg.sync_status()
        r = oracle.decode_units(dec.q, dec.kcache, dec.cu_seqlens, 2, top_k, Kc, mode, bi.ravel(), hh.ravel())
        want = r["out"].reshape(3, H, 2, top_k).transpose(0, 2, 1, 3)
        edge = r["edge"].reshape(3, H, 2, 2).transpose(0, 2, 1, 3)
        cedge = None
        if mode == oracle.REFINE:
            cedge = np.broadcast_to(r["cand_edge"].reshape(3, H, 1, 2).transpose(0, 2, 1, 3), (3, 2, H, 2))
        dpos = np.broadcast_to((dec.n_ctx[:, None] + np.arange(2)[None, :])[:, :, None], (3, 2, H))
        assert_parity(compare(out.cpu().numpy(), want, edge, dpos, cedge), f"bare pivot_decode_index {mode}")


# ------------------------------------------------- the sparse-attention consumer
ATT_TOL = 1e-4   # fp32 online softmax over <= 4096 terms against the fp64 oracle


def assert_attention_close(got, want, what):
    err = np.abs(got.astype(np.float64) - want) / np.maximum(1.0, np.abs(want))
    assert err.max() <= ATT_TOL, f"{what}: max relative error {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}"


@pytest.mark.parametrize("d", [64, 128])
def test_sparse_attention_prefill(d):
    """The demo's consumer ("Show Me The Code"): softmax(q . k[sel] / sqrt(d)) @ v[sel]
    per position and head, over the rows that the Refine indexer wrote (and a
    ragged random set of rows with padding), against the fp64 oracle; position 0
    has no index and gets zeros."""
    L, H, g, top_k, Kc = 1024, 4, 8, 64, 128
    q, k = synthetic.gen_prefill(L, H, d, seed=d + 1, rho=0.9)
    v, _ = synthetic.gen_iid(L, H, d, seed=d + 2)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    idx = qg.pivot_index(qd, kd, g, top_k, Kc, qg.REFINE)
    out = qg.sparse_attention(qd, kd, vd, idx)
    qg.sync_status()
    want = oracle.sparse_attention(q, k, v, idx.cpu().numpy())
    got = out.cpu().numpy()
    assert_attention_close(got, want, f"prefill d={d}")
    assert np.all(got[0] == 0)
    # ragged rows: random valid prefixes of a width that no stream count divides
    rng = np.random.default_rng(d)
    tk = 37
    ridx = -np.ones((L, H, tk), np.int32)
    for pos in range(1, L):
        n = int(rng.integers(0, min(tk, pos) + 1))
        ridx[pos, :, :n] = np.sort(rng.choice(pos, size=n, replace=False))
    out2 = qg.sparse_attention(qd, kd, vd, torch.from_numpy(ridx).cuda())
    assert_attention_close(out2.cpu().numpy(), oracle.sparse_attention(q, k, v, ridx), f"ragged d={d}")


def test_sparse_attention_decode():
    """The consumer after an MTP decode step: q [B, g, H, d], the packed key and
    value caches, the decode indexer's rows."""
    B, H, d, g, top_k, Kc = 4, 2, 128, 2, 256, 512
    dec = synthetic.gen_decode(B, H, d, g, seed=77, lo=100, hi=3000)
    rows = dec.kcache.shape[0]
    v, _ = synthetic.gen_iid(rows, H, d, seed=78)
    max_seqlen = int(np.diff(dec.cu_seqlens).max())
    qd, kd, vd = to_dev(dec.q), to_dev(dec.kcache), to_dev(v)
    cu = torch.from_numpy(dec.cu_seqlens).cuda()
    idx = qg.pivot_decode_index(qd, kd, cu, g, top_k, Kc, qg.REFINE, max_seqlen=max_seqlen)
    out = qg.sparse_attention(qd, kd, vd, idx, cu_seqlens=cu, g=g)
    qg.sync_status()
    want = oracle.sparse_attention(dec.q, dec.kcache, v, idx.cpu().numpy().reshape(B * g, H, top_k),
                                   cu_seqlens=dec.cu_seqlens, g=g)
    assert_attention_close(out.cpu().numpy().reshape(B * g, H, d), want, "decode")


def test_sparse_attention_c4_sampled():
    """The consumer at the decode workload's full size, in the launch
    configuration the bench times (64 sequences, 19 GB of keys and as many
    values, the decode indexer's rows): whole sequences checked by the oracle,
    the longest and the shortest included."""
    c = synthetic.CONFIGS["C4"]
    g, top_k, Kc, H, d = c["g"], c["top_k"], c["Kc"], c["H"], c["d"]
    q, kc, cu, n_ctx = synthetic.gen_decode_device(c["B"], H, d, g, c["seed"], c["lo"], c["hi"],
                                                   c["rho"], c["heavy_frac"], c["heavy_scale"])
    max_seqlen = int((n_ctx + g).max())
    gen = torch.Generator(device="cuda")
    gen.manual_seed(c["seed"] * 7 + 1)
    vc = torch.randn(kc.shape, generator=gen, device="cuda", dtype=torch.bfloat16)
    idx = qg.pivot_decode_index(q, kc, cu, g, top_k, Kc, qg.REFINE, max_seqlen=max_seqlen)
    out = qg.sparse_attention(q, kc, vc, idx, cu_seqlens=cu, g=g)
    qg.sync_status()
    cu_h = cu.cpu().numpy()
    rng = np.random.default_rng(45)
    for b in [int(np.argmax(n_ctx)), int(np.argmin(n_ctx))] + list(rng.integers(0, c["B"], size=1)):
        rows = slice(int(cu_h[b]), int(cu_h[b + 1]))
        kb = kc[rows].cpu().view(torch.int16).numpy().view(np.uint16)
        vb = vc[rows].cpu().view(torch.int16).numpy().view(np.uint16)
        qb = q[b].cpu().view(torch.int16).numpy().view(np.uint16)          # [g, H, d]
        want = oracle.sparse_attention(qb, kb, vb, idx[b].cpu().numpy(), cu_seqlens=np.array([0, kb.shape[0]], np.int32),
                                       g=g)
        assert_attention_close(out[b].cpu().numpy(), want, f"C4 consumer seq={b} n_ctx={n_ctx[b]}")
    del kc, vc, out, idx
    torch.cuda.empty_cache()


def test_paged_decode_c4_equals_packed():
    """The paged cache at the decode workload's full size: the 64 sequences'
    keys moved into 64-row pages in a random order on the device; every row
    and score must equal the packed cache's (Refine and Reuse)."""
    c = synthetic.CONFIGS["C4"]
    g, top_k, Kc, H, d = c["g"], c["top_k"], c["Kc"], c["H"], c["d"]
    q, kc, cu, n_ctx = synthetic.gen_decode_device(c["B"], H, d, g, c["seed"], c["lo"], c["hi"],
                                                   c["rho"], c["heavy_frac"], c["heavy_scale"])
    max_seqlen = int((n_ctx + g).max())
    ps = 64
    cu_h = cu.cpu().numpy().astype(np.int64)
    lens = np.diff(cu_h)
    npages = (lens + ps - 1) // ps
    total = int(npages.sum())
    order = np.random.default_rng(46).permutation(total)
    table = np.zeros((c["B"], int(npages.max())), np.int32)
    src, dst = [], []
    at = 0
    for b in range(c["B"]):
        for pg in range(int(npages[b])):
            table[b, pg] = order[at]
            r0 = pg * ps
            n = int(min(ps, lens[b] - r0))
            src.append(np.arange(cu_h[b] + r0, cu_h[b] + r0 + n))
            dst.append(order[at] * ps + np.arange(n))
            at += 1
    kp = torch.zeros((total * ps, H, d), dtype=torch.bfloat16, device="cuda")
    kp[torch.from_numpy(np.concatenate(dst)).cuda()] = kc[torch.from_numpy(np.concatenate(src)).cuda()]
    kp = kp.view(total, ps, H, d)
    bt = torch.from_numpy(table).cuda()
    sl = torch.from_numpy(lens.astype(np.int32)).cuda()
    for mode in (qg.REFINE, qg.REUSE):
        sa = torch.empty((c["B"], g, H, top_k), dtype=torch.float32, device="cuda")
        sb = torch.empty_like(sa)
        a = qg.pivot_decode_index(q, kc, cu, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=sa)
        b = qg.pivot_decode_index_paged(q, kp, bt, sl, g, top_k, Kc, mode, max_seqlen=max_seqlen, out_scores=sb)
        qg.sync_status()
        assert torch.equal(a, b), f"mode={mode}"
        assert torch.equal(sa.view(torch.int32), sb.view(torch.int32)), f"mode={mode}"
    del kc, kp
    torch.cuda.empty_cache()
