"""Pins of the CPU oracle against things other than itself.

* brute force on tiny inputs (tests/brute.py: numpy + lexsort, written apart);
* hand-worked fixtures (tests/golden/*.txt, each with its derivation);
* closed forms (ramps, constant keys) whose answer is known without a program;
* invariants that the method's definition implies (g=1, Kc >= prefix,
  causality, Reuse sharing, row sizes);
* the pages' demo shape (seq_len, num_heads, top_k) = (1024, 8, 64).
"""
import os

import numpy as np
import pytest

import oracle
import synthetic
from tests import brute

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def int_inputs(rng, L, H, d, lo=-3, hi=3):
    """Small-integer inputs: every dot product and proxy sum is exact, ties are frequent."""
    q = rng.integers(lo, hi + 1, size=(L, H, d)).astype(np.float32)
    k = rng.integers(lo, hi + 1, size=(L, H, d)).astype(np.float32)
    return synthetic.bf16_from_f32(q), synthetic.bf16_from_f32(k)


def bits(vals):
    return synthetic.bf16_from_f32(np.asarray(vals, dtype=np.float32))


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", range(24))
def test_prefill_matches_brute_force_exact_inputs(seed):
    rng = np.random.default_rng(1000 + seed)
    L = int(rng.integers(1, 60))
    H = int(rng.integers(1, 3))
    d = int(rng.choice([2, 4, 8]))
    g = int(rng.choice([1, 2, 3, 5, 8]))
    top_k = int(rng.integers(1, 9))
    Kc = int(rng.integers(top_k, 3 * top_k + 1))
    q, k = int_inputs(rng, L, H, d, -2, 2)
    for mode in (oracle.REFINE, oracle.REUSE, oracle.REFINE_PER_MEMBER):
        for prec in oracle.PROXY_PRECISIONS:
            got = oracle.prefill(q, k, g, top_k, Kc, mode, proxy=prec)["out"]
            want = brute.prefill(q, k, g, top_k, Kc, mode, prec)
            np.testing.assert_array_equal(got, want, err_msg=f"mode={mode} {prec} L={L} g={g} k={top_k} Kc={Kc}")
    got = oracle.dense(q, k, top_k)["out"]
    np.testing.assert_array_equal(got, brute.dense(q, k, top_k))


@pytest.mark.parametrize("seed", range(8))
def test_prefill_matches_brute_force_gaussian(seed):
    rng = np.random.default_rng(2000 + seed)
    L = int(rng.integers(20, 120))
    g = int(rng.choice([2, 4, 8]))
    q, k = synthetic.gen_prefill(L, 2, 16, seed=seed, rho=0.9)
    for mode in (oracle.REFINE, oracle.REUSE, oracle.REFINE_PER_MEMBER):
        for prec in oracle.PROXY_PRECISIONS:
            got = oracle.prefill(q, k, g, 6, 12, mode, proxy=prec)["out"]
            np.testing.assert_array_equal(got, brute.prefill(q, k, g, 6, 12, mode, prec), err_msg=f"{mode} {prec}")
    np.testing.assert_array_equal(oracle.dense(q, k, 6)["out"], brute.dense(q, k, 6))


@pytest.mark.parametrize("seed", range(6))
def test_decode_matches_brute_force(seed):
    rng = np.random.default_rng(3000 + seed)
    g = int(rng.choice([1, 2, 3]))
    B = int(rng.integers(1, 4))
    lens = rng.integers(0, 40, size=B) + g
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    H, d = 2, 4
    q = synthetic.bf16_from_f32(rng.integers(-2, 3, size=(B, g, H, d)).astype(np.float32))
    kc = synthetic.bf16_from_f32(rng.integers(-2, 3, size=(int(cu[-1]), H, d)).astype(np.float32))
    bi, hi = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    for mode in (oracle.REFINE, oracle.REUSE, oracle.REFINE_PER_MEMBER):
        for prec in oracle.PROXY_PRECISIONS:
            r = oracle.decode_units(q, kc, cu, g, 4, 9, mode, bi.ravel(), hi.ravel(), proxy=prec)
            got = r["out"].reshape(B, H, g, 4).transpose(0, 2, 1, 3)
            np.testing.assert_array_equal(got, brute.decode(q, kc, cu, g, 4, 9, mode, prec), err_msg=f"{mode} {prec}")


@pytest.mark.parametrize("seed", range(4))
def test_decode_gaussian_matches_brute_force(seed):
    """Gaussian decode inputs (fp32 means that are not bf16 values) for both
    proxy precisions."""
    g = 2 + seed % 2
    dec = synthetic.gen_decode(3, 2, 16, g, seed=50 + seed, lo=5, hi=60)
    bi, hi = np.meshgrid(np.arange(3), np.arange(2), indexing="ij")
    for mode in (oracle.REFINE, oracle.REUSE):
        for prec in oracle.PROXY_PRECISIONS:
            r = oracle.decode_units(dec.q, dec.kcache, dec.cu_seqlens, g, 5, 11, mode, bi.ravel(), hi.ravel(),
                                    proxy=prec)
            got = r["out"].reshape(3, 2, g, 5).transpose(0, 2, 1, 3)
            np.testing.assert_array_equal(got, brute.decode(dec.q, dec.kcache, dec.cu_seqlens, g, 5, 11, mode, prec))


# ------------------------------------------------------------ golden fixtures
def _load_worked():
    rows = {}
    vals = {}
    with open(os.path.join(GOLD, "worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, *rest = line.split()
            if head in ("keys", "queries", "proxies"):
                vals[head] = [[float(x) for x in v.split(",")] for v in rest]
            else:
                top_k, Kc = int(rest[0]), int(rest[1])
                body = " ".join(rest[2:]).split("|")
                rows[(head, top_k, Kc)] = [[int(x) for x in r.split(",")] for r in body]
    return vals, rows


def test_worked_example():
    vals, rows = _load_worked()
    k = bits(vals["keys"])[:, None, :]
    q = bits(vals["queries"])[:, None, :]
    for (mode, top_k, Kc), want in rows.items():
        if mode == "dense":
            got = oracle.dense(q, k, top_k)["out"][:, 0]
        else:
            m = oracle.REFINE if mode == "refine" else oracle.REUSE
            r = oracle.prefill(q, k, 2, top_k, Kc, m)
            got = r["out"][:, 0]
            np.testing.assert_array_equal(r["proxy"][:, 0], np.asarray(vals["proxies"], np.float32))
        np.testing.assert_array_equal(got, np.asarray(want), err_msg=f"{mode} k={top_k} Kc={Kc}")


def _proxy_cases(name):
    with open(os.path.join(GOLD, name)) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                members, want = ln.split()
                m = [float(x) for x in members.split(",")]
                n = len(m)
                q = bits(m)[:, None, None]                       # [n, 1, 1]: one group of n members
                k = bits([1.0] * n)[:, None, None]
                yield members, want, oracle.prefill_units(q, k, n, 1, 1, oracle.REFINE, [0], [0])


def test_proxy_rounding_fixture_fp32():
    """The proxy is the fp32 mean: hand-rounded cases, ties to even included."""
    from fractions import Fraction
    for members, want, r in _proxy_cases("proxy_rounding_fp32.txt"):
        got = r["proxy"][0][0]
        assert Fraction(float(got)) == Fraction(want), (members, float(got))


def test_proxy_rounding_fixture_bf16_variant():
    """The bf16 variant rounds the fp32 mean once more, to bf16."""
    for members, want, r in _proxy_cases("proxy_rounding.txt"):
        assert synthetic.bf16_to_f32(r["proxy_bf16"][0])[0] == np.float32(float(want)), members


def test_fp32_proxy_changes_the_candidate_set_where_bf16_rounding_would():
    """Closed form: two keys e_1 (index 0) and e_0 (index 1); a group of four
    members whose mean is (1 + 1/256, 1 + 1/512).  Both coordinates are exact
    in fp32, so key 1 (score 1 + 1/256) beats key 0 (score 1 + 1/512).  Rounded
    to bf16 both coordinates become 1, the scores tie and the tie goes to key 0.
    Keys 2..7 score -2.  With Kc = top_k = 1 every member of the group keeps
    the single candidate, and Reuse shares it."""
    L, d, g = 8, 2, 4
    k = np.full((L, 1, d), -1.0, np.float32)
    k[0, 0] = (0.0, 1.0)
    k[1, 0] = (1.0, 0.0)
    q = np.zeros((L, 1, d), np.float32)
    q[4:, 0, 0] = (1.0, 1.0, 1.0078125, 1.0078125)
    q[4:, 0, 1] = (1.0, 1.0, 1.0, 1.0078125)
    qb, kb = synthetic.bf16_from_f32(q), synthetic.bf16_from_f32(k)
    for mode in (oracle.REFINE, oracle.REUSE):
        f32 = oracle.prefill(qb, kb, g, 1, 1, mode)
        b16 = oracle.prefill(qb, kb, g, 1, 1, mode, proxy="bf16")
        assert f32["proxy"][1, 0].tolist() == [1.00390625, 1.001953125]
        assert synthetic.bf16_to_f32(b16["proxy_bf16"][1, 0]).tolist() == [1.0, 1.0]
        assert np.all(f32["out"][4:, 0, 0] == 1), f32["out"][4:, 0]
        assert np.all(b16["out"][4:, 0, 0] == 0), b16["out"][4:, 0]


# --------------------------------------------------------------- closed forms
def ramp_keys(L, d, sign=1.0):
    """k_j = sign*(j+1)*e_0 (exact in bf16 for j < 256)."""
    k = np.zeros((L, 1, d), np.float32)
    k[:, 0, 0] = sign * (np.arange(L) + 1)
    return synthetic.bf16_from_f32(k)


@pytest.mark.parametrize("top_k", [1, 3, 8])
def test_dense_ramp_picks_latest_keys(top_k):
    L, d = 40, 4
    q = np.zeros((L, 1, d), np.float32)
    q[:, 0, 0] = 1.0
    out = oracle.dense(synthetic.bf16_from_f32(q), ramp_keys(L, d), top_k)["out"][:, 0]
    for pos in range(L):
        want = list(range(max(0, pos - top_k), pos)) + [-1] * max(0, top_k - pos)
        assert list(out[pos]) == want, pos


def test_constant_keys_ties_go_to_lowest_index():
    L, d, top_k = 30, 4, 5
    rng = np.random.default_rng(7)
    q = synthetic.bf16_from_f32(rng.standard_normal((L, 1, d)).astype(np.float32))
    k = synthetic.bf16_from_f32(np.ones((L, 1, d), np.float32))
    want = np.array([[j if j < min(top_k, pos) else -1 for j in range(top_k)] for pos in range(L)])
    np.testing.assert_array_equal(oracle.dense(q, k, top_k)["out"][:, 0], want)
    for g in (2, 4):
        r = oracle.prefill(q, k, g, top_k, 2 * top_k, oracle.REFINE)["out"][:, 0]
        np.testing.assert_array_equal(r, want)
        r = oracle.prefill(q, k, g, top_k, 2 * top_k, oracle.REUSE)["out"][:, 0]
        for pos in range(L):
            s = (pos // g) * g
            assert list(r[pos]) == [j if j < min(top_k, s) else -1 for j in range(top_k)]


def test_refine_rescoring_uses_member_queries():
    """Proxy points up the ramp, the second member points down: its picks are the oldest candidates."""
    L, d, g, top_k, Kc = 48, 4, 2, 3, 6
    q = np.zeros((L, 1, d), np.float32)
    q[0::2, 0, 0] = 3.0     # first member of each group
    q[1::2, 0, 0] = -1.0    # second member; proxy = +1 e_0
    r = oracle.prefill(synthetic.bf16_from_f32(q), ramp_keys(L, d), g, top_k, Kc, oracle.REFINE)
    out = r["out"][:, 0]
    for s in range(0, L, g):
        last = s + 1
        C = list(range(max(0, last - Kc), last))            # the Kc largest j < last
        V0 = [j for j in C if j < s]
        assert list(out[s]) == (V0[-top_k:] + [-1] * (top_k - len(V0[-top_k:]))), s
        V1 = [j for j in C if j < s + 1]
        sel = V1[:top_k]
        assert list(out[s + 1]) == sel + [-1] * (top_k - len(sel)), s + 1


# ------------------------------------------------------------------ invariants
@pytest.mark.parametrize("seed", range(4))
def test_invariants(seed):
    rng = np.random.default_rng(4000 + seed)
    L, H, d = int(rng.integers(30, 90)), 2, 8
    q, k = synthetic.gen_prefill(L, H, d, seed=seed)
    top_k = int(rng.integers(2, 9))
    dense = oracle.dense(q, k, top_k)["out"]
    # g = 1: the proxy of one query is that query, so Refine and Reuse are dense.
    np.testing.assert_array_equal(oracle.prefill(q, k, 1, top_k, 2 * top_k, oracle.REFINE)["out"], dense)
    np.testing.assert_array_equal(oracle.prefill(q, k, 1, top_k, top_k, oracle.REUSE)["out"], dense)
    for g in (3, 8):
        # Kc >= every scan prefix: Refine sees every key and equals dense.
        np.testing.assert_array_equal(oracle.prefill(q, k, g, top_k, L, oracle.REFINE)["out"], dense)
        ref = oracle.prefill(q, k, g, top_k, 2 * top_k, oracle.REFINE)["out"]
        reu = oracle.prefill(q, k, g, top_k, 2 * top_k, oracle.REUSE)["out"]
        pos = np.arange(L)[:, None, None]
        for out in (ref, reu, dense):
            valid = out >= 0
            assert np.all(out[valid] < np.broadcast_to(pos, out.shape)[valid])       # causal
            # valid entries first, strictly ascending, unique
            assert np.all(np.diff(valid.astype(int), axis=-1) <= 0)
            o = np.where(valid, out, 10**9)
            assert np.all(np.diff(o, axis=-1)[valid[..., 1:]] > 0)
        for s in range(0, L, g):                                   # Reuse shared in a group
            e = min(s + g, L)
            assert np.all(reu[s:e] == reu[s])
        n_valid = (ref >= 0).sum(-1)
        want = np.minimum(top_k, np.arange(L))[:, None]
        if 2 * top_k >= top_k + g - 1:
            np.testing.assert_array_equal(n_valid, np.broadcast_to(want, n_valid.shape))
        np.testing.assert_array_equal((dense >= 0).sum(-1), np.broadcast_to(want, n_valid.shape))


def test_edges_and_scores_consistent():
    q, k = synthetic.gen_prefill(64, 1, 8, seed=11)
    r = oracle.dense(q, k, 4)
    qf, kf = brute.decode_bf16(q), brute.decode_bf16(k)
    for pos in range(5, 64):
        sel = r["out"][pos, 0]
        np.testing.assert_allclose(r["score"][pos, 0], kf[sel, 0] @ qf[pos, 0], rtol=1e-12)
        allsc = np.sort(kf[:pos, 0] @ qf[pos, 0])[::-1]
        np.testing.assert_allclose(r["edge"][pos, 0], allsc[3:5], rtol=1e-12)


def test_demo_shape_c0():
    """The pages' demo: S=1024, H=8, D=64, top_k=64, g=8 -> index shape (1024, 8, 64)."""
    q, k = synthetic.make_prefill("C0")
    c = synthetic.CONFIGS["C0"]
    r = oracle.prefill(q, k, c["g"], c["top_k"], c["Kc"], oracle.REFINE)
    assert r["out"].shape == (1024, 8, 64)
    assert np.all(r["out"][0] == -1)
    assert np.all((r["out"] >= 0).sum(-1)[1:] == np.minimum(64, np.arange(1, 1024))[:, None])


# ------------------------------------------------- the listing's own Refine
@pytest.mark.parametrize("seed", range(4))
def test_per_member_refine_reductions(seed):
    """The listing's Refine (a proxy scan per member over its own prefix):
    with g = 1 the proxy is the query, so it is the dense indexer; with
    Kc >= L every prefix is whole, so again dense; and a group's last member
    scans exactly the prefix of the single-scan reading, so its rows agree."""
    rng = np.random.default_rng(300 + seed)
    L, H, d, top_k = 150, 2, 16, 7
    q, k = synthetic.gen_prefill(L, H, d, seed=seed, rho=0.9)
    dense = oracle.dense(q, k, top_k)["out"]
    pm = oracle.REFINE_PER_MEMBER
    np.testing.assert_array_equal(oracle.prefill(q, k, 1, top_k, 2 * top_k, pm)["out"], dense)
    g = int(rng.choice([3, 4, 8]))
    np.testing.assert_array_equal(oracle.prefill(q, k, g, top_k, L, pm)["out"], dense)
    a = oracle.prefill(q, k, g, top_k, 2 * top_k, pm)["out"]
    b = oracle.prefill(q, k, g, top_k, 2 * top_k, oracle.REFINE)["out"]
    last = np.minimum(np.arange(0, L, g) + g, L) - 1
    np.testing.assert_array_equal(a[last], b[last])


def test_proxy_precisions_agree_for_single_members():
    """With g = 1 the mean of one bf16 query is that query exactly, in fp32 as
    in bf16, so both proxy precisions give the same rows (all three modes)."""
    q, k = synthetic.gen_prefill(120, 2, 16, seed=4, rho=0.9)
    for mode in (oracle.REFINE, oracle.REUSE, oracle.REFINE_PER_MEMBER):
        a = oracle.prefill(q, k, 1, 5, 10, mode)["out"]
        b = oracle.prefill(q, k, 1, 5, 10, mode, proxy="bf16")["out"]
        np.testing.assert_array_equal(a, b)


def test_threaded_oracle_runs_equal_serial_runs():
    """The tests and the bench spread oracle units over host threads; the
    joined results must be those of one serial call."""
    from tests.parity import oracle_threads
    q, k = synthetic.gen_prefill(300, 3, 16, seed=12, rho=0.9)
    gi = np.array([0, 5, 37, 12, 8, 20, 1], np.int32)
    hi = np.array([0, 1, 2, 2, 1, 0, 1], np.int32)
    for mode in (oracle.REFINE, oracle.REUSE):
        a = oracle.prefill_units(q, k, 8, 5, 11, mode, gi, hi, want_cand=True)
        b = oracle_threads(oracle.prefill_units, q, k, 8, 5, 11, mode, gi, hi, threads=3, want_cand=True)
        for key in a:
            np.testing.assert_array_equal(a[key], b[key], err_msg=key)


def test_member_candidate_edges_are_each_members_own_boundary():
    """In the listing's Refine each member's candidate set is the top-Kc of the
    group proxy's scores over its own prefix; the oracle reports that select's
    Kc-th and (Kc+1)-th scores per member (the near-tie test of the CUDA
    comparison).  Brute force: sort the member's prefix scores."""
    import tests.brute as brute
    L, H, d, g, top_k, Kc = 90, 2, 16, 4, 3, 10
    q, k = synthetic.gen_prefill(L, H, d, seed=21, rho=0.9)
    r = oracle.prefill(q, k, g, top_k, Kc, oracle.REFINE_PER_MEMBER)
    qd, kd = brute.decode_bf16(q), brute.decode_bf16(k)
    for h in range(H):
        for pos in range(L):
            s = pos // g * g
            proxy = qd[s:min(s + g, L), h].mean(axis=0).astype(np.float32).astype(np.float64)
            sc = np.sort(kd[:pos, h] @ proxy)[::-1]
            K = min(Kc, pos)
            exp = [sc[K - 1] if K >= 1 else np.nan, sc[K] if pos > K and K >= 1 else np.nan]
            np.testing.assert_allclose(r["member_cand_edge"][pos, h], exp, rtol=1e-12, atol=0)


# ------------------------------------------------- the sparse-attention consumer
def _attend_brute(q, k, v, idx, base=None):
    """numpy restatement: softmax over each row's valid indices of
    (q . k_j) / sqrt(d), times v_j; zeros for a row without indices."""
    import tests.brute as brute
    qd, kd, vd = brute.decode_bf16(q), brute.decode_bf16(k), brute.decode_bf16(v)
    R, H, d = qd.shape
    out = np.zeros((R, H, d))
    for r in range(R):
        b0 = 0 if base is None else base[r]
        for h in range(H):
            sel = idx[r, h][idx[r, h] >= 0] + b0
            if sel.size == 0:
                continue
            s = kd[sel, h] @ qd[r, h] / np.sqrt(d)
            w = np.exp(s - s.max())
            out[r, h] = (w / w.sum()) @ vd[sel, h]
    return out


def test_sparse_attention_matches_brute_force():
    rng = np.random.default_rng(40)
    L, H, d, top_k = 40, 3, 16, 6
    q, k = synthetic.gen_iid(L, H, d, seed=41)
    v, _ = synthetic.gen_iid(L, H, d, seed=42)
    idx = -np.ones((L, H, top_k), np.int32)
    for pos in range(L):
        for h in range(H):
            n = min(top_k, pos) - int(rng.integers(0, 2))
            if n > 0:
                idx[pos, h, :n] = np.sort(rng.choice(pos, size=n, replace=False))
    got = oracle.sparse_attention(q, k, v, idx)
    np.testing.assert_allclose(got, _attend_brute(q, k, v, idx), rtol=1e-12, atol=1e-12)
    # decode layout: rows of sequence b start at cu[b]
    B, g = 4, 2
    cu = np.array([0, 9, 20, 30, 40], np.int32)
    qd, _ = synthetic.gen_iid(B * g, H, d, seed=43)
    idx2 = -np.ones((B * g, H, top_k), np.int32)
    for r in range(B * g):
        n_b = int(cu[r // g + 1] - cu[r // g]) - g
        pos = n_b + r % g
        for h in range(H):
            idx2[r, h, :min(top_k, pos)] = np.sort(rng.choice(pos, size=min(top_k, pos), replace=False))
    got2 = oracle.sparse_attention(qd, k, v, idx2, cu_seqlens=cu, g=g)
    want2 = _attend_brute(qd, k, v, idx2, base=np.repeat(cu[:-1], g))
    np.testing.assert_allclose(got2, want2, rtol=1e-12, atol=1e-12)


def test_sparse_attention_closed_forms():
    """One index: the output is that value row exactly.  Equal keys: equal
    weights, the mean of the selected value rows.  No index: zeros.  The
    demo's shape ("Show Me The Code"): (1024, 8, 64)."""
    L, H, d = 12, 2, 8
    q, k = synthetic.gen_iid(L, H, d, seed=44)
    v, _ = synthetic.gen_iid(L, H, d, seed=45)
    import tests.brute as brute
    vd = brute.decode_bf16(v)
    idx = -np.ones((L, H, 4), np.int32)
    idx[5, 0, 0] = 3
    idx[7, 1, :3] = [0, 2, 6]
    kc = synthetic.bf16_from_f32(np.ones((L, H, d), np.float32))
    out = oracle.sparse_attention(q, kc, v, idx)
    np.testing.assert_array_equal(out[5, 0], vd[3, 0])
    np.testing.assert_allclose(out[7, 1], vd[[0, 2, 6], 1].mean(axis=0), rtol=1e-14, atol=1e-15)
    assert np.all(out[0] == 0) and np.all(out[6] == 0)
    q0, k0 = synthetic.make_prefill("C0")
    idx0 = np.zeros((1024, 8, 64), np.int32)
    assert oracle.sparse_attention(q0, k0, k0, idx0).shape == (1024, 8, 64)
