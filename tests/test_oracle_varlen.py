"""Pins of the oracle's packed-batch functions against a masked brute force.

A packed batch is several independent causal sequences laid end to end on the
token axis.  The oracle computes it by slicing each sequence out and running the
single-sequence definition (arXiv 2606.07703, Abstract; gist.science technical
report §2.1) on the slice.  The brute force here never slices: it works on the
whole packed axis with a block-diagonal causal mask (key j is visible to query i
iff both lie in the same sequence and j <= i), in numpy, and ranks keys by
counting.  A wrong sequence offset, a position that does not restart at 0, a key
leaking across sequences or a dropped empty sequence fails one of these tests.
"""
import numpy as np
import pytest

import tam_synth

CU = [0, 5, 5, 17, 40, 41, 70]            # includes an empty and a one-token sequence


def _packed(T, Hq, Hkv, d, seed):
    w = tam_synth.custom("v", T, Hq, Hkv, d, dtype="f32", seed=seed)
    inp = tam_synth.make_inputs(w)
    return inp.q.numpy(), inp.k.numpy(), inp.v.numpy()


def _mask(cu):
    cu = np.asarray(cu)
    T = cu[-1]
    seq = np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    i = np.arange(T)
    allowed = (seq[:, None] == seq[None, :]) & (i[None, :] <= i[:, None])
    return seq, allowed


def _brute_probs(q, k, cu):
    """Per-head softmax over the visible keys, [Hq, T, T] fp64."""
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    kh = k.astype(np.float64)[:, np.arange(Hq) // G, :]
    s = np.einsum("ihc,jhc->hij", q.astype(np.float64), kh) / np.sqrt(d)
    _, allowed = _mask(cu)
    s = np.where(allowed[None], s, -np.inf)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    return p / p.sum(axis=-1, keepdims=True)


def _rank_select(values, cand, budget):
    """Indices of the `budget` largest among `cand` (ties -> smaller index) by counting."""
    chosen = []
    for j in cand:
        rank = sum(1 for j2 in cand if values[j2] > values[j] or (values[j2] == values[j] and j2 < j))
        if rank < budget:
            chosen.append(j)
    return sorted(chosen)


def test_packed_mass_matches_masked_bruteforce(oracle_mod):
    q, k, _ = _packed(CU[-1], 4, 2, 8, seed=11)
    P = oracle_mod.varlen_mass_packed(q, k, CU)
    ref = _brute_probs(q, k, CU).mean(axis=0)
    np.testing.assert_allclose(P, ref, rtol=0, atol=1e-12)
    _, allowed = _mask(CU)
    assert np.all(P[~allowed] == 0)


@pytest.mark.parametrize("budget", [1, 3, 8])
def test_packed_per_query_support(oracle_mod, budget):
    q, k, _ = _packed(CU[-1], 4, 2, 8, seed=12)
    idx, ln, val = oracle_mod.varlen_support(q, k, CU, budget)
    P = _brute_probs(q, k, CU).mean(axis=0)
    seq, allowed = _mask(CU)
    cu = np.asarray(CU)
    assert idx.shape == (CU[-1], budget)
    for i in range(CU[-1]):
        t0 = cu[seq[i]]
        cand = list(np.nonzero(allowed[i])[0])
        want = [j - t0 for j in _rank_select(P[i], cand, budget)]   # local positions
        assert ln[i] == min(budget, i - t0 + 1)
        assert list(idx[i, :ln[i]]) == want, i
        assert np.all(idx[i, ln[i]:] == -1)
        np.testing.assert_allclose(val[i, :ln[i]], P[i, np.array(want) + t0], atol=1e-12)


@pytest.mark.parametrize("budget,block_q", [(3, 4), (6, 8)])
def test_packed_block_support(oracle_mod, budget, block_q):
    q, k, _ = _packed(CU[-1], 4, 2, 8, seed=13)
    idx, ln, val = oracle_mod.varlen_support(q, k, CU, budget, block_q)
    P = _brute_probs(q, k, CU).mean(axis=0)
    row = 0
    for t0, t1 in zip(CU[:-1], CU[1:]):
        for b0 in range(t0, t1, block_q):
            e = min(t1, b0 + block_q) - 1
            M = P[b0:e + 1].sum(axis=0)            # masked P is 0 for j > i and across sequences
            want = [j - t0 for j in _rank_select(M, list(range(t0, e + 1)), budget)]
            assert ln[row] == min(budget, e - t0 + 1)
            assert list(idx[row, :ln[row]]) == want, (t0, b0)
            np.testing.assert_allclose(val[row, :ln[row]], M[np.array(want) + t0], atol=1e-12)
            row += 1
    assert row == idx.shape[0]


def test_packed_dense_attention(oracle_mod):
    q, k, v = _packed(CU[-1], 4, 2, 8, seed=14)
    out, lse = oracle_mod.varlen_attn(q, k, v, CU)
    p = _brute_probs(q, k, CU)
    G = 2
    vh = v.astype(np.float64)[:, np.arange(4) // G, :]
    np.testing.assert_allclose(out, np.einsum("hij,jhc->ihc", p, vh), rtol=0, atol=1e-12)
    # lse of the visible scores, from the same masked scores
    T, Hq, d = q.shape
    kh = k.astype(np.float64)[:, np.arange(Hq) // G, :]
    s = np.einsum("ihc,jhc->hij", q.astype(np.float64), kh) / np.sqrt(d)
    _, allowed = _mask(CU)
    ref_lse = np.log(np.where(allowed[None], np.exp(s), 0).sum(axis=-1)).T
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("block_q", [1, 4])
def test_packed_sparse_attention_on_support(oracle_mod, block_q):
    q, k, v = _packed(CU[-1], 4, 2, 8, seed=15)
    budget = 4
    idx, ln, _ = oracle_mod.varlen_support(q, k, CU, budget, block_q)
    out, _ = oracle_mod.varlen_attn(q, k, v, CU, sup=idx, sup_len=ln, block_q=block_q)
    T, Hq, d = q.shape
    G = 2
    seq, _ = _mask(CU)
    cu = np.asarray(CU)
    kh = k.astype(np.float64)[:, np.arange(Hq) // G, :]
    vh = v.astype(np.float64)[:, np.arange(Hq) // G, :]
    sel0 = np.concatenate([[0], np.cumsum([(n if block_q == 1 else -(-n // block_q))
                                           for n in np.diff(cu)])])
    for i in range(T):
        s_, t0 = seq[i], cu[seq[i]]
        r = sel0[s_] + (i - t0) // block_q
        keys = [t0 + j for j in idx[r, :ln[r]] if j <= i - t0]
        sc = np.einsum("hc,jhc->hj", q[i].astype(np.float64), kh[keys]) / np.sqrt(d)
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(out[i], np.einsum("hj,jhc->hc", p, vh[keys]), atol=1e-12)


def _brute_indexer_scores(qx, kx, cu):
    s = qx.astype(np.float64) @ kx.astype(np.float64).T
    _, allowed = _mask(cu)
    return np.where(allowed, s, -np.inf), allowed


@pytest.mark.parametrize("budget", [1, 4, 9])
def test_packed_indexer_per_query(oracle_mod, budget):
    rng = np.random.default_rng(21)
    T = CU[-1]
    qx = rng.standard_normal((T, 16)).astype(np.float32)
    kx = rng.standard_normal((T, 16)).astype(np.float32)
    idx, ln, val = oracle_mod.varlen_indexer_support(qx, kx, CU, budget)
    s, allowed = _brute_indexer_scores(qx, kx, CU)
    seq, _ = _mask(CU)
    cu = np.asarray(CU)
    for i in range(T):
        t0 = cu[seq[i]]
        want = [j - t0 for j in _rank_select(s[i], list(np.nonzero(allowed[i])[0]), budget)]
        assert ln[i] == min(budget, i - t0 + 1)
        assert list(idx[i, :ln[i]]) == want, i
        np.testing.assert_allclose(val[i, :ln[i]], s[i, np.array(want) + t0], atol=1e-9)


@pytest.mark.parametrize("budget,block_q", [(3, 4), (5, 8)])
def test_packed_indexer_block(oracle_mod, budget, block_q):
    rng = np.random.default_rng(22)
    T = CU[-1]
    qx = rng.standard_normal((T, 16)).astype(np.float32)
    kx = rng.standard_normal((T, 16)).astype(np.float32)
    idx, ln, val = oracle_mod.varlen_indexer_support(qx, kx, CU, budget, block_q)
    s, _ = _brute_indexer_scores(qx, kx, CU)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)               # per-query softmax over visible keys
    row = 0
    for t0, t1 in zip(CU[:-1], CU[1:]):
        for b0 in range(t0, t1, block_q):
            e = min(t1, b0 + block_q) - 1
            M = p[b0:e + 1].sum(axis=0)
            want = [j - t0 for j in _rank_select(M, list(range(t0, e + 1)), budget)]
            assert ln[row] == min(budget, e - t0 + 1)
            assert list(idx[row, :ln[row]]) == want, (t0, b0)
            np.testing.assert_allclose(val[row, :ln[row]], M[np.array(want) + t0], atol=1e-12)
            row += 1
    assert row == idx.shape[0]
