"""Pins of the fp64 oracle against things other than itself.

Each test ties the oracle to a fact that the sources or plain mathematics fix:
a closed form, a textbook/library routine (torch SDPA, softmax), an invariant,
a brute force on tiny inputs, or the sparsity figures the technical report
prints (gist.science technical report on arXiv 2606.07703, §3.1).  The tests
are chosen so that a plausible mistake (a dropped scale, a wrong head map, a sum
for a mean, a reversed tie rule) fails at least one of them; test_oracle_mutations
plants exactly those mistakes and checks that they are caught.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import tam_synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(N, Hq, Hkv, d, seed=0, dtype="f32"):
    w = tam_synth.custom("t", N, Hq, Hkv, d, dtype=dtype, seed=seed)
    inp = tam_synth.make_inputs(w)
    return inp.q, inp.k, inp.v


# ---------------------------------------------------------------- closed forms / library routines

@pytest.mark.parametrize("N,Hq,Hkv,d", [(37, 4, 1, 16), (70, 8, 2, 32), (129, 4, 4, 16)])
def test_mass_rows_sum_to_one(oracle_mod, N, Hq, Hkv, d):
    q, k, _ = _rand(N, Hq, Hkv, d, seed=1)
    P = oracle_mod.mass_rows(q, k)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P >= 0)
    assert np.all(np.triu(P, 1) == 0)           # no mass on future keys


@pytest.mark.parametrize("N,Hq,Hkv,d", [(33, 4, 1, 16), (65, 8, 2, 32), (40, 6, 3, 8)])
def test_dense_equals_torch_sdpa(oracle_mod, N, Hq, Hkv, d):
    """Dense rows are ordinary causal GQA attention (torch SDPA in fp64, enable_gqa)."""
    q, k, v = _rand(N, Hq, Hkv, d, seed=2, dtype="bf16")
    out, lse = oracle_mod.attn_rows(q, k, v)
    qt = q.double().permute(1, 0, 2)[None]
    kt = k.double().permute(1, 0, 2)[None]
    vt = v.double().permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                           enable_gqa=True)
    ref = ref[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # lse against torch.logsumexp of explicitly formed scores
    G = Hq // Hkv
    kk = kt.repeat_interleave(G, dim=1)
    s = (qt @ kk.transpose(-1, -2)) / math.sqrt(d)
    mask = torch.ones(N, N, dtype=torch.bool).tril()
    s = s.masked_fill(~mask, float("-inf"))
    ref_lse = torch.logsumexp(s, dim=-1)[0].T.numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle_mod.lse_rows(q, k), ref_lse, rtol=0, atol=1e-12)


def test_single_head_mass_is_softmax(oracle_mod):
    """With Hq = Hkv = 1 the mass row is one softmax row."""
    N, d = 50, 16
    q, k, _ = _rand(N, 1, 1, d, seed=3)
    P = oracle_mod.mass_rows(q, k)
    s = (q.double()[:, 0] @ k.double()[:, 0].T) / math.sqrt(d)
    s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(P, torch.softmax(s, dim=-1).numpy(), rtol=0, atol=1e-13)


def test_zero_queries_closed_form(oracle_mod):
    """Q = 0: P_i[j] = 1/(i+1); the tie rule gives S_i = {0..k-1}; o = mean of V over S_i."""
    N, Hq, Hkv, d, kb = 40, 4, 2, 8, 5
    q, k, v = _rand(N, Hq, Hkv, d, seed=4)
    q = torch.zeros_like(q)
    P = oracle_mod.mass_rows(q, k)
    for i in range(N):
        np.testing.assert_allclose(P[i, :i + 1], 1.0 / (i + 1), rtol=1e-14)
    idx, ln, ms = oracle_mod.topk_rows(q, k, kb)
    for i in range(N):
        n = min(kb, i + 1)
        assert ln[i] == n
        assert list(idx[i, :n]) == list(range(n))
        assert np.all(idx[i, n:] == -1)
    out, _ = oracle_mod.attn_rows(q, k, v, sup=idx, sup_len=ln)
    G = Hq // Hkv
    for i in range(N):
        n = min(kb, i + 1)
        for h in range(Hq):
            ref = v[:n, h // G].double().mean(dim=0).numpy()
            np.testing.assert_allclose(out[i, h], ref, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- invariants

def test_full_budget_reproduces_dense(oracle_mod):
    """k >= i+1 selects every causal key, so the sparse output equals dense attention."""
    N, Hq, Hkv, d = 48, 8, 2, 16
    q, k, v = _rand(N, Hq, Hkv, d, seed=5, dtype="bf16")
    idx, ln, ms = oracle_mod.topk_rows(q, k, N)
    for i in range(N):
        assert ln[i] == i + 1 and list(idx[i, :i + 1]) == list(range(i + 1))
    sp, _ = oracle_mod.attn_rows(q, k, v, sup=idx, sup_len=ln)
    de, _ = oracle_mod.attn_rows(q, k, v)
    np.testing.assert_allclose(sp, de, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ms.sum(axis=1), 1.0, atol=1e-12)


def test_support_monotone_and_nested(oracle_mod):
    N, Hq, Hkv, d = 60, 4, 2, 16
    q, k, _ = _rand(N, Hq, Hkv, d, seed=6)
    prev_sets, prev_mass = None, None
    for kb in range(1, 20):
        idx, ln, ms = oracle_mod.topk_rows(q, k, kb)
        sets = [set(idx[i, :ln[i]].tolist()) for i in range(N)]
        mass = ms.sum(axis=1)
        if prev_sets is not None:
            assert all(a <= b for a, b in zip(prev_sets, sets))
            assert np.all(mass >= prev_mass - 1e-15)
        prev_sets, prev_mass = sets, mass


def test_key_shift_invariance(oracle_mod):
    """Adding one vector c to every key of a KV head shifts each score row by a constant."""
    N, Hq, Hkv, d = 45, 4, 2, 16
    q, k, v = _rand(N, Hq, Hkv, d, seed=7)
    # multiples of 1/16 keep k + c exact in fp32, so the only change is the shift itself
    k = torch.round(k * 16) / 16
    gen = torch.Generator().manual_seed(0)
    c = torch.round(torch.randn(d, generator=gen) * 8) / 16
    k2 = k.clone()
    k2[:, 1, :] += c
    P1, P2 = oracle_mod.mass_rows(q, k), oracle_mod.mass_rows(q, k2)
    np.testing.assert_allclose(P1, P2, rtol=0, atol=1e-12)
    idx, ln, _ = oracle_mod.topk_rows(q, k, 7)
    o1, _ = oracle_mod.attn_rows(q, k, v, sup=idx, sup_len=ln)
    o2, _ = oracle_mod.attn_rows(q, k2, v, sup=idx, sup_len=ln)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-11)


def test_block_of_one_equals_per_query(oracle_mod):
    N, Hq, Hkv, d, kb = 50, 8, 4, 16, 6
    q, k, _ = _rand(N, Hq, Hkv, d, seed=8)
    i1, l1, m1 = oracle_mod.topk_rows(q, k, kb)
    i2, l2, m2 = oracle_mod.block_topk(q, k, 1, kb)
    assert np.array_equal(i1, i2) and np.array_equal(l1, l2)
    np.testing.assert_allclose(m1, m2, rtol=0, atol=1e-15)


def test_block_mass_brute_force(oracle_mod):
    """M_b[j] = sum over the block's queries i >= j of P_i[j] (direct sum of mass rows)."""
    N, Hq, Hkv, d, Bq = 37, 4, 2, 8, 8
    q, k, _ = _rand(N, Hq, Hkv, d, seed=9)
    P = oracle_mod.mass_rows(q, k)
    M = oracle_mod.block_mass(q, k, Bq)
    nb = -(-N // Bq)
    for b in range(nb):
        ref = np.zeros(N)
        for i in range(b * Bq, min(N, (b + 1) * Bq)):
            for j in range(i + 1):
                ref[j] += P[i, j]
        np.testing.assert_allclose(M[b], ref, rtol=0, atol=1e-14)
        e = min(N, (b + 1) * Bq) - 1
        np.testing.assert_allclose(M[b].sum(), e - b * Bq + 1, atol=1e-12)


# ---------------------------------------------------------------- brute force (pure Python)

def _py_mass(qf, kf, N, Hq, Hkv, d):
    """P_i[j] by direct exp/sum (no log-sum-exp), pure Python floats."""
    G = Hq // Hkv
    P = [[0.0] * N for _ in range(N)]
    for i in range(N):
        for h in range(Hq):
            g = h // G
            e = []
            for j in range(i + 1):
                s = sum(qf[i][h][c] * kf[j][g][c] for c in range(d)) / math.sqrt(d)
                e.append(math.exp(s))
            z = sum(e)
            for j in range(i + 1):
                P[i][j] += e[j] / z / Hq
    return P


def _py_select(row, n, kb):
    """rank(j) = #{j': P[j'] > P[j] or (P[j'] == P[j] and j' < j)}; keep rank < k."""
    sel = []
    for j in range(n):
        rank = sum(1 for jj in range(n) if row[jj] > row[j] or (row[jj] == row[j] and jj < j))
        if rank < kb:
            sel.append(j)
    return sel


@pytest.mark.parametrize("N,Hq,Hkv,d,kb", [(24, 4, 2, 8, 3), (33, 2, 1, 4, 5), (16, 6, 3, 4, 2)])
def test_brute_force_tiny(oracle_mod, N, Hq, Hkv, d, kb):
    q, k, v = _rand(N, Hq, Hkv, d, seed=10 + N)
    qf, kf, vf = q.double().tolist(), k.double().tolist(), v.double().tolist()
    P = _py_mass(qf, kf, N, Hq, Hkv, d)
    np.testing.assert_allclose(oracle_mod.mass_rows(q, k), np.array(P), rtol=0, atol=1e-13)
    idx, ln, ms = oracle_mod.topk_rows(q, k, kb)
    out, _ = oracle_mod.attn_rows(q, k, v, sup=idx, sup_len=ln)
    G = Hq // Hkv
    for i in range(N):
        sel = _py_select(P[i], i + 1, kb)
        assert ln[i] == len(sel) and list(idx[i, :ln[i]]) == sel
        # exhaustive: the chosen set has the largest mass of all k-subsets
        n = i + 1
        if n <= 16 and kb <= 4 and n > kb:
            best = max(itertools.combinations(range(n), kb), key=lambda S: sum(P[i][j] for j in S))
            assert math.isclose(sum(P[i][j] for j in best), sum(P[i][j] for j in sel),
                                rel_tol=0, abs_tol=1e-15)
        # sparse output by the direct formula
        for h in range(Hq):
            g = h // G
            e = [math.exp(sum(qf[i][h][c] * kf[j][g][c] for c in range(d)) / math.sqrt(d))
                 for j in sel]
            z = sum(e)
            ref = [sum(e[t] / z * vf[j][g][c] for t, j in enumerate(sel)) for c in range(d)]
            np.testing.assert_allclose(out[i, h], ref, rtol=0, atol=1e-13)


def test_indexer_brute_force_and_closed_form(oracle_mod):
    N, dx, kb = 40, 6, 5
    g = torch.Generator().manual_seed(3)
    qx = torch.randn(N, dx, generator=g)
    kx = torch.randn(N, dx, generator=g)
    idx, ln, sc = oracle_mod.indexer_topk_rows(qx, kx, kb)
    qd, kd = qx.double().tolist(), kx.double().tolist()
    for i in range(N):
        row = [sum(qd[i][c] * kd[j][c] for c in range(dx)) for j in range(i + 1)]
        sel = _py_select(row, i + 1, kb)
        assert list(idx[i, :ln[i]]) == sel
        np.testing.assert_allclose(sc[i, :ln[i]], [row[j] for j in sel], rtol=0, atol=1e-13)
    # closed form: k_idx_j = j*e0 and q_idx_i[0] > 0 -> the last min(k, i+1) keys win
    kx2 = torch.zeros(N, dx)
    kx2[:, 0] = torch.arange(N, dtype=torch.float32)
    qx2 = torch.zeros(N, dx)
    qx2[:, 0] = 1.0
    idx2, ln2, _ = oracle_mod.indexer_topk_rows(qx2, kx2, kb)
    for i in range(N):
        n = min(kb, i + 1)
        assert list(idx2[i, :n]) == list(range(i + 1 - n, i + 1))


# ---------------------------------------------------------------- printed figures

def test_sparsity_endpoints_printed_in_report(oracle_mod):
    """Support size min(k, i+1) reproduces the 87.9 % / 96.0 % sparsity the report prints."""
    with open(os.path.join(GOLDEN, "sparsity_endpoints.json")) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        N, kb = case["N"], case["k"]
        sizes = np.minimum(kb, np.arange(N, dtype=np.int64) + 1)
        sp = 100.0 * oracle_mod.sparsity(sizes, N)
        assert round(sp, 1) == case["sparsity_pct_printed"], (N, kb, sp)
    # and the oracle's own supports have exactly that size
    q, k, _ = _rand(300, 4, 2, 8, seed=12)
    for kb in (1, 17, 256, 400):
        _, ln, _ = oracle_mod.topk_rows(q, k, kb)
        assert np.array_equal(ln, np.minimum(kb, np.arange(300) + 1))


# ------------------------------------------------------------------ block-shared indexer
def test_indexer_block_brute_force(oracle_mod):
    """Block sums of the per-query softmax of indexer scores, written out directly: exp of
    each score over the sum of exps (no log-sum-exp helper), summed over the block's
    queries with j <= i; selection by counting ranks."""
    N, dx, bq, kb = 37, 5, 8, 6
    g = torch.Generator().manual_seed(21)
    qx = torch.randn(N, dx, generator=g)
    kx = torch.randn(N, dx, generator=g)
    qd, kd = qx.double().tolist(), kx.double().tolist()
    nb = -(-N // bq)
    M = np.zeros((nb, N))
    for b in range(nb):
        for i in range(b * bq, min(N, (b + 1) * bq)):
            e = [math.exp(sum(qd[i][c] * kd[j][c] for c in range(dx))) for j in range(i + 1)]
            z = sum(e)
            for j in range(i + 1):
                M[b, j] += e[j] / z
    np.testing.assert_allclose(oracle_mod.indexer_block_mass(qx, kx, bq), M, rtol=0, atol=1e-12)
    idx, ln, ms = oracle_mod.indexer_block_topk(qx, kx, bq, kb)
    for b in range(nb):
        last = min(N, (b + 1) * bq) - 1
        sel = _py_select(list(M[b, :last + 1]), last + 1, kb)
        assert list(idx[b, :ln[b]]) == sel
        np.testing.assert_allclose(ms[b, :ln[b]], M[b, sel], rtol=0, atol=1e-12)


def test_indexer_block_invariants(oracle_mod):
    N, dx = 300, 16
    g = torch.Generator().manual_seed(22)
    qx = torch.randn(N, dx, generator=g) * 0.5
    kx = torch.randn(N, dx, generator=g) * 0.5
    # every query's softmax sums to one: a block's mass sums to its number of queries
    for bq in (1, 7, 64):
        M = oracle_mod.indexer_block_mass(qx, kx, bq)
        sizes = [min(N, (b + 1) * bq) - b * bq for b in range(M.shape[0])]
        np.testing.assert_allclose(M.sum(axis=1), sizes, rtol=1e-12)
    # a block of one query: softmax is monotone in the score, so the support is the
    # per-query indexer support and the values are the softmax probabilities
    idx1, ln1, _ = oracle_mod.indexer_block_topk(qx, kx, 1, 20)
    idx0, ln0, sc0 = oracle_mod.indexer_topk_rows(qx, kx, 20)
    assert np.array_equal(idx1, idx0) and np.array_equal(ln1, ln0)
    # q_idx = 0: every row is uniform, M_b[j] = sum_{i in b, i >= j} 1/(i+1) falls with j,
    # so the support is the first min(k, e_b+1) keys
    idx, ln, ms = oracle_mod.indexer_block_topk(torch.zeros(N, dx), kx, 64, 10)
    for b in range(len(ln)):
        last = min(N, (b + 1) * 64) - 1
        assert list(idx[b, :ln[b]]) == list(range(min(10, last + 1)))
        want = [sum(1.0 / (i + 1) for i in range(max(j, b * 64), last + 1)) for j in range(ln[b])]
        np.testing.assert_allclose(ms[b, :ln[b]], want, rtol=1e-12)


# ------------------------------------------------------------------ distillation target
def test_distill_kl_brute_force_and_zero(oracle_mod):
    """KL(P_i || softmax(indexer scores)) written out directly on a tiny input; it is
    zero when the indexer reproduces a one-head layer's own distribution, and positive
    otherwise."""
    N, Hq, Hkv, d, dx = 21, 4, 2, 8, 5
    q, k, _ = _rand(N, Hq, Hkv, d, seed=31)
    g = torch.Generator().manual_seed(32)
    qx, kx = torch.randn(N, dx, generator=g), torch.randn(N, dx, generator=g)
    P = _py_mass(q.double().tolist(), k.double().tolist(), N, Hq, Hkv, d)
    qd, kd = qx.double().tolist(), kx.double().tolist()
    want = []
    for i in range(N):
        e = [math.exp(sum(qd[i][c] * kd[j][c] for c in range(dx))) for j in range(i + 1)]
        z = sum(e)
        want.append(sum(P[i][j] * math.log(P[i][j] / (e[j] / z)) for j in range(i + 1)
                        if P[i][j] > 0))
    kl = oracle_mod.distill_kl_rows(q, k, qx, kx)
    np.testing.assert_allclose(kl, want, rtol=1e-10, atol=1e-12)
    assert np.all(kl[1:] > 0) and abs(kl[0]) < 1e-15          # row 0: both distributions are {0: 1}
    # one head, indexer = the layer's own scaled scores: identical distributions
    q1, k1, _ = _rand(N, 1, 1, 16, seed=33)
    kl0 = oracle_mod.distill_kl_rows(q1, k1, q1[:, 0, :] / 4.0, k1[:, 0, :])
    np.testing.assert_allclose(kl0, 0.0, atol=1e-12)


# ------------------------------------------------------------------ budget sweep
def test_support_mass_curve(oracle_mod):
    """The support mass at budget k equals the summed mass of the oracle's own top-k
    support (selection, a different code path), grows with k, and is 1 once k covers
    the causal prefix."""
    N = 200
    q, k, _ = _rand(N, 4, 2, 16, seed=41)
    ks = [1, 5, 32, 150, 300]
    curve = oracle_mod.support_mass_curve(q, k, ks)
    P = oracle_mod.mass_rows(q, k)
    for t, kb in enumerate(ks):
        idx, ln, ms = oracle_mod.topk_rows(q, k, kb)
        np.testing.assert_allclose(curve[:, t], ms.sum(axis=1), rtol=1e-12, atol=1e-15)
        direct = [P[i, idx[i, :ln[i]]].sum() for i in range(N)]
        np.testing.assert_allclose(curve[:, t], direct, rtol=1e-12, atol=1e-15)
    assert np.all(np.diff(curve, axis=1) >= -1e-15)
    full = np.arange(N) + 1 <= 300
    np.testing.assert_allclose(curve[full, -1], 1.0, rtol=1e-12)
