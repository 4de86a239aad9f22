"""Tensor-core kernels (bf16): pass-1 LSE for every head-group size, the row top-k
on long rows, in workspace-bounded chunks and under massive ties (more tied keys
than the selection stages in shared memory), and the device error paths.

The error-path tests fault nothing: a debug environment switch parks one role of
the kernel on a barrier nobody arrives on (its bounded wait gives up after 20 ms
and the kernel winds down).  The next call on the same context must succeed.
"""
import numpy as np
import pytest
import torch

import tam_synth
from parity_util import LSE_ATOL, MASS_ATOL, OUT_ATOL, check_close, check_support

pytestmark = pytest.mark.gpu


def _inputs(N, Hq, Hkv, d, seed=0, **kw):
    w = tam_synth.custom("tc", N, Hq, Hkv, d, dtype="bf16", seed=seed, **kw)
    return tam_synth.make_inputs(w)


@pytest.mark.parametrize("N,Hq,Hkv,d", [
    (1, 4, 1, 128), (100, 4, 1, 64), (128, 8, 8, 128), (129, 16, 8, 128), (300, 32, 8, 128),
    (1000, 16, 1, 64), (777, 32, 2, 128), (513, 16, 16, 64), (260, 32, 4, 128)])
def test_attention_lse_shapes(tam_lib, oracle_mod, N, Hq, Hkv, d):
    inp = _inputs(N, Hq, Hkv, d, seed=N + Hq, sink=True)
    lse = tam_lib.attention_lse(inp.q.cuda(), inp.k.cuda())
    check_close(lse.cpu().numpy().T, oracle_mod.lse_rows(inp.q, inp.k), LSE_ATOL, "lse")


@pytest.mark.parametrize("N,Hq,Hkv,d,kb", [(3000, 8, 2, 128, 8), (2049, 32, 8, 128, 1),
                                           (1500, 4, 1, 64, 300), (700, 16, 4, 128, 64)])
def test_mass_select_small_budget_long_rows(tam_lib, oracle_mod, N, Hq, Hkv, d, kb):
    """Small k on long rows: the row top-k keeps a few keys of thousands."""
    inp = _inputs(N, Hq, Hkv, d, seed=kb, sink=True, needles=4)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    res = tam_lib.mass_select(q, k, lse, kb, 1)
    rows = tam_synth.sample_rows(N, inp.needle_i, n_random=96)
    oi, ol, _ = oracle_mod.topk_rows(inp.q, inp.k, kb, rows)
    P = oracle_mod.mass_rows(inp.q, inp.k, rows)
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, P, MASS_ATOL, "small budget")


@pytest.mark.parametrize("N,bq", [(1200, 1), (1200, 64), (9000, 1)])
def test_massive_ties_keep_smallest_indices(tam_lib, N, bq):
    """Identical keys make every mass of a row equal; the smallest indices must win.
    At N = 9000 the tie at the k-th value spans more keys than the row top-k can
    stage in shared memory (8192), which takes its bisection path."""
    kb = 50
    inp = _inputs(N, 8, 2, 128, seed=2)
    k = inp.k.clone()
    k[:] = k[0:1]
    q = inp.q.cuda()
    kc = k.cuda()
    lse = tam_lib.attention_lse(q, kc)
    res = tam_lib.mass_select(q, kc, lse, kb, bq)
    gi, gl = res.idx.cpu().numpy(), res.length.cpu().numpy()
    for r in range(len(gl)):
        last = r if bq == 1 else min(N, (r + 1) * bq) - 1
        n = min(kb, last + 1)
        assert gl[r] == n and list(gi[r, :n]) == list(range(n)), r


def test_block_mass_values(tam_lib, oracle_mod):
    """Block-shared mass of the selected keys vs the oracle's M_b, several block sizes."""
    inp = _inputs(1100, 32, 8, 128, seed=4, sink=True)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    for bq in (16, 64, 100, 128):
        res = tam_lib.mass_select(q, k, lse, 90, bq)
        oi, ol, _ = oracle_mod.block_topk(inp.q, inp.k, bq, 90)
        M = oracle_mod.block_mass(inp.q, inp.k, bq)
        check_support(res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy(),
                      oi, ol, M, MASS_ATOL * bq, f"block {bq}")


def test_forced_wait_timeout_is_reported(tam_lib, oracle_mod, monkeypatch):
    inp = _inputs(300, 8, 2, 128, seed=6)
    q, k = inp.q.cuda(), inp.k.cuda()
    monkeypatch.setenv("TAM_DEBUG_FORCE_TIMEOUT", "1")
    with pytest.raises(tam_lib.TamError) as e:
        tam_lib.attention_lse(q, k)
    assert e.value.code == tam_lib.TAM_ERR_TIMEOUT
    lse_ref = tam_lib.attention_lse  # same call, switch off: the context must still work
    monkeypatch.delenv("TAM_DEBUG_FORCE_TIMEOUT")
    lse = lse_ref(q, k)
    check_close(lse.cpu().numpy().T, oracle_mod.lse_rows(inp.q, inp.k), LSE_ATOL, "lse after")
    monkeypatch.setenv("TAM_DEBUG_FORCE_TIMEOUT", "1")
    with pytest.raises(tam_lib.TamError) as e:
        tam_lib.mass_select(q, k, lse, 16, 1)
    assert e.value.code == tam_lib.TAM_ERR_TIMEOUT
    monkeypatch.delenv("TAM_DEBUG_FORCE_TIMEOUT")
    tam_lib.mass_select(q, k, lse, 16, 1)


@pytest.mark.parametrize("frac", [0.3, 0.0])
def test_mass_select_in_workspace_bounded_chunks(tam_lib, frac):
    """Per query the mass rows go through a slab in the workspace.  A workspace below
    the preferred size (frac of the way from the minimum to it; 0 = the minimum) means
    more chunks and must give bit-identical supports; one byte less than the minimum
    is refused before anything runs."""
    N, Hq, Hkv, d, kb = 3000, 32, 8, 128, 100
    inp = _inputs(N, Hq, Hkv, d, seed=5, sink=True, needles=4)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ref = tam_lib.mass_select(q, k, lse, kb, 1)
    L = tam_lib.lib()
    pref = L.tam_mass_select_workspace(N, Hq, Hkv, d, 0, kb, 1)
    lo = L.tam_mass_workspace_min(N, Hq, Hkv, d, 0, kb, 1)
    assert 0 < lo < pref
    res = tam_lib.mass_select(q, k, lse, kb, 1, workspace_bytes=int(lo + frac * (pref - lo)))
    assert torch.equal(res.length, ref.length) and torch.equal(res.idx, ref.idx)
    assert torch.equal(res.value, ref.value)
    with pytest.raises(tam_lib.TamError) as e:
        tam_lib.mass_select(q, k, lse, kb, 1, workspace_bytes=lo - 1)
    assert e.value.code == tam_lib.TAM_ERR_WORKSPACE


def test_indexer_in_workspace_bounded_chunks(tam_lib):
    N, kb = 2500, 300
    inp = _inputs(N, 8, 2, 128, seed=6, sink=True, needles=5)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    qx, kx = qx.cuda(), kx.cuda()
    ref = tam_lib.indexer_topk(qx, kx, kb)
    lo = tam_lib.lib().tam_indexer_workspace_min(N, 64, 0, kb, 1)
    res = tam_lib.indexer_topk(qx, kx, kb, workspace_bytes=lo)
    assert torch.equal(res.length, ref.length) and torch.equal(res.idx, ref.idx)
    assert torch.equal(res.value, ref.value)


@pytest.mark.parametrize("N,Hq,Hkv,d", [(129, 8, 8, 128), (700, 32, 2, 128), (450, 16, 8, 64),
                                        (1000, 32, 8, 128), (257, 8, 1, 128), (3000, 16, 4, 128)])
def test_dense_tensorcore_shapes(tam_lib, oracle_mod, N, Hq, Hkv, d):
    inp = _inputs(N, Hq, Hkv, d, seed=N, sink=True, needles=3)
    out, lse = tam_lib.dense_gqa_prefill(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), return_lse=True)
    rows = tam_synth.sample_rows(N, inp.needle_i, n_random=64) if N > 1000 else None
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows)
    got = out.float().cpu().numpy()
    gl = lse.cpu().numpy().T
    if rows is not None:
        got, gl = got[rows], gl[rows]
    check_close(got, ref, OUT_ATOL["bf16"], "dense")
    check_close(gl, rl, LSE_ATOL, "dense lse")


@pytest.mark.parametrize("N,Hq,Hkv,d", [(1, 4, 1, 64), (333, 32, 8, 128), (1000, 16, 4, 64),
                                         (2100, 8, 8, 128), (777, 16, 1, 128)])
def test_dense_on_the_two_tile_pipeline(tam_lib, oracle_mod, monkeypatch, N, Hq, Hkv, d):
    """The A/B form of the dense comparator (TAM_DENSE_PAIR_TILES=1: the block-shared
    pass-3 pipeline over every key, two query tiles per CTA, odd tile counts included)."""
    inp = _inputs(N, Hq, Hkv, d, seed=N + 1, sink=True)
    monkeypatch.setenv("TAM_DENSE_PAIR_TILES", "1")
    out, lse = tam_lib.dense_gqa_prefill(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), return_lse=True)
    torch.cuda.synchronize()
    monkeypatch.delenv("TAM_DENSE_PAIR_TILES")
    rows = tam_synth.sample_rows(N, n_random=64) if N > 1000 else None
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows)
    got, gl = out.float().cpu().numpy(), lse.cpu().numpy().T
    if rows is not None:
        got, gl = got[rows], gl[rows]
    check_close(got, ref, OUT_ATOL["bf16"], "dense, two-tile pipeline")
    check_close(gl, rl, LSE_ATOL, "dense lse, two-tile pipeline")


@pytest.mark.parametrize("N,Hq,Hkv,d", [(700, 32, 8, 128), (300, 8, 2, 64), (260, 8, 2, 256),
                                         (150, 16, 1, 128)])
def test_gather_skips_invalid_support_entries(tam_lib, oracle_mod, N, Hq, Hkv, d):
    """Per-query pass 3 on supports mixing valid keys with negative ones, keys after the
    query and keys past the sequence (never read): the result is the oracle's on the
    valid entries, and a row with no valid entry gives a zero row and lse = -inf."""
    inp = _inputs(N, Hq, Hkv, d, seed=N + d, sink=True)
    rng = np.random.default_rng(N + d)
    kmax = 48
    sup = rng.integers(0, N, size=(N, kmax)).astype(np.int32)      # about half after i
    sup[:, ::5] = -7
    sup[:, 1::7] = N + 1000000
    sup[:, 2::9] = np.iinfo(np.int32).max
    ln = rng.integers(0, kmax + 1, size=N).astype(np.int32)
    ln[N // 2] = kmax
    sup[N // 2, :] = -1
    out, lse = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(),
                                                torch.from_numpy(sup).cuda(),
                                                torch.from_numpy(ln).cuda(), 1, return_lse=True)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, None, sup=sup, sup_len=ln)
    check_close(out.float().cpu().numpy(), ref, OUT_ATOL["bf16"], "pass 3, invalid entries")
    check_close(lse.cpu().numpy().T, rl, LSE_ATOL, "pass 3 lse, invalid entries")
    assert not out[N // 2].float().abs().any()


@pytest.mark.parametrize("N,Hq,Hkv,d,kb,bq", [
    (600, 8, 8, 128, 50, 1), (600, 32, 2, 128, 50, 1), (500, 16, 8, 64, 33, 1),
    (900, 32, 8, 128, 100, 64), (900, 16, 4, 128, 200, 128), (500, 8, 2, 128, 40, 8),
    (400, 32, 2, 64, 60, 16), (300, 4, 4, 128, 17, 100)])
def test_sparse_attention_gather_shapes(tam_lib, oracle_mod, N, Hq, Hkv, d, kb, bq):
    """Pass 3 on a random support for every head-group size, per query and block-shared
    (large blocks use the shared-chunk kernel, small ones the per-query gather)."""
    inp = _inputs(N, Hq, Hkv, d, seed=kb)
    n_sel = N if bq == 1 else -(-N // bq)
    last = np.arange(n_sel) if bq == 1 else np.minimum(N - 1, (np.arange(n_sel) + 1) * bq - 1)
    idx, ln = tam_synth.stress_support(N, kb, seed=3, rows=last)
    out, lse = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(),
                                                torch.from_numpy(idx).cuda(),
                                                torch.from_numpy(ln).cuda(), bq, return_lse=True)
    if bq == 1:
        rows, s, sl = np.arange(N), idx, ln
    else:
        rows, s, sl = oracle_mod.block_rows_support(idx, ln, bq, N)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=s, sup_len=sl)
    check_close(out.float().cpu().numpy()[rows], ref, OUT_ATOL["bf16"], "gather output")
    check_close(lse.cpu().numpy().T[rows], rl, LSE_ATOL, "gather lse")


@pytest.mark.parametrize("N", [900, 9000])
def test_indexer_ties_keep_smallest_indices(tam_lib, N):
    """q_idx = 0 makes every score 0: the smallest key indices must be chosen."""
    kb = 40
    inp = _inputs(N, 8, 2, 128, seed=3)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    qx = torch.zeros_like(qx)
    res = tam_lib.indexer_topk(qx.cuda(), kx.cuda(), kb)
    gi, gl, gs = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    for i in range(N):
        n = min(kb, i + 1)
        assert gl[i] == n and list(gi[i, :n]) == list(range(n)) and np.all(gs[i, :n] == 0)


@pytest.mark.parametrize("N,kb", [(3000, 4), (2500, 300)])
def test_indexer_small_budget_long_rows(tam_lib, oracle_mod, N, kb):
    inp = _inputs(N, 8, 2, 128, seed=kb, sink=True, needles=5)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    res = tam_lib.indexer_topk(qx.cuda(), kx.cuda(), kb)
    rows = tam_synth.sample_rows(N, inp.needle_i, n_random=80)
    oi, ol, _ = oracle_mod.indexer_topk_rows(qx, kx, kb, rows)
    S = qx.double().numpy()[rows] @ kx.double().numpy().T
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, S, 1e-3, "indexer small budget")


def test_indexer_forced_timeout_is_reported(tam_lib, monkeypatch):
    inp = _inputs(400, 8, 2, 128, seed=9)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    qx, kx = qx.cuda(), kx.cuda()
    monkeypatch.setenv("TAM_DEBUG_FORCE_TIMEOUT", "1")
    with pytest.raises(tam_lib.TamError) as e:
        tam_lib.indexer_topk(qx, kx, 32)
    assert e.value.code == tam_lib.TAM_ERR_TIMEOUT
    monkeypatch.delenv("TAM_DEBUG_FORCE_TIMEOUT")
    res = tam_lib.indexer_topk(qx, kx, 32)
    assert int(res.length[-1]) == 32


@pytest.mark.parametrize("N,Hq,Hkv,d,kb,bq", [(1500, 32, 8, 128, 100, 1), (1500, 32, 8, 128, 100, 64),
                                              (777, 16, 2, 128, 40, 1), (900, 32, 4, 64, 60, 1),
                                              (2100, 16, 4, 128, 300, 128), (300, 64, 4, 128, 30, 1)])
def test_pair_kernel_matches_single_cta_kernel(tam_lib, oracle_mod, monkeypatch, N, Hq, Hkv, d, kb, bq):
    """The 2-SM pass-2 kernel and the single-CTA one give the same supports (and both
    match the oracle)."""
    inp = _inputs(N, Hq, Hkv, d, seed=N + kb, sink=True, needles=4)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    a = tam_lib.mass_select(q, k, lse, kb, bq)
    monkeypatch.setenv("TAM_DISABLE_PAIR_KERNELS", "1")
    b = tam_lib.mass_select(q, k, lse, kb, bq)
    monkeypatch.delenv("TAM_DISABLE_PAIR_KERNELS")
    assert torch.equal(a.length, b.length)
    assert torch.equal(a.idx, b.idx)
    assert (a.value - b.value).abs().max().item() <= 1e-6 * bq
    if bq == 1:
        rows = tam_synth.sample_rows(N, inp.needle_i, n_random=48)
        oi, ol, _ = oracle_mod.topk_rows(inp.q, inp.k, kb, rows)
        P = oracle_mod.mass_rows(inp.q, inp.k, rows)
        check_support(a.idx.cpu().numpy()[rows], a.length.cpu().numpy()[rows],
                      a.value.cpu().numpy()[rows], oi, ol, P, MASS_ATOL, "pair")


@pytest.mark.parametrize("N,Hq,Hkv,d,kb,bq", [(1000, 32, 8, 128, 100, 64), (777, 16, 4, 128, 300, 128),
                                              (600, 8, 1, 64, 80, 64), (513, 16, 2, 128, 50, 32)])
def test_block_pass3_tensorcore_matches(tam_lib, oracle_mod, monkeypatch, N, Hq, Hkv, d, kb, bq):
    """Block-shared pass 3 on tcgen05 over gathered chunks agrees with the oracle and with
    the mma.sync kernel (TAM_DISABLE_BLOCK_TC=1)."""
    inp = _inputs(N, Hq, Hkv, d, seed=N + bq, sink=True, needles=3)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    lse0 = tam_lib.attention_lse(q, k)
    sup = tam_lib.mass_select(q, k, lse0, kb, bq)
    out, lse = tam_lib.sparse_support_attention(q, k, v, sup.idx, sup.length, bq, return_lse=True)
    monkeypatch.setenv("TAM_DISABLE_BLOCK_TC", "1")
    out2, lse2 = tam_lib.sparse_support_attention(q, k, v, sup.idx, sup.length, bq, return_lse=True)
    monkeypatch.delenv("TAM_DISABLE_BLOCK_TC")
    gi, gl = sup.idx.cpu().numpy(), sup.length.cpu().numpy()
    rows, s, sl = oracle_mod.block_rows_support(gi, gl, bq, N)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=s, sup_len=sl)
    check_close(out.float().cpu().numpy()[rows], ref, OUT_ATOL["bf16"], "block tc output")
    check_close(lse.cpu().numpy().T[rows], rl, LSE_ATOL, "block tc lse")
    assert (out.float() - out2.float()).abs().max().item() <= OUT_ATOL["bf16"]


def test_block_pass3_tensorcore_empty_rows(tam_lib, oracle_mod):
    """Hand-made block supports: queries before their block's first key (and a tile with
    none at all) get a zero row and lse = -inf; keys past a query are masked."""
    N, Hq, Hkv, d, bq, kmax = 256, 16, 4, 128, 64, 8
    inp = _inputs(N, Hq, Hkv, d, seed=9)
    rows_sup = [[40, 41, 42, 50], [0, 5, 100, 120, 127], [], [255]]
    idx = np.full((4, kmax), -1, np.int32)
    ln = np.zeros(4, np.int32)
    for b, r in enumerate(rows_sup):
        idx[b, :len(r)] = r
        ln[b] = len(r)
    out, lse = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(),
                                                torch.from_numpy(idx).cuda(),
                                                torch.from_numpy(ln).cuda(), bq, return_lse=True)
    rows, s, sl = oracle_mod.block_rows_support(idx, ln, bq, N)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=s, sup_len=sl)
    o = out.float().cpu().numpy()[rows]
    check_close(o, ref, OUT_ATOL["bf16"], "block tc output (empty rows)")
    lg = lse.cpu().numpy().T[rows]
    empty = ~np.isfinite(rl)
    assert np.array_equal(empty, ~np.isfinite(lg))
    assert np.all(o[empty.all(axis=1)] == 0)
    check_close(lg[~empty], rl[~empty], LSE_ATOL, "block tc lse (empty rows)")
