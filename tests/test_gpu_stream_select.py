"""The streamed per-query selection (sampled thresholds, candidate segments, fallback rows).

Per query, pass 2 and the indexer keep only the keys at or above a sampled threshold
and select exactly from those; rows whose candidates fall short or overflow are
recomputed whole on the CUDA cores.  These tests check, through the C ABI:
* the streamed supports and values are bit-identical to selecting from the
  materialised rows (TAM_MATERIALISE_ROWS=1), for the CTA-pair and single-CTA
  kernels and for the indexer: both select exactly over the same fp32 values;
* a workspace at its minimum size (many chunks) gives bit-identical results;
* rows forced onto the fallback path (threshold above every key, or below every key
  so that the segments overflow) still match the fp64 oracle;
* on the seeded workloads no row needs the fallback.
"""
import numpy as np
import pytest
import torch

import tam_synth
from parity_util import MASS_ATOL, check_support

pytestmark = pytest.mark.gpu


def _inputs(N, Hq, Hkv, d, seed, **kw):
    w = tam_synth.custom("s", N, Hq, Hkv, d, dtype="bf16", seed=seed, **kw)
    return tam_synth.make_inputs(w)


def _select(tam, q, k, lse, kb, ws, **kw):
    res = tam.mass_select(q, k, lse, kb, 1, workspace=ws, **kw)
    torch.cuda.synchronize()
    return res


SHAPES = [
    # N, Hq, Hkv, d, k      (G = 4, 8, 16 run on CTA pairs; G = 1, 2 on single CTAs)
    (3000, 32, 8, 128, 100),
    (2500, 16, 2, 128, 64),
    (2100, 16, 1, 64, 40),
    (2600, 4, 4, 128, 80),
    (2200, 8, 4, 64, 50),
    (4500, 32, 8, 128, 655),
]


@pytest.mark.parametrize("N,Hq,Hkv,d,kb", SHAPES)
def test_stream_equals_materialised_rows(tam_lib, monkeypatch, N, Hq, Hkv, d, kb):
    inp = _inputs(N, Hq, Hkv, d, seed=N + kb, sink=True, needles=6)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ws = tam_lib.Workspace()
    a = _select(tam_lib, q, k, lse, kb, ws)
    assert tam_lib.mass_fallback_rows(q, k, kb, ws) == 0
    monkeypatch.setenv("TAM_MATERIALISE_ROWS", "1")
    b = _select(tam_lib, q, k, lse, kb, tam_lib.Workspace())
    monkeypatch.delenv("TAM_MATERIALISE_ROWS")
    assert torch.equal(a.length, b.length)
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.value, b.value)


@pytest.mark.parametrize("N,kb", [(3000, 100), (5000, 1024), (2048, 7)])
def test_indexer_stream_equals_materialised_rows(tam_lib, monkeypatch, N, kb):
    inp = _inputs(N, 32, 8, 128, seed=N, sink=True, needles=4)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=3)
    qx, kx = qx.cuda(), kx.cuda()
    ws = tam_lib.Workspace()
    a = tam_lib.indexer_topk(qx, kx, kb, workspace=ws)
    torch.cuda.synchronize()
    assert tam_lib.indexer_fallback_rows(qx, kb, ws) == 0
    monkeypatch.setenv("TAM_MATERIALISE_ROWS", "1")
    b = tam_lib.indexer_topk(qx, kx, kb, workspace=tam_lib.Workspace())
    torch.cuda.synchronize()
    monkeypatch.delenv("TAM_MATERIALISE_ROWS")
    assert torch.equal(a.length, b.length)
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.value, b.value)


def test_minimum_workspace_gives_identical_results(tam_lib):
    N, kb = 6000, 300
    inp = _inputs(N, 32, 8, 128, seed=5, sink=True, needles=8)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    L = tam_lib.lib()
    lo = L.tam_mass_workspace_min(N, 32, 8, 128, tam_lib.TAM_BF16, kb, 1)
    hi = L.tam_mass_oracle_workspace(N, 32, 8, 128, tam_lib.TAM_BF16, kb, 1)
    assert hi > 4 * lo                      # the small one really runs in several chunks
    a = _select(tam_lib, q, k, lse, kb, tam_lib.Workspace())
    b = _select(tam_lib, q, k, lse, kb, tam_lib.Workspace(), workspace_bytes=lo)
    assert torch.equal(a.idx, b.idx) and torch.equal(a.length, b.length)
    assert torch.equal(a.value, b.value)


@pytest.mark.parametrize("force", ["1", "2"])
def test_forced_fallback_rows_match_the_oracle(tam_lib, oracle_mod, monkeypatch, force):
    """force=1: every sampled row gets a threshold above all of its keys (no candidate,
    too few keys); force=2: a threshold below all of them (every key passes, the
    segments overflow).  Either way those rows are recomputed on the CUDA cores."""
    N, kb = 2600, 60
    inp = _inputs(N, 32, 8, 128, seed=11, sink=True, needles=5)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ws = tam_lib.Workspace()
    monkeypatch.setenv("TAM_DEBUG_FORCE_FALLBACK", force)
    res = _select(tam_lib, q, k, lse, kb, ws)
    n_fb = tam_lib.mass_fallback_rows(q, k, kb, ws)
    monkeypatch.delenv("TAM_DEBUG_FORCE_FALLBACK")
    assert n_fb > N // 2
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(N - 200, N),
                                     np.linspace(0, N - 1, 120).astype(np.int64)]))
    gi, gl, gm = (res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy())
    oi, ol, _ = oracle_mod.topk_rows(inp.q, inp.k, kb, rows)
    P = oracle_mod.mass_rows(inp.q, inp.k, rows)
    check_support(gi[rows], gl[rows], gm[rows], oi, ol, P, MASS_ATOL, "forced fallback")


@pytest.mark.parametrize("force", ["1", "2"])
def test_forced_fallback_indexer_rows_match_the_oracle(tam_lib, oracle_mod, monkeypatch, force):
    N, kb = 2600, 60
    inp = _inputs(N, 32, 8, 128, seed=12, sink=True, needles=5)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=4)
    ws = tam_lib.Workspace()
    monkeypatch.setenv("TAM_DEBUG_FORCE_FALLBACK", force)
    res = tam_lib.indexer_topk(qx.cuda(), kx.cuda(), kb, workspace=ws)
    torch.cuda.synchronize()
    n_fb = tam_lib.indexer_fallback_rows(qx.cuda(), kb, ws)
    monkeypatch.delenv("TAM_DEBUG_FORCE_FALLBACK")
    assert n_fb > N // 2
    rows = np.linspace(0, N - 1, 150).astype(np.int64)
    oi, ol, _ = oracle_mod.indexer_topk_rows(qx, kx, kb, rows)
    S = qx.double().numpy()[rows] @ kx.double().numpy().T     # value lookup for the check
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, S, 1e-3, "forced indexer fallback")


@pytest.mark.slow
def test_gqa32k_needs_no_fallback(tam_lib):
    w = tam_synth.WORKLOADS["gqa32k_2pct"]
    inp = tam_synth.make_inputs(w)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ws = tam_lib.Workspace()
    _select(tam_lib, q, k, lse, w.budget_k, ws)
    assert tam_lib.mass_fallback_rows(q, k, w.budget_k, ws) == 0


def test_rope_grid_needles_need_almost_no_fallback(tam_lib, oracle_mod):
    """The long-context tensors (RoPE, sink, needles on a grid of N/32 positions) per
    query: the sampled thresholds hold (at most one row in a thousand falls back), and
    sampled rows match the oracle."""
    w = tam_synth.WORKLOADS["longctx_16384"]
    inp = tam_synth.make_inputs(w)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ws = tam_lib.Workspace()
    kb = 655
    res = _select(tam_lib, q, k, lse, kb, ws)
    assert tam_lib.mass_fallback_rows(q, k, kb, ws) <= w.N // 1000
    rows = tam_synth.sample_rows(w.N, inp.needle_i, n_random=64)
    oi, ol, _ = oracle_mod.topk_rows(inp.q, inp.k, kb, rows)
    P = oracle_mod.mass_rows(inp.q, inp.k, rows)
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, P, MASS_ATOL, "rope grid needles")
