"""Full-size workloads, in the launch configuration the benchmark times, checked on
sampled rows and blocks (rows are independent given K and V, so a sampled row is an
exact check of that row): the long-context sweep up to N = 102400 (block-shared,
B_q = 128, RoPE), the 32K head-collapsed indexer (k = 1024) with pass 3 on its
support, and the 32K random-support stress row."""
import numpy as np
import pytest
import torch

import tam_synth
from parity_util import LSE_ATOL, MASS_ATOL, OUT_ATOL, check_close, check_support

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("N", [65536, 102400])
def test_longctx_full(tam_lib, oracle_mod, N):
    w = tam_synth.WORKLOADS[f"longctx_{N}"]
    inp = tam_synth.make_inputs(w)
    bq, kb = w.block_q[0], w.budget_k
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    res = tam_lib.mass_oracle_prefill(q, k, v, kb, bq)
    torch.cuda.synchronize()
    nb = -(-N // bq)
    blocks = tam_synth.sample_blocks(nb, 4)
    gi, gl, gm = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    oi, ol, _ = oracle_mod.block_topk(inp.q, inp.k, bq, kb, blocks)
    M = oracle_mod.block_mass(inp.q, inp.k, bq, blocks)
    check_support(gi[blocks], gl[blocks], gm[blocks], oi, ol, M, MASS_ATOL * bq, f"longctx {N}")
    # outputs and lse on a few rows of those blocks
    r, s, sl = oracle_mod.block_rows_support(gi[blocks], gl[blocks], bq, N, blocks)
    pick = np.linspace(0, len(r) - 1, 48).astype(int)
    ref, _ = oracle_mod.attn_rows(inp.q, inp.k, inp.v, r[pick], sup=s[pick], sup_len=sl[pick])
    check_close(res.out.float().cpu().numpy()[r[pick]], ref, OUT_ATOL["bf16"], "longctx output")
    rows = np.concatenate([np.arange(8), [N // 2, N - 1]])
    check_close(res.lse.cpu().numpy()[:, rows].T, oracle_mod.lse_rows(inp.q, inp.k, rows),
                LSE_ATOL, "longctx lse")


def test_indexer32k_full(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w)
    res = tam_lib.indexer_topk(inp.q_idx.cuda(), inp.k_idx.cuda(), w.budget_k)
    out = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), res.idx,
                                           res.length, 1)
    torch.cuda.synchronize()
    rows = tam_synth.sample_rows(w.N, inp.needle_i, n_random=96)
    gi, gl, gs = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    oi, ol, _ = oracle_mod.indexer_topk_rows(inp.q_idx, inp.k_idx, w.budget_k, rows)
    S = inp.q_idx.double().numpy()[rows] @ inp.k_idx.double().numpy().T
    check_support(gi[rows], gl[rows], gs[rows], oi, ol, S, 1e-3, "indexer32k")
    ref, _ = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=gi[rows], sup_len=gl[rows])
    check_close(out.float().cpu().numpy()[rows], ref, OUT_ATOL["bf16"], "indexer32k output")


def test_stress_row_32k(tam_lib, oracle_mod):
    """Uniform-random support (the random-init stress row) at the 32K shape, k = 1024."""
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w)
    idx, ln = tam_synth.stress_support(w.N, 1024, seed=7)
    out, lse = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(),
                                                torch.from_numpy(idx).cuda(),
                                                torch.from_numpy(ln).cuda(), 1, return_lse=True)
    rows = tam_synth.sample_rows(w.N, n_random=64)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=idx[rows], sup_len=ln[rows])
    check_close(out.float().cpu().numpy()[rows], ref, OUT_ATOL["bf16"], "stress output")
    check_close(lse.cpu().numpy().T[rows], rl, LSE_ATOL, "stress lse")


def test_indexer32k_block_shared_full(tam_lib, oracle_mod):
    """The fused, selection-block-shared indexer at the 32K shape (k = 1024, B_q = 64),
    checked on sampled blocks, with pass 3 on a few of their rows."""
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w)
    bq = 64
    res = tam_lib.indexer_topk(inp.q_idx.cuda(), inp.k_idx.cuda(), w.budget_k, bq)
    out = tam_lib.sparse_support_attention(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), res.idx,
                                           res.length, bq)
    torch.cuda.synchronize()
    nb = -(-w.N // bq)
    blocks = tam_synth.sample_blocks(nb, 4)
    gi, gl, gm = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    oi, ol, _ = oracle_mod.indexer_block_topk(inp.q_idx, inp.k_idx, bq, w.budget_k, blocks)
    M = oracle_mod.indexer_block_mass(inp.q_idx, inp.k_idx, bq, blocks)
    check_support(gi[blocks], gl[blocks], gm[blocks], oi, ol, M, MASS_ATOL * bq, "indexer block 32k")
    r, s, sl = oracle_mod.block_rows_support(gi[blocks], gl[blocks], bq, w.N, blocks)
    pick = np.linspace(0, len(r) - 1, 32).astype(int)
    ref, _ = oracle_mod.attn_rows(inp.q, inp.k, inp.v, r[pick], sup=s[pick], sup_len=sl[pick])
    check_close(out.float().cpu().numpy()[r[pick]], ref, OUT_ATOL["bf16"], "indexer block output")


def test_distill_kl_32k_sampled_rows(tam_lib, oracle_mod):
    """The indexer's distillation target at the 32K shape, on sampled rows."""
    from parity_util import KL_ATOL
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    kl = tam_lib.distill_kl(q, k, lse, inp.q_idx.cuda(), inp.k_idx.cuda()).cpu().numpy()
    rows = tam_synth.sample_rows(w.N, inp.needle_i, n_random=24)
    check_close(kl[rows], oracle_mod.distill_kl_rows(inp.q, inp.k, inp.q_idx, inp.k_idx, rows),
                KL_ATOL, "distill kl 32k")


def test_per_query_65k_in_chunks(tam_lib, oracle_mod):
    """Per-query pass 2 at N = 65536 (16/4 heads, k = 2048): the mass rows (8.6 GB) exceed
    the 4 GiB preferred slab, so they go through in chunks; sampled rows vs the oracle."""
    w = tam_synth.WORKLOADS["longctx_65536"]
    inp = tam_synth.make_inputs(w)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    res = tam_lib.mass_select(q, k, lse, w.budget_k, 1)
    torch.cuda.synchronize()
    rows = np.concatenate([tam_synth.sample_rows(w.N, n_random=10), [w.N - 1, w.N // 2 + 31]])
    oi, ol, _ = oracle_mod.topk_rows(inp.q, inp.k, w.budget_k, rows)
    P = oracle_mod.mass_rows(inp.q, inp.k, rows)
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, P, MASS_ATOL, "per query 65k")
