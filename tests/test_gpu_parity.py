"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small shapes span several 128-wide tiles and ragged tails; the workload shapes
are checked on sampled rows and blocks (rows are independent given K and V, so
a sampled row is an exact check of that row).
"""
import numpy as np
import pytest
import torch

import tam_synth
from parity_util import KL_ATOL, LSE_ATOL, MASS_ATOL, OUT_ATOL, check_close, check_support

pytestmark = pytest.mark.gpu


def _inputs(N, Hq, Hkv, d, dtype="bf16", seed=0, **kw):
    w = tam_synth.custom("p", N, Hq, Hkv, d, dtype=dtype, seed=seed, **kw)
    return tam_synth.make_inputs(w)


def _cuda(*ts):
    return [None if t is None else t.cuda() for t in ts]


def run_mass_case(tam, oracle, inp, budget, block_q, rows=None, blocks=None, dtype="bf16"):
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    N, Hq, d = inp.q.shape
    res = tam.mass_oracle_prefill(q, k, v, budget, block_q)
    torch.cuda.synchronize()
    gi, gl, gm = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    out = res.out.float().cpu().numpy()
    lse = res.lse.cpu().numpy()
    if rows is None:
        rows = np.arange(N)
    # pass 1
    check_close(lse[:, rows].T, oracle.lse_rows(inp.q, inp.k, rows), LSE_ATOL, "lse")
    if block_q == 1:
        oi, ol, _ = oracle.topk_rows(inp.q, inp.k, budget, rows)
        P = oracle.mass_rows(inp.q, inp.k, rows)
        ndiff = check_support(gi[rows], gl[rows], gm[rows], oi, ol, P, MASS_ATOL, "per-query")
        # pass 3 alone: the oracle on the GPU's own support
        ref, _ = oracle.attn_rows(inp.q, inp.k, inp.v, rows, sup=gi[rows], sup_len=gl[rows])
        check_close(out[rows], ref, OUT_ATOL[dtype], "sparse output")
        # end to end: the oracle's output on its own support (differs from the line above
        # only on rows whose supports differ at near-ties)
        ref_e2e, _ = oracle.attn_rows(inp.q, inp.k, inp.v, rows, sup=oi, sup_len=ol)
        check_close(out[rows], ref_e2e, OUT_ATOL[dtype], "end-to-end sparse output")
    else:
        nb = -(-N // block_q)
        if blocks is None:
            blocks = np.arange(nb)
        oi, ol, _ = oracle.block_topk(inp.q, inp.k, block_q, budget, blocks)
        M = oracle.block_mass(inp.q, inp.k, block_q, blocks)
        ndiff = check_support(gi[blocks], gl[blocks], gm[blocks], oi, ol, M,
                              MASS_ATOL * block_q, "block")
        # query rows of the listed blocks, each with its block's GPU support
        r, s, sl = oracle.block_rows_support(gi[blocks], gl[blocks], block_q, N, blocks)
        ref, _ = oracle.attn_rows(inp.q, inp.k, inp.v, r, sup=s, sup_len=sl)
        check_close(out[r], ref, OUT_ATOL[dtype], "block sparse output")
        r2, s2, sl2 = oracle.block_rows_support(oi, ol, block_q, N, blocks)
        ref_e2e, _ = oracle.attn_rows(inp.q, inp.k, inp.v, r2, sup=s2, sup_len=sl2)
        check_close(out[r2], ref_e2e, OUT_ATOL[dtype], "end-to-end block sparse output")
    return ndiff


SMALL = [
    # N, Hq, Hkv, d, dtype, k, block_q
    (1, 4, 1, 64, "f32", 1, 1),
    (2, 4, 1, 64, "bf16", 1, 1),
    (63, 1, 1, 64, "bf16", 2, 1),
    (65, 4, 1, 64, "f32", 31, 1),
    (129, 8, 2, 128, "bf16", 32, 1),
    (300, 32, 8, 128, "bf16", 40, 1),
    (512, 4, 1, 64, "f32", 32, 1),
    (1000, 32, 8, 128, "bf16", 64, 1),
    (127, 4, 1, 128, "bf16", 200, 1),          # k > N: full causal support
    (129, 8, 2, 128, "bf16", 16, 64),
    (300, 32, 8, 128, "bf16", 40, 64),
    (1000, 16, 4, 128, "bf16", 128, 128),
    (200, 4, 1, 64, "f32", 8, 1),
    (200, 4, 1, 64, "f32", 24, 16),
]


@pytest.mark.parametrize("N,Hq,Hkv,d,dtype,kb,bq", SMALL)
def test_mass_oracle_small(tam_lib, oracle_mod, N, Hq, Hkv, d, dtype, kb, bq):
    inp = _inputs(N, Hq, Hkv, d, dtype, seed=N, sink=True)
    run_mass_case(tam_lib, oracle_mod, inp, kb, bq, dtype=dtype)


def test_tiny_fp32_workload(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["tiny_fp32"]
    inp = tam_synth.make_inputs(w)
    run_mass_case(tam_lib, oracle_mod, inp, w.budget_k, 1, dtype="f32")


def test_gqa4k_needles_workload(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["gqa4k_needles"]
    inp = tam_synth.make_inputs(w)
    rows = tam_synth.sample_rows(w.N, inp.needle_i, n_random=128)
    run_mass_case(tam_lib, oracle_mod, inp, w.budget_k, 1, rows=rows)


@pytest.mark.slow
def test_gqa32k_workload_per_query(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["gqa32k_2pct"]
    inp = tam_synth.make_inputs(w)
    rows = tam_synth.sample_rows(w.N, inp.needle_i, n_random=256)
    run_mass_case(tam_lib, oracle_mod, inp, w.budget_k, 1, rows=rows)


@pytest.mark.slow
def test_gqa32k_workload_block_shared(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["gqa32k_2pct"]
    inp = tam_synth.make_inputs(w)
    nb = -(-w.N // 64)
    blocks = tam_synth.sample_blocks(nb, 16)
    run_mass_case(tam_lib, oracle_mod, inp, w.budget_k, 64, blocks=blocks)


@pytest.mark.parametrize("N", [4096, 16384])
def test_longctx_workload(tam_lib, oracle_mod, N):
    w = tam_synth.WORKLOADS[f"longctx_{N}"]
    inp = tam_synth.make_inputs(w)
    nb = -(-N // w.block_q[0])
    blocks = tam_synth.sample_blocks(nb, 6)
    run_mass_case(tam_lib, oracle_mod, inp, w.budget_k, w.block_q[0], blocks=blocks)


def test_zero_queries_tie_rule(tam_lib, oracle_mod):
    """Q = 0 makes every key of a row tie; the tie rule keeps the smallest indices."""
    inp = _inputs(300, 8, 2, 128, "bf16", seed=3)
    inp.q.zero_()
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    res = tam_lib.mass_oracle_prefill(q, k, v, 20, 1)
    gi, gl = res.idx.cpu().numpy(), res.length.cpu().numpy()
    for i in range(300):
        n = min(20, i + 1)
        assert gl[i] == n and list(gi[i, :n]) == list(range(n))
    mean_v = torch.stack([inp.v[:min(20, i + 1)].float().mean(0) for i in range(300)])  # [N,Hkv,d]
    ref = mean_v.repeat_interleave(4, dim=1)
    check_close(res.out.float().cpu(), ref, OUT_ATOL["bf16"], "zero-q output")


def test_full_budget_equals_dense(tam_lib, oracle_mod):
    inp = _inputs(257, 8, 2, 128, "bf16", seed=5)
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    res = tam_lib.mass_oracle_prefill(q, k, v, 300, 1)
    dense = tam_lib.dense_gqa_prefill(q, k, v)
    check_close(res.out.float().cpu(), dense.float().cpu(), OUT_ATOL["bf16"], "k>=N vs dense")


@pytest.mark.parametrize("N,Hq,Hkv,d,dtype", [(1, 4, 1, 64, "f32"), (200, 4, 1, 64, "f32"),
                                              (333, 32, 8, 128, "bf16"), (1000, 16, 4, 64, "bf16")])
def test_dense_prefill(tam_lib, oracle_mod, N, Hq, Hkv, d, dtype):
    inp = _inputs(N, Hq, Hkv, d, dtype, seed=7)
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    out, lse = tam_lib.dense_gqa_prefill(q, k, v, return_lse=True)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v)
    check_close(out.float().cpu(), ref, OUT_ATOL[dtype], "dense")
    check_close(lse.cpu().numpy().T, rl, LSE_ATOL, "dense lse")


@pytest.mark.parametrize("N,Hq,Hkv,d,kb,bq", [(500, 32, 8, 128, 64, 1), (700, 16, 4, 128, 100, 64),
                                              (130, 4, 1, 64, 7, 1)])
def test_sparse_attention_stress_support(tam_lib, oracle_mod, N, Hq, Hkv, d, kb, bq):
    """Pass 3 alone on a uniform-random support (the random-init stress row)."""
    inp = _inputs(N, Hq, Hkv, d, "bf16", seed=9)
    n_sel = N if bq == 1 else -(-N // bq)
    rows_last = np.arange(n_sel) if bq == 1 else np.minimum(N - 1, (np.arange(n_sel) + 1) * bq - 1)
    idx, ln = tam_synth.stress_support(N, kb, seed=1, rows=rows_last)
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    out, lse = tam_lib.sparse_support_attention(q, k, v, torch.from_numpy(idx).cuda(),
                                                torch.from_numpy(ln).cuda(), bq, return_lse=True)
    if bq == 1:
        rows, s, sl = np.arange(N), idx, ln
    else:
        rows, s, sl = oracle_mod.block_rows_support(idx, ln, bq, N)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v, rows, sup=s, sup_len=sl)
    check_close(out.float().cpu().numpy()[rows], ref, OUT_ATOL["bf16"], "stress sparse output")
    check_close(lse.cpu().numpy().T[rows], rl, LSE_ATOL, "stress sparse lse")


@pytest.mark.parametrize("N,dx,kb", [(1, 64, 4), (300, 64, 32), (1000, 64, 128), (517, 32, 600)])
def test_indexer_topk(tam_lib, oracle_mod, N, dx, kb):
    inp = _inputs(N, 8, 2, 128, "bf16", seed=11)
    qx, kx = tam_synth.indexer_projections(inp, dx, seed=2)
    res = tam_lib.indexer_topk(qx.cuda(), kx.cuda(), kb)
    oi, ol, _ = oracle_mod.indexer_topk_rows(qx, kx, kb)
    S = qx.double().numpy() @ kx.double().numpy().T
    # scores are exact in fp32 accumulation up to rounding; ranking tolerance as for mass
    check_support(res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy(),
                  oi, ol, S, 1e-3, "indexer")


def test_indexer_workload_rows(tam_lib, oracle_mod):
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w, N=8192)
    res = tam_lib.indexer_topk(inp.q_idx.cuda(), inp.k_idx.cuda(), w.budget_k)
    rows = tam_synth.sample_rows(8192, inp.needle_i, n_random=64)
    oi, ol, _ = oracle_mod.indexer_topk_rows(inp.q_idx, inp.k_idx, w.budget_k, rows)
    S = inp.q_idx.double().numpy()[rows] @ inp.k_idx.double().numpy().T
    check_support(res.idx.cpu().numpy()[rows], res.length.cpu().numpy()[rows],
                  res.value.cpu().numpy()[rows], oi, ol, S, 1e-3, "indexer32k")


@pytest.mark.parametrize("N,dx,kb,bq,dtype", [(300, 64, 32, 64, "bf16"), (1000, 64, 128, 64, "bf16"),
                                               (777, 128, 100, 128, "bf16"), (450, 64, 40, 16, "f32"),
                                               (129, 64, 200, 64, "bf16")])
def test_indexer_block_shared(tam_lib, oracle_mod, N, dx, kb, bq, dtype):
    """The fused, selection-block-shared indexer: block sums of each query's softmax of
    its indexer scores, top-k per block; then pass 3 on that support."""
    inp = _inputs(N, 8, 2, 128, dtype, seed=13 + N, sink=True, needles=3)
    qx, kx = tam_synth.indexer_projections(inp, dx, seed=2)
    if dtype == "f32":
        qx, kx = qx.float(), kx.float()
    # (the projections give scores with a standard deviation of about 4: a peaked but
    # not one-hot softmax over the prefix)
    res = tam_lib.indexer_topk(qx.cuda(), kx.cuda(), kb, bq)
    gi, gl, gm = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    oi, ol, _ = oracle_mod.indexer_block_topk(qx, kx, bq, kb)
    M = oracle_mod.indexer_block_mass(qx, kx, bq)
    check_support(gi, gl, gm, oi, ol, M, MASS_ATOL * bq, "indexer block")
    out = tam_lib.sparse_support_attention(*_cuda(inp.q, inp.k, inp.v), res.idx, res.length, bq)
    r, sup, sl = oracle_mod.block_rows_support(gi, gl, bq, N)
    ref, _ = oracle_mod.attn_rows(inp.q, inp.k, inp.v, r, sup=sup, sup_len=sl)
    check_close(out.float().cpu().numpy()[r], ref, OUT_ATOL[dtype], "indexer block output")


def test_indexer_block_shared_ties(tam_lib):
    """q_idx = 0: every query's softmax is uniform, so a block's sums fall with the key
    index and the support is the first keys."""
    N, kb, bq = 700, 30, 64
    inp = _inputs(N, 8, 2, 128, "bf16", seed=3)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    res = tam_lib.indexer_topk(torch.zeros_like(qx).cuda(), kx.cuda(), kb, bq)
    gi, gl = res.idx.cpu().numpy(), res.length.cpu().numpy()
    for b in range(len(gl)):
        n = min(kb, min(N, (b + 1) * bq))
        assert gl[b] == n and list(gi[b, :n]) == list(range(n)), b


@pytest.mark.parametrize("N,Hq,Hkv,d,dx", [(300, 32, 8, 128, 64), (1000, 16, 4, 128, 64),
                                          (777, 8, 2, 64, 128), (129, 16, 1, 128, 64)])
def test_distill_kl(tam_lib, oracle_mod, N, Hq, Hkv, d, dx):
    """KL(P_i || softmax of indexer scores) per query against the oracle."""
    inp = _inputs(N, Hq, Hkv, d, "bf16", seed=17 + N, sink=True, needles=3)
    qx, kx = tam_synth.indexer_projections(inp, dx, seed=2)
    q, k = _cuda(inp.q, inp.k)
    lse = tam_lib.attention_lse(q, k)
    kl = tam_lib.distill_kl(q, k, lse, qx.cuda(), kx.cuda()).cpu().numpy()
    check_close(kl, oracle_mod.distill_kl_rows(inp.q, inp.k, qx, kx), KL_ATOL, "distill kl")


def test_distill_kl_in_chunks(tam_lib):
    """The smallest workspace (more chunks) gives the same values."""
    N = 1500
    inp = _inputs(N, 32, 8, 128, "bf16", seed=5)
    qx, kx = tam_synth.indexer_projections(inp, 64, seed=2)
    q, k = _cuda(inp.q, inp.k)
    lse = tam_lib.attention_lse(q, k)
    ref = tam_lib.distill_kl(q, k, lse, qx.cuda(), kx.cuda())
    lo = tam_lib.lib().tam_distill_kl_workspace_min(N, 32, 8, 128, 0, 64)
    got = tam_lib.distill_kl(q, k, lse, qx.cuda(), kx.cuda(), workspace_bytes=lo)
    assert torch.equal(ref, got)


@pytest.mark.parametrize("N,Hq,Hkv,d,kmax,bq", [(1000, 32, 8, 128, 256, 1), (600, 16, 4, 128, 700, 1),
                                               (900, 32, 8, 128, 128, 64)])
def test_support_mass_curve(tam_lib, oracle_mod, N, Hq, Hkv, d, kmax, bq):
    """Budget sweep from one top-kmax pass 2: per row, the mass of the top-k for several k."""
    inp = _inputs(N, Hq, Hkv, d, "bf16", seed=23 + N, sink=True, needles=4)
    q, k = _cuda(inp.q, inp.k)
    lse = tam_lib.attention_lse(q, k)
    sup = tam_lib.mass_select(q, k, lse, kmax, bq)
    ks = [1, 16, kmax // 2, kmax, kmax + 50]
    curve = tam_lib.support_mass_curve(sup.value, sup.length, ks).cpu().numpy()
    if bq == 1:
        ref = oracle_mod.support_mass_curve(inp.q, inp.k, ks[:-1])
        check_close(curve[:, :-1], ref, 1e-3, "support mass curve")
    # a budget above kmax can only sum the whole top-kmax row
    assert np.array_equal(curve[:, -1], curve[:, -2])
    # and against the GPU's own top-k supports at each budget
    for t, kb in enumerate(ks[:-1]):
        s2 = tam_lib.mass_select(q, k, lse, kb, bq)
        check_close(curve[:, t], s2.value.sum(dim=1).cpu().numpy(), 1e-3 * bq, f"k={kb}")


def test_support_mass_curve_rejects(tam_lib):
    x = torch.zeros(4, 8, device="cuda")
    ln = torch.full((4,), 8, dtype=torch.int32, device="cuda")
    with pytest.raises(tam_lib.TamError):
        tam_lib.support_mass_curve(x, ln, [0])
    with pytest.raises(tam_lib.TamError):
        tam_lib.support_mass_curve(x, ln, list(range(1, 18)))


def test_run_twice_bitwise_identical(tam_lib):
    inp = _inputs(700, 32, 8, 128, "bf16", seed=13, sink=True)
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    a = tam_lib.mass_oracle_prefill(q, k, v, 50, 1)
    b = tam_lib.mass_oracle_prefill(q, k, v, 50, 1)
    assert torch.equal(a.idx, b.idx) and torch.equal(a.value, b.value)
    assert torch.equal(a.out, b.out) and torch.equal(a.lse, b.lse)
    c = tam_lib.mass_oracle_prefill(q, k, v, 50, 64)
    e = tam_lib.mass_oracle_prefill(q, k, v, 50, 64)
    assert torch.equal(c.idx, e.idx) and torch.equal(c.value, e.value) and torch.equal(c.out, e.out)


def test_host_buffers_round_trip(tam_lib):
    """CPU (pinned) inputs: the binding copies in, runs on the GPU, copies results out."""
    inp = _inputs(256, 8, 2, 128, "bf16", seed=17)
    q, k, v = inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()
    r_host = tam_lib.mass_oracle_prefill(q, k, v, 16, 1)
    r_dev = tam_lib.mass_oracle_prefill(q.cuda(), k.cuda(), v.cuda(), 16, 1)
    assert not r_host.idx.is_cuda
    assert torch.equal(r_host.idx, r_dev.idx.cpu()) and torch.equal(r_host.out, r_dev.out.cpu())


def test_workspace_too_small_is_rejected(tam_lib):
    inp = _inputs(64, 4, 1, 64, "bf16")
    q, k, v = _cuda(inp.q, inp.k, inp.v)
    L = tam_lib.lib()
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    idx = torch.empty(64, 8, dtype=torch.int32, device="cuda")
    ln = torch.empty(64, dtype=torch.int32, device="cuda")
    ms = torch.empty(64, 8, dtype=torch.float32, device="cuda")
    rc = L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, q.data_ptr(), k.data_ptr(), v.data_ptr(), 8, 1,
                                   idx.data_ptr(), ln.data_ptr(), ms.data_ptr(), None, None,
                                   ws.data_ptr(), 16, None)
    assert rc == tam_lib.TAM_ERR_WORKSPACE
