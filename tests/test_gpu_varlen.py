"""Packed batches and head dim 256 on the CUDA path vs the fp64 oracle.

A packed batch runs every sequence as its own causal problem; each sequence is
checked against the oracle on its slice (support, mass, lse) and the whole
batch's outputs against the oracle on the GPU's support.  The varlen call must
also reproduce, bit for bit, the single-sequence call on each slice.
"""
import numpy as np
import pytest
import torch

import tam_synth
from parity_util import LSE_ATOL, MASS_ATOL, OUT_ATOL, check_close, check_support

pytestmark = pytest.mark.gpu


def _inputs(N, Hq, Hkv, d, dtype="bf16", seed=0, **kw):
    w = tam_synth.custom("p", N, Hq, Hkv, d, dtype=dtype, seed=seed, **kw)
    return tam_synth.make_inputs(w)


VARLEN = [
    # cu_seqlens, Hq, Hkv, d, dtype, k, block_q
    ([0, 1, 130, 130, 393, 457, 1000], 8, 2, 128, "bf16", 32, 1),
    ([0, 1, 130, 130, 393, 457, 1000], 8, 2, 128, "bf16", 16, 64),
    ([0, 300, 363, 700], 32, 8, 128, "bf16", 40, 64),
    ([0, 640, 1160], 16, 4, 64, "bf16", 100, 1),
    ([0, 77, 300, 301], 4, 1, 64, "f32", 8, 1),
    ([0, 77, 300, 301], 4, 1, 64, "f32", 8, 16),
    ([0, 150, 170, 300], 8, 2, 256, "bf16", 16, 1),
]


def _per_sequence_checks(tam, oracle, inp, cu, res, kb, bq, Hq):
    gi, gl, gm = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    lse = res.lse.cpu().numpy()
    sel = tam.selection_offsets(cu, bq).numpy()
    assert gi.shape[0] == sel[-1]
    for s, (t0, t1) in enumerate(oracle.seq_slices(cu)):
        if t1 == t0:
            assert sel[s + 1] == sel[s]
            continue
        qs, ks = inp.q[t0:t1], inp.k[t0:t1]
        r0, r1 = sel[s], sel[s + 1]
        check_close(lse[Hq * t0:Hq * t1].reshape(Hq, t1 - t0).T, oracle.lse_rows(qs, ks),
                    LSE_ATOL, f"lse seq {s}")
        if bq == 1:
            oi, ol, _ = oracle.topk_rows(qs, ks, kb)
            P = oracle.mass_rows(qs, ks)
        else:
            oi, ol, _ = oracle.block_topk(qs, ks, bq, kb)
            P = oracle.block_mass(qs, ks, bq)
        check_support(gi[r0:r1], gl[r0:r1], gm[r0:r1], oi, ol, P, MASS_ATOL * bq, f"seq {s}")
    return gi, gl


@pytest.mark.parametrize("cu,Hq,Hkv,d,dtype,kb,bq", VARLEN)
def test_mass_oracle_varlen(tam_lib, oracle_mod, cu, Hq, Hkv, d, dtype, kb, bq):
    inp = _inputs(cu[-1], Hq, Hkv, d, dtype, seed=len(cu) + cu[-1], sink=True)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    res = tam_lib.mass_oracle_prefill_varlen(q, k, v, cu, kb, bq)
    torch.cuda.synchronize()
    gi, gl = _per_sequence_checks(tam_lib, oracle_mod, inp, cu, res, kb, bq, Hq)
    ref, _ = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu, sup=gi, sup_len=gl, block_q=bq)
    check_close(res.out.float().cpu().numpy(), ref, OUT_ATOL[dtype], "varlen sparse output")


def test_varlen_equals_single_sequence_calls(tam_lib):
    cu = [0, 1, 130, 130, 393, 457, 1000]
    inp = _inputs(cu[-1], 8, 2, 128, "bf16", seed=3)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    for bq in (1, 64):
        res = tam_lib.mass_oracle_prefill_varlen(q, k, v, cu, 24, bq)
        sel = tam_lib.selection_offsets(cu, bq)
        for s in range(len(cu) - 1):
            t0, t1 = cu[s], cu[s + 1]
            if t1 == t0:
                continue
            one = tam_lib.mass_oracle_prefill(q[t0:t1], k[t0:t1], v[t0:t1], 24, bq)
            r0, r1 = int(sel[s]), int(sel[s + 1])
            assert torch.equal(one.idx, res.idx[r0:r1]) and torch.equal(one.length, res.length[r0:r1])
            assert torch.equal(one.value, res.value[r0:r1])
            assert torch.equal(one.out, res.out[t0:t1])
            assert torch.equal(one.lse, tam_lib.lse_block(res.lse, cu, s))


@pytest.mark.parametrize("cu,Hq,Hkv,d,dtype", [([0, 1, 130, 130, 393, 1000], 16, 4, 128, "bf16"),
                                               ([0, 200, 201, 450], 4, 1, 64, "f32"),
                                               ([0, 90, 300], 8, 2, 256, "bf16")])
def test_dense_varlen(tam_lib, oracle_mod, cu, Hq, Hkv, d, dtype):
    inp = _inputs(cu[-1], Hq, Hkv, d, dtype, seed=cu[-1])
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    out, lse = tam_lib.dense_gqa_prefill_varlen(q, k, v, cu, return_lse=True)
    ref, rl = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu)
    check_close(out.float().cpu().numpy(), ref, OUT_ATOL[dtype], "dense varlen")
    for s in range(len(cu) - 1):
        if cu[s + 1] > cu[s]:
            check_close(tam_lib.lse_block(lse, cu, s).cpu().numpy().T, rl[cu[s]:cu[s + 1]],
                        LSE_ATOL, f"dense varlen lse seq {s}")


def test_varlen_rejects_bad_offsets(tam_lib):
    inp = _inputs(64, 4, 1, 64, "bf16")
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    for cu in ([1, 64], [0, 40, 30, 64]):
        with pytest.raises(tam_lib.TamError):
            tam_lib.mass_oracle_prefill_varlen(q, k, v, cu, 8)
        with pytest.raises(tam_lib.TamError):
            tam_lib.dense_gqa_prefill_varlen(q, k, v, cu)
    with pytest.raises(ValueError):
        tam_lib.mass_oracle_prefill_varlen(q, k, v, [0, 63], 8)      # does not cover the tokens


@pytest.mark.parametrize("cu,dx,kb,bq", [([0, 1, 130, 130, 393, 457, 1000], 64, 32, 1),
                                         ([0, 1, 130, 130, 393, 457, 1000], 64, 24, 64),
                                         ([0, 300, 301, 700], 32, 16, 1)])
def test_indexer_varlen(tam_lib, oracle_mod, cu, dx, kb, bq):
    """Indexer support over a packed batch: each sequence against the oracle on its
    slice and bit for bit against the single-sequence call; then pass 3 on it."""
    inp = _inputs(cu[-1], 8, 2, 128, "bf16", seed=cu[-1] + bq, sink=True)
    qx, kx = tam_synth.indexer_projections(inp, dx, seed=2)
    res = tam_lib.indexer_topk_varlen(qx.cuda(), kx.cuda(), cu, kb, bq)
    gi, gl, gv = res.idx.cpu().numpy(), res.length.cpu().numpy(), res.value.cpu().numpy()
    sel = tam_lib.selection_offsets(cu, bq).numpy()
    assert gi.shape[0] == sel[-1]
    for s in range(len(cu) - 1):
        t0, t1 = cu[s], cu[s + 1]
        if t1 == t0:
            continue
        r0, r1 = sel[s], sel[s + 1]
        one = tam_lib.indexer_topk(qx[t0:t1].cuda(), kx[t0:t1].cuda(), kb, bq)
        assert torch.equal(one.idx.cpu(), res.idx[r0:r1].cpu())
        assert torch.equal(one.value.cpu(), res.value[r0:r1].cpu())
        if bq == 1:
            oi, ol, _ = oracle_mod.indexer_topk_rows(qx[t0:t1], kx[t0:t1], kb)
            S = qx[t0:t1].double().numpy() @ kx[t0:t1].double().numpy().T
            check_support(gi[r0:r1], gl[r0:r1], gv[r0:r1], oi, ol, S, 1e-3, f"indexer seq {s}")
        else:
            oi, ol, _ = oracle_mod.indexer_block_topk(qx[t0:t1], kx[t0:t1], bq, kb)
            M = oracle_mod.indexer_block_mass(qx[t0:t1], kx[t0:t1], bq)
            check_support(gi[r0:r1], gl[r0:r1], gv[r0:r1], oi, ol, M, MASS_ATOL * bq,
                          f"indexer block seq {s}")
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    out = tam_lib.sparse_support_attention_varlen(q, k, v, res.idx, res.length, cu, bq)
    ref, _ = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu, sup=gi, sup_len=gl, block_q=bq)
    check_close(out.float().cpu().numpy(), ref, OUT_ATOL["bf16"], "varlen pass 3 on indexer")
    for s in range(len(cu) - 1):
        t0, t1 = cu[s], cu[s + 1]
        if t1 > t0:
            # (copies: a slice of the lengths need not start on a 16-byte boundary)
            one = tam_lib.sparse_support_attention(q[t0:t1], k[t0:t1], v[t0:t1],
                                                   res.idx[sel[s]:sel[s + 1]].clone(),
                                                   res.length[sel[s]:sel[s + 1]].clone(), bq)
            assert torch.equal(one, out[t0:t1])


# ---------------------------------------------------------------- head dim 256

@pytest.mark.parametrize("N,Hq,Hkv,dtype,kb,bq", [(200, 4, 1, "f32", 8, 1),
                                                   (150, 8, 2, "bf16", 16, 1),
                                                   (150, 8, 2, "bf16", 16, 32)])
def test_head_dim_256(tam_lib, oracle_mod, N, Hq, Hkv, dtype, kb, bq):
    inp = _inputs(N, Hq, Hkv, 256, dtype, seed=N + bq, sink=True)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    res = tam_lib.mass_oracle_prefill(q, k, v, kb, bq)
    torch.cuda.synchronize()
    cu = [0, N]
    gi, gl = _per_sequence_checks(tam_lib, oracle_mod, inp, cu, _flat_lse(res), kb, bq, Hq)
    ref, _ = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu, sup=gi, sup_len=gl, block_q=bq)
    check_close(res.out.float().cpu().numpy(), ref, OUT_ATOL[dtype], "d=256 sparse output")
    dense = tam_lib.dense_gqa_prefill(q, k, v)
    dref, _ = oracle_mod.attn_rows(inp.q, inp.k, inp.v)
    check_close(dense.float().cpu().numpy(), dref, OUT_ATOL[dtype], "d=256 dense")


@pytest.mark.parametrize("N,Hq,Hkv,kb,bq", [(700, 8, 2, 40, 1), (300, 4, 4, 17, 1),
                                             (1000, 16, 1, 64, 1), (520, 16, 4, 33, 64),
                                             (1000, 16, 1, 64, 128), (389, 8, 8, 20, 16)])
def test_head_dim_256_tensor_cores(tam_lib, oracle_mod, N, Hq, Hkv, kb, bq):
    """bf16 at d = 256 on the tensor-core kernels (pass 1, the single-CTA pass 2 with
    the streamed selection or the block sums, the 256-wide gather or the block-shared
    tcgen05 pass 3): several tiles with a ragged tail, every head ratio shape."""
    inp = _inputs(N, Hq, Hkv, 256, "bf16", seed=N + Hq + bq, sink=True, needles=2)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    res = tam_lib.mass_oracle_prefill(q, k, v, kb, bq)
    torch.cuda.synchronize()
    cu = [0, N]
    gi, gl = _per_sequence_checks(tam_lib, oracle_mod, inp, cu, _flat_lse(res), kb, bq, Hq)
    ref, _ = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu, sup=gi, sup_len=gl, block_q=bq)
    check_close(res.out.float().cpu().numpy(), ref, OUT_ATOL["bf16"], "d=256 sparse output")


@pytest.mark.parametrize("N,Hq,Hkv", [(1, 4, 1), (777, 16, 2), (300, 32, 2), (129, 8, 8)])
def test_dense_head_dim_256_tensor_cores(tam_lib, oracle_mod, N, Hq, Hkv):
    inp = _inputs(N, Hq, Hkv, 256, "bf16", seed=N + 5, sink=True)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    out, lse = tam_lib.dense_gqa_prefill(q, k, v, return_lse=True)
    ref, rl = oracle_mod.attn_rows(inp.q, inp.k, inp.v)
    check_close(out.float().cpu().numpy(), ref, OUT_ATOL["bf16"], "d=256 dense")
    check_close(lse.cpu().numpy().T, rl, LSE_ATOL, "d=256 dense lse")


# ---------------------------------------------------------------- one launch per batch

def _ragged_cu(n_seq, max_len, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, max_len + 1, size=n_seq)
    lens[rng.integers(0, n_seq)] = max_len            # one full-length sequence
    return [0] + np.cumsum(lens).tolist()


@pytest.mark.parametrize("n_seq,max_len,d", [(8, 700, 128), (300, 40, 128), (140, 90, 64)])
def test_dense_varlen_one_launch_per_table(tam_lib, n_seq, max_len, d):
    """The packed dense call is one launch per table of up to 128 sequences, and every
    sequence's rows equal the single-sequence call on its slice bit for bit."""
    cu = _ragged_cu(n_seq, max_len, seed=n_seq)
    inp = _inputs(cu[-1], 16, 4, d, "bf16", seed=n_seq + 1)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    n0 = tam_lib.kernel_launches()
    out, lse = tam_lib.dense_gqa_prefill_varlen(q, k, v, cu, return_lse=True)
    torch.cuda.synchronize()
    assert tam_lib.kernel_launches() - n0 == (n_seq + 127) // 128
    for s in range(n_seq):
        t0, t1 = cu[s], cu[s + 1]
        if t1 == t0:
            continue
        one, ol = tam_lib.dense_gqa_prefill(q[t0:t1], k[t0:t1], v[t0:t1], return_lse=True)
        assert torch.equal(one, out[t0:t1]), s
        assert torch.equal(ol, tam_lib.lse_block(lse, cu, s)), s


def test_mass_oracle_varlen_many_sequences(tam_lib, oracle_mod):
    """A batch of 300 short sequences (three tables): pass 1 and pass 3 as one launch per
    table, and every sequence bit for bit equal to the single-sequence call."""
    cu = _ragged_cu(300, 48, seed=7)
    inp = _inputs(cu[-1], 8, 2, 128, "bf16", seed=11, sink=True)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    res = tam_lib.mass_oracle_prefill_varlen(q, k, v, cu, 12, 1)
    torch.cuda.synchronize()
    for s in range(0, 300, 7):
        t0, t1 = cu[s], cu[s + 1]
        if t1 == t0:
            continue
        one = tam_lib.mass_oracle_prefill(q[t0:t1], k[t0:t1], v[t0:t1], 12, 1)
        assert torch.equal(one.idx, res.idx[t0:t1]) and torch.equal(one.length, res.length[t0:t1])
        assert torch.equal(one.value, res.value[t0:t1])
        assert torch.equal(one.out, res.out[t0:t1])
        assert torch.equal(one.lse, tam_lib.lse_block(res.lse, cu, s))
    gi, gl = res.idx.cpu().numpy(), res.length.cpu().numpy()
    ref, _ = oracle_mod.varlen_attn(inp.q, inp.k, inp.v, cu, sup=gi, sup_len=gl, block_q=1)
    check_close(res.out.float().cpu().numpy(), ref, OUT_ATOL["bf16"], "varlen 300 sequences")


def _flat_lse(res):
    """A single sequence's [Hq, N] lse is its own packed block."""
    return type(res)(res.idx, res.length, res.value, res.lse.reshape(-1), res.out)
