"""Run one row of the hot path a few times on a seeded input, for ncu captures.

    python -m top_attention_mass_b200.profile_case --row pass1_lse --N 16384 [--reps 3]

Rows: pass1_lse, pass2_mass_topk, pass2_block_mass_topk, pass3_gather, pass3_block,
indexer_topk, dense_prefill.  Shapes are those of the 32K workload (Hq=32, Hkv=8,
d=128, bf16, k=655, B_q=64, indexer d_idx=64 / k=1024) at the given N, so that a
capture fits the profiler's size rules while the kernels are the benchmarked ones.
pass3_gather_stress is the benchmark's out-of-L2 gather: per-query pass 3 on
device-drawn inputs of the same head shape with a random support of k = 2048 (one
uniform key per stratum of [0, i]); at N = 262144 its K/V halves are 537 MB each.
Every launch is checked through the library's status block.
"""
import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import tam_synth  # noqa: E402
import top_attention_mass_b200 as tam  # noqa: E402

ROWS = ("pass1_lse", "pass2_mass_topk", "pass2_block_mass_topk", "pass3_gather", "pass3_block",
        "indexer_topk", "dense_prefill", "pass3_gather_stress")


def gather_stress(N, reps):
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    q = torch.randn(N, 32, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(N, 8, 128, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(N, 8, 128, generator=g, device="cuda").to(torch.bfloat16)
    idx, ln = tam_synth.stratified_support(N, 2048, seed=9, device="cuda")
    for _ in range(reps):
        tam.sparse_support_attention(q, k, v, idx, ln, 1)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--row", choices=ROWS, required=True)
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    if a.row == "pass3_gather_stress":
        gather_stress(a.N, a.reps)
        print(f"profile_case {a.row} N={a.N} reps={a.reps} ok")
        return
    w = tam_synth.WORKLOADS["indexer32k"]
    inp = tam_synth.make_inputs(w, N=a.N)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    qx, kx = inp.q_idx.cuda(), inp.k_idx.cuda()
    lse = tam.attention_lse(q, k)
    # supports only for the pass-3 rows, so the first launches of a pass-2 kernel are the
    # row's own
    s1 = tam.mass_select(q, k, lse, 655, 1) if a.row == "pass3_gather" else None
    s2 = tam.mass_select(q, k, lse, 655, 64) if a.row == "pass3_block" else None
    for _ in range(a.reps):
        if a.row == "pass1_lse":
            tam.attention_lse(q, k)
        elif a.row == "pass2_mass_topk":
            tam.mass_select(q, k, lse, 655, 1)
        elif a.row == "pass2_block_mass_topk":
            tam.mass_select(q, k, lse, 655, 64)
        elif a.row == "pass3_gather":
            tam.sparse_support_attention(q, k, v, s1.idx, s1.length, 1)
        elif a.row == "pass3_block":
            tam.sparse_support_attention(q, k, v, s2.idx, s2.length, 64)
        elif a.row == "indexer_topk":
            tam.indexer_topk(qx, kx, 1024)
        else:
            tam.dense_gqa_prefill(q, k, v)
    torch.cuda.synchronize()
    print(f"profile_case {a.row} N={a.N} reps={a.reps} ok")


if __name__ == "__main__":
    main()
