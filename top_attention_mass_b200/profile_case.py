"""Run one row of the hot path a few times on a seeded input, for ncu captures.

    python -m top_attention_mass_b200.profile_case --row pass1_lse --N 16384 [--reps 3]

Rows: pass1_lse, pass2_mass_topk, pass2_block_mass_topk, pass3_gather, pass3_block,
indexer_topk, dense_prefill.  Shapes are those of the 32K workload (Hq=32, Hkv=8,
d=128, bf16, k=655, B_q=64, indexer d_idx=64 / k=1024) at the given N, so that a
capture fits the profiler's size rules while the kernels are the benchmarked ones;
`--head-dim 256` takes a Hq 16 / Hkv 8, d 256 layer instead.
pass3_gather_stress is the benchmark's out-of-L2 gather: per-query pass 3 on
device-drawn inputs of the same head shape with a random support of k = 2048 (one
uniform key per stratum of [0, i]); at N = 262144 its K/V halves are 537 MB each.
`--row all` runs every row once, in the benchmark's order, after one untimed round, and
prints the library's kernel-launch count of each row in the last round as JSON, so that
a one-pass capture of the whole sequence can be split by row.
Every launch is checked through the library's status block.
"""
import argparse
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import tam_synth  # noqa: E402
import top_attention_mass_b200 as tam  # noqa: E402

ROWS = ("pass1_lse", "pass2_mass_topk", "pass2_block_mass_topk", "pass3_gather", "pass3_block",
        "indexer_topk", "dense_prefill", "pass3_gather_stress", "all")
# the benchmark's order of the rows of the hot path
ALL_ORDER = ("pass1_lse", "pass2_mass_topk", "pass3_gather", "pass2_block_mass_topk", "pass3_block",
             "indexer_topk", "pass3_indexer_support", "dense_prefill")


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
    ap.add_argument("--head-dim", type=int, default=128, choices=(128, 256),
                    help="256: a Hq 16 / Hkv 8, d 256 layer (same bytes per token)")
    a = ap.parse_args()
    if a.row == "pass3_gather_stress":
        gather_stress(a.N, a.reps)
        print(f"profile_case {a.row} N={a.N} reps={a.reps} ok")
        return
    w = tam_synth.WORKLOADS["indexer32k"]
    if a.head_dim == 256:
        w = tam_synth.custom("hd256", a.N, 16, 8, 256, "bf16", 655, (1, 64), sink=True,
                             needles=64, d_idx=64)
    inp = tam_synth.make_inputs(w, N=a.N)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    qx, kx = inp.q_idx.cuda(), inp.k_idx.cuda()
    ws = tam.Workspace(q.device)
    box = {"lse": tam.attention_lse(q, k, workspace=ws)}

    def run(row):
        if row == "pass1_lse":
            box["lse"] = tam.attention_lse(q, k, workspace=ws)
        elif row == "pass2_mass_topk":
            box["s1"] = tam.mass_select(q, k, box["lse"], 655, 1, workspace=ws)
        elif row == "pass2_block_mass_topk":
            box["s2"] = tam.mass_select(q, k, box["lse"], 655, 64, workspace=ws)
        elif row == "pass3_gather":
            tam.sparse_support_attention(q, k, v, box["s1"].idx, box["s1"].length, 1, workspace=ws)
        elif row == "pass3_block":
            tam.sparse_support_attention(q, k, v, box["s2"].idx, box["s2"].length, 64, workspace=ws)
        elif row == "indexer_topk":
            box["s3"] = tam.indexer_topk(qx, kx, 1024, workspace=ws)
        elif row == "pass3_indexer_support":
            tam.sparse_support_attention(q, k, v, box["s3"].idx, box["s3"].length, 1, workspace=ws)
        else:
            tam.dense_gqa_prefill(q, k, v, workspace=ws)

    if a.row == "all":
        for row in ALL_ORDER:
            run(row)
        counts = {}
        for _ in range(a.reps):
            for row in ALL_ORDER:
                n0 = tam.kernel_launches()
                run(row)
                counts[row] = tam.kernel_launches() - n0
        torch.cuda.synchronize()
        print(json.dumps({"launches_per_row": counts}))
    else:
        # supports only for the pass-3 rows, so the first launches of a pass-2 kernel are
        # the row's own
        if a.row == "pass3_gather":
            run("pass2_mass_topk")
        if a.row == "pass3_block":
            run("pass2_block_mass_topk")
        for _ in range(a.reps):
            run(a.row)
    torch.cuda.synchronize()
    print(f"profile_case {a.row} N={a.N} reps={a.reps} ok")


if __name__ == "__main__":
    main()
