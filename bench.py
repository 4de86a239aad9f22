#!/usr/bin/env python
"""Benchmark of the attention-mass top-k path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of every step of the hot path over one layer of the 32K
workload (N=32768, Hq=32, Hkv=8, d=128, bf16; sink at token 0, 64 planted
needles):
  pass 1  per-head LSE                            (attention_lse)
  pass 2  mass + per-query top-k, k=655           (mass_select, block_q=1)
  pass 3  per-query gathered sparse attention     (sparse_support_attention)
  pass 2  mass + block-shared top-k, B_q=64       (mass_select, block_q=64)
  pass 3  block-shared sparse attention           (sparse_support_attention)
  indexer top-k, d_idx=64, k=1024                 (indexer_topk)
  pass 3  on the indexer support                  (sparse_support_attention)
  dense causal GQA prefill (comparator)           (dense_gqa_prefill)
value = query tokens of all ranks / step time (max over ranks).  With N > 1 GPUs
every rank runs an independent replica of the workload (weak scaling, no
collective on the data path).  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import tam_synth  # noqa: E402

METRIC = "query-tokens/s per GQA layer (mass-oracle, sparse pass) at 32K; % of roofline"
UNIT = "q-tok/s"
WORKLOAD = "gqa32k_2pct"
BLOCK_Q = 64
INDEXER_K = 1024
D_IDX = 64
# packed batch of mixed lengths (sums to the 32K workload's token count)
VARLEN_SEQS = (8192, 4096, 2048, 6144, 1024, 3072, 5120, 3072)
VARLEN_K = 256
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def causal_pairs(N: int) -> int:
    return N * (N + 1) // 2


def support_pairs(N: int, k: int) -> int:
    i = np.arange(N, dtype=np.int64)
    return int(np.minimum(k, i + 1).sum())


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            target = str(self.device)
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", target, f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1].split()[0]))
                    smax.append(float(parts[2].split()[0]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ the device step

ROWS_ALL = ("pass1_lse", "pass2_mass_topk", "pass3_gather", "pass2_block_mass_topk",
            "pass3_block", "indexer_topk", "pass3_indexer_support", "dense_prefill")


def rows_of(w) -> tuple:
    """Rows of the hot path a workload exercises (the 32K default runs all of them)."""
    rows = ["pass1_lse"]
    if 1 in w.block_q:
        rows += ["pass2_mass_topk", "pass3_gather"]
    if any(b > 1 for b in w.block_q):
        rows += ["pass2_block_mass_topk", "pass3_block"]
    if w.d_idx:
        rows += ["indexer_topk", "pass3_indexer_support"]
    rows.append("dense_prefill")
    return tuple(rows)


class Step:
    """The workload's rows of the hot path on device-resident inputs; CUDA events between
    calls (events[i] .. events[i+1] brackets row i)."""

    def __init__(self, tam, w, q, k, v, qx=None, kx=None):
        self.tam, self.w = tam, w
        self.q, self.k, self.v, self.qx, self.kx = q, k, v, qx, kx
        self.rows = rows_of(w)
        self.block_q = max(w.block_q)
        self.ws = tam.Workspace(q.device)
        self.outputs = {}

    def run(self, events=None):
        t, w, ws = self.tam, self.w, self.ws
        ev = events or [None] * (len(self.rows) + 1)
        out = {}
        lse = None
        for n, row in enumerate(self.rows):
            if ev[n] is not None:
                ev[n].record()
            if row == "pass1_lse":
                lse = out["lse"] = t.attention_lse(self.q, self.k, workspace=ws, check=False)
            elif row == "pass2_mass_topk":
                s = t.mass_select(self.q, self.k, lse, w.budget_k, 1, workspace=ws, check=False)
                out.update(s1_idx=s.idx, s1_len=s.length, s1_mass=s.value)
            elif row == "pass3_gather":
                out["o1"] = t.sparse_support_attention(self.q, self.k, self.v, out["s1_idx"],
                                                       out["s1_len"], 1, workspace=ws, check=False)
            elif row == "pass2_block_mass_topk":
                s = t.mass_select(self.q, self.k, lse, w.budget_k, self.block_q, workspace=ws,
                                  check=False)
                out.update(s2_idx=s.idx, s2_len=s.length, s2_mass=s.value)
            elif row == "pass3_block":
                out["o2"] = t.sparse_support_attention(self.q, self.k, self.v, out["s2_idx"],
                                                       out["s2_len"], self.block_q, workspace=ws,
                                                       check=False)
            elif row == "indexer_topk":
                s = t.indexer_topk(self.qx, self.kx, self.indexer_k, workspace=ws, check=False)
                out.update(s3_idx=s.idx, s3_len=s.length, s3_score=s.value)
            elif row == "pass3_indexer_support":
                out["o3"] = t.sparse_support_attention(self.q, self.k, self.v, out["s3_idx"],
                                                       out["s3_len"], 1, workspace=ws, check=False)
            elif row == "dense_prefill":
                out["od"] = t.dense_gqa_prefill(self.q, self.k, self.v, workspace=ws, check=False)
        if ev[len(self.rows)] is not None:
            ev[len(self.rows)].record()
        self.outputs = out
        return out

    @property
    def indexer_k(self):
        return INDEXER_K if self.w.name == WORKLOAD else self.w.budget_k


def algorithmic_work(step, N):
    """Per-row algorithmic flops/bytes (what the method must do, not what it avoids)."""
    w, outs = step.w, step.outputs
    Hq, Hkv, d = w.Hq, w.Hkv, w.d
    elt = 2
    cp = causal_pairs(N)
    qo = 2 * N * Hq * d * elt                         # read Q, write O
    gather = lambda pairs: pairs * Hkv * 2 * d * elt  # noqa: E731  K and V rows of every group
    work = {
        "pass1_lse": {"bound": "tensor", "flops": 2.0 * d * Hq * cp},
        "pass2_mass_topk": {"bound": "tensor", "flops": 2.0 * d * Hq * cp},
        "pass2_block_mass_topk": {"bound": "tensor", "flops": 2.0 * d * Hq * cp},
        "indexer_topk": {"bound": "tensor", "flops": 2.0 * (w.d_idx or D_IDX) * cp},
        "dense_prefill": {"bound": "tensor", "flops": 4.0 * d * Hq * cp},
    }
    if "pass3_gather" in step.rows:
        sp1 = support_pairs(N, w.budget_k)
        work["pass3_gather"] = {"bound": "hbm",
                                "bytes": float(gather(sp1) + qo + N * w.budget_k * 4 + N * 4)}
    if "pass3_indexer_support" in step.rows:
        kx = step.indexer_k
        sp3 = support_pairs(N, kx)
        work["pass3_indexer_support"] = {"bound": "hbm",
                                         "bytes": float(gather(sp3) + qo + N * kx * 4 + N * 4)}
    if "pass3_block" in step.rows:
        bq = step.block_q
        s2_len = outs["s2_len"].cpu().numpy().astype(np.int64)
        s2_idx = outs["s2_idx"].cpu().numpy()
        nb = len(s2_len)
        attended = 0
        for b in range(nb):
            sel = np.sort(s2_idx[b, :s2_len[b]])
            rows = np.arange(b * bq, min(N, (b + 1) * bq))
            attended += int(np.searchsorted(sel, rows, side="right").sum())
        work["pass3_block"] = {"bound": "hbm",
                               "bytes": float(gather(int(s2_len.sum())) + qo + nb * w.budget_k * 4),
                               "flops": 4.0 * d * Hq * attended}
    return work


# Random 256-byte row gather from a 140 MB table (the 32K layer's K+V is 134 MB), measured
# on this machine's B200 with CUDA events (profiles/probe_b200_memory_and_mufu.md): the rate
# an L2-resident gather can reach, given next to the HBM copy peak for the gather rows.
L2_GATHER_GBS = 11074.1


def traffic_table():
    """DRAM bytes per launch from the committed ncu capture, for rows whose kernel sources
    are all unchanged since the capture (sha256 match); other rows get None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_dram_traffic_gqa32k_step.json")
    try:
        with open(path) as f:
            tab = json.load(f)["rows"]
    except Exception:
        return {}
    out = {}
    for row, ent in tab.items():
        try:
            same = True
            for src, digest in ent["sources"].items():
                with open(os.path.join(ROOT, src), "rb") as f:
                    same = same and hashlib.sha256(f.read()).hexdigest() == digest
            if same:
                out[row] = ent["dram_bytes_per_launch"]
        except Exception:
            pass
    return out


def roofline_of(work, ms, pk, pk_kind, traffic=None):
    tf_peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    if work["bound"] == "tensor":
        ach = work["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": ach / tf_peak, "traffic": traffic,
                "peak_kind": f"bf16 dense, sustained, of {pk_kind}"}
    ach = work["bytes"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": traffic, "peak_kind": f"HBM copy, of {pk_kind}",
            "l2_gather_peak": L2_GATHER_GBS, "frac_of_l2_gather_peak": ach / L2_GATHER_GBS}


# ------------------------------------------------------------------ oracle (CPU) arm

def oracle_sample_step(inp, w, n_rows: int):
    """The fp64 oracle on a bounded, stratified sample of the step; returns the time it
    would take for the whole step, extrapolated by each part's per-row work."""
    import oracle
    N = w.N
    rows = np.array([int((m + 0.5) * N / n_rows) for m in range(n_rows)], dtype=np.int64)
    wr = (rows + 1).astype(np.float64)
    w_all = float(causal_pairs(N))
    kq = np.minimum(w.budget_k, rows + 1).astype(np.float64)
    kq_all = float(support_pairs(N, w.budget_k))
    ki = np.minimum(INDEXER_K, rows + 1).astype(np.float64)
    ki_all = float(support_pairs(N, INDEXER_K))
    total = 0.0
    # pass 1 + pass 2 per query (LSE and mass are computed inside the selection)
    t0 = time.perf_counter()
    idx, ln, _ = oracle.topk_rows(inp.q, inp.k, w.budget_k, rows)
    t1 = time.perf_counter()
    oracle.attn_rows(inp.q, inp.k, inp.v, rows, sup=idx, sup_len=ln)
    t2 = time.perf_counter()
    total += (t1 - t0) * w_all / wr.sum() + (t2 - t1) * kq_all / kq.sum()
    # block-shared: one block in the middle
    nb = -(-N // BLOCK_Q)
    b = nb // 2
    brows = np.arange(b * BLOCK_Q, min(N, (b + 1) * BLOCK_Q))
    t0 = time.perf_counter()
    bidx, bln, _ = oracle.block_topk(inp.q, inp.k, BLOCK_Q, w.budget_k, [b])
    t1 = time.perf_counter()
    r, s, sl = oracle.block_rows_support(bidx, bln, BLOCK_Q, N, [b])
    oracle.attn_rows(inp.q, inp.k, inp.v, r, sup=s, sup_len=sl)
    t2 = time.perf_counter()
    total += (t1 - t0) * w_all / float((brows + 1).sum()) + (t2 - t1) * nb
    # indexer
    t0 = time.perf_counter()
    xidx, xln, _ = oracle.indexer_topk_rows(inp.q_idx, inp.k_idx, INDEXER_K, rows)
    t1 = time.perf_counter()
    oracle.attn_rows(inp.q, inp.k, inp.v, rows, sup=xidx, sup_len=xln)
    t2 = time.perf_counter()
    total += (t1 - t0) * w_all / wr.sum() + (t2 - t1) * ki_all / ki.sum()
    # dense
    t0 = time.perf_counter()
    oracle.attn_rows(inp.q, inp.k, inp.v, rows)
    t1 = time.perf_counter()
    total += (t1 - t0) * w_all / wr.sum()
    return total


def calibrate_rows(inp, w, target_s: float):
    t0 = time.perf_counter()
    oracle_sample_step(inp, w, 4)
    dt = time.perf_counter() - t0
    return int(max(4, min(256, round(4 * target_s / max(dt, 1e-3)))))


def cpu_sample_desc(n_rows):
    return (f"{n_rows} stratified query rows (plus one block of {BLOCK_Q}) of the "
            f"{WORKLOAD} workload through every step; time extrapolated to all rows by "
            "per-row work ((i+1) for scoring, min(k, i+1) for the sparse recompute)")


def run_reference(args, w, inp, rank, world):
    import oracle
    if rank != 0:
        return
    n_rows = calibrate_rows(inp, w, 6.0)
    for _ in range(args.warmup):
        oracle_sample_step(inp, w, n_rows)
    ext = [oracle_sample_step(inp, w, n_rows) for _ in range(args.steps)]
    ms = 1e3 * statistics.mean(ext)
    value = w.N / (ms * 1e-3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; stands in for the pages' 4K-100K long-context evaluations)",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": cpu_sample_desc(n_rows)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, world, launch=None):
    idx_k = INDEXER_K if w.name == WORKLOAD else (w.budget_k if w.d_idx else None)
    extra = {"step_launch": launch} if launch else {}
    return {**extra, "workload": w.name, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "budget_k": w.budget_k, "block_q": list(w.block_q), "indexer_k": idx_k,
            "d_idx": w.d_idx or None, "rope": w.rope_base, "global_batch": world, "seq_len": w.N,
            "parallelism": f"replicas x{world} (independent layers, no collective)",
            "l2": "256 MB buffer written before every step (L2 is 126 MB)"}


# ------------------------------------------------------------------ our arm

def run_ours(args, w, inp, rank, world, local_rank):
    import top_attention_mass_b200 as tam
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    qx = inp.q_idx.to(dev) if inp.q_idx is not None else None
    kx = inp.k_idx.to(dev) if inp.k_idx is not None else None
    step = Step(tam, w, q, k, v, qx, kx)
    names = step.rows
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        step.run()
    tam.check_status(step.ws.get(256))
    torch.cuda.synchronize()
    work = algorithmic_work(step, w.N)

    # per-row breakdown: eager calls with CUDA events between them (same inputs)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(args.steps)]
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        step.run(ev[s])
    torch.cuda.synchronize()
    tam.check_status(step.ws.get(256))
    row_ms = {n: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
              for i, n in enumerate(names)}

    next_rows = measure_next_rows(args, tam, w, step, flush) if w.name == WORKLOAD else None

    # The step is captured once as a CUDA graph (every library launch of the step,
    # recorded on the capture stream) and replayed in the timed region, so host-side
    # enqueue time between the rows does not enter the device time.  --no-graph times
    # the eager calls instead.
    graph, per_step_launches = None, 0
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step.run()                      # warm-up on the capture's side stream
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = tam.kernel_launches()
        with torch.cuda.graph(graph):
            step.run()
        per_step_launches = tam.kernel_launches() - n0
        graph.replay()
        torch.cuda.synchronize()
        tam.check_status(step.ws.get(256))

    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(world, local_rank)
    torch.cuda.synchronize()
    clocks.start()
    launches0 = tam.kernel_launches()
    t_start.record()
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        if graph is not None:
            graph.replay()
        else:
            step.run()
    t_stop.record()
    torch.cuda.synchronize()
    launches = (per_step_launches * args.steps if graph is not None
                else tam.kernel_launches() - launches0)
    barrier(world, local_rank)
    clk = clocks.stop()
    tam.check_status(step.ws.get(256))
    total_ms = t_start.elapsed_time(t_stop)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / args.steps


    pk, pk_kind = peaks()
    traffic = traffic_table()
    rows = {}
    for n in names:
        r = roofline_of(work[n], row_ms[n], pk, pk_kind, traffic.get(n))
        rows[n] = {"ms": row_ms[n], "q_tok_s": w.N / (row_ms[n] * 1e-3), "roofline": r}
    dominant = max(names, key=lambda n: row_ms[n])

    e2e = measure_e2e(args, tam, w, inp, dev, world, local_rank)

    if rank != 0:
        return
    value = job_value(world, w.N, ms_step)
    oracle_sparsity = 1.0 - support_pairs(w.N, w.budget_k) / causal_pairs(w.N)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; stands in for the pages' 4K-100K long-context evaluations)",
        "config": config_dict(w, world, "CUDA graph replay of the step's library calls"
                              if graph is not None else "eager library calls"),
        "roofline": {**rows[dominant]["roofline"], "kernel": dominant},
        "rows": rows,
        "sparse_pass": sparse_pass_summary(w, row_ms),
        "support_quality": support_quality(step),
        "sparsity_selfcheck": {
            "this_workload": oracle_sparsity,
            "N4096_k256": 1.0 - support_pairs(4096, 256) / causal_pairs(4096),
            "N102400_k2048": 1.0 - support_pairs(102400, 2048) / causal_pairs(102400),
        },
        "clocks": clk,
        "next_rows": next_rows,
        "e2e": e2e,
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline and w.name == WORKLOAD:
        import oracle
        n_rows = calibrate_rows(inp, w, 15.0)
        t = oracle_sample_step(inp, w, n_rows)
        line["cpu_baseline"] = {"value": w.N / t, "unit": UNIT, "cores": oracle.threads(),
                                "kind": "oracle", "sample": cpu_sample_desc(n_rows)}
    print(json.dumps(line), flush=True)


def measure_next_rows(args, tam, w, step, flush):
    """Rows beyond the step (reported, not part of `value`): the fused, selection-block-
    shared indexer (block sums of each query's softmax of its indexer scores, top-k per
    block of BLOCK_Q queries), pass 3 on that support, the indexer's distillation
    target (KL of the indexer's distribution from the head-averaged mass), and a budget
    sweep (support mass at k = 256..2048 from one pass 2 at k = 2048)."""
    bq, kx = BLOCK_Q, INDEXER_K
    lse = tam.attention_lse(step.q, step.k, workspace=step.ws, check=False)
    # warm-up (first launches load the kernels; the workspace grows to its largest size)
    for _ in range(2):
        sup = tam.indexer_topk(step.qx, step.kx, kx, bq, workspace=step.ws, check=False)
        tam.sparse_support_attention(step.q, step.k, step.v, sup.idx, sup.length, bq,
                                     workspace=step.ws, check=False)
        tam.distill_kl(step.q, step.k, lse, step.qx, step.kx, workspace=step.ws, check=False)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        ev[s][0].record()
        sup = tam.indexer_topk(step.qx, step.kx, kx, bq, workspace=step.ws, check=False)
        ev[s][1].record()
        tam.sparse_support_attention(step.q, step.k, step.v, sup.idx, sup.length, bq,
                                     workspace=step.ws, check=False)
        ev[s][2].record()
    torch.cuda.synchronize()
    tam.check_status(step.ws.get(256))
    t_sel = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    t_att = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    n_sel = sup.length.cpu().numpy().astype(np.int64)
    # the indexer's distillation target (pass 1's lse is an input, as for pass 2)
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        evk[s][0].record()
        tam.distill_kl(step.q, step.k, lse, step.qx, step.kx, workspace=step.ws, check=False)
        evk[s][1].record()
    torch.cuda.synchronize()
    tam.check_status(step.ws.get(256))
    t_kl = statistics.mean(e[0].elapsed_time(e[1]) for e in evk)
    # budget sweep from one pass 2 at k_max = 2048: per-query support mass at 256..2048
    lse1 = lse
    budgets = [256, 512, 1024, 2048]
    sup = tam.mass_select(step.q, step.k, lse1, budgets[-1], 1, workspace=step.ws, check=False)
    tam.support_mass_curve(sup.value, sup.length, budgets)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        evs[s][0].record()
        sup = tam.mass_select(step.q, step.k, lse1, budgets[-1], 1, workspace=step.ws, check=False)
        evs[s][1].record()
        curve = tam.support_mass_curve(sup.value, sup.length, budgets)
        evs[s][2].record()
    torch.cuda.synchronize()
    tam.check_status(step.ws.get(256))
    t_p2 = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_cv = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    mean_mass = curve.mean(dim=0).cpu().tolist()
    # packed batch: the step's tokens as VARLEN_SEQS independent sequences, per-query
    # support at VARLEN_K (passes 1-3), and the dense comparator on the same batch
    cu = [0]
    for n in VARLEN_SEQS:
        cu.append(cu[-1] + n)
    vl = None
    if cu[-1] == w.N:
        for _ in range(2):
            tam.mass_oracle_prefill_varlen(step.q, step.k, step.v, cu, VARLEN_K, 1,
                                           workspace=step.ws, check=False)
            tam.dense_gqa_prefill_varlen(step.q, step.k, step.v, cu, workspace=step.ws,
                                         check=False)
        torch.cuda.synchronize()
        evv = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for s in range(args.steps):
            flush.fill_(s & 0xff)
            evv[s][0].record()
            tam.mass_oracle_prefill_varlen(step.q, step.k, step.v, cu, VARLEN_K, 1,
                                           workspace=step.ws, check=False)
            evv[s][1].record()
            tam.dense_gqa_prefill_varlen(step.q, step.k, step.v, cu, workspace=step.ws,
                                         check=False)
            evv[s][2].record()
        torch.cuda.synchronize()
        tam.check_status(step.ws.get(256))
        t_vo = statistics.mean(e[0].elapsed_time(e[1]) for e in evv)
        t_vd = statistics.mean(e[1].elapsed_time(e[2]) for e in evv)
        vl = {"seq_lens": list(VARLEN_SEQS), "budget_k": VARLEN_K,
              "ms_oracle_passes_1_3": t_vo, "q_tok_s_oracle": w.N / (t_vo * 1e-3),
              "ms_dense": t_vd, "q_tok_s_dense": w.N / (t_vd * 1e-3)}
    return {
        "varlen_batch": vl,
        "budget_sweep": {"ms_pass2_kmax": t_p2, "ms_curve": t_cv, "budgets": budgets,
                         "mean_support_mass": mean_mass,
                         "sparsity": [1.0 - support_pairs(w.N, b) / causal_pairs(w.N) for b in budgets]},
        "distill_kl": {"ms": t_kl, "q_tok_s": w.N / (t_kl * 1e-3),
                       "what": "KL(P_i || softmax(q_idx_i . k_idx)) per query, lse given"},
        "indexer_block_topk": {"ms": t_sel, "q_tok_s": w.N / (t_sel * 1e-3), "budget_k": kx,
                               "block_q": bq},
        "pass3_indexer_block": {"ms": t_att, "q_tok_s": w.N / (t_att * 1e-3),
                                "gathered_rows": int(n_sel.sum()) * w.Hkv},
    }


def measure_e2e(args, tam, w, inp, dev, world, local_rank):
    """Same step through the public API with pinned host inputs and results.

    Every step copies its inputs in from pinned host memory and every output back,
    on two copy streams next to the compute stream: inputs go to one of two device
    sets (the copy for step s+1 overlaps step s), and each row's outputs start back
    to the host as soon as that row is done.  The timed region runs from the first
    input copy to the last output copy."""
    if args.no_e2e:
        return None
    host_in = [inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()]
    if inp.q_idx is not None:
        host_in += [inp.q_idx.pin_memory(), inp.k_idx.pin_memory()]
    sets = [[torch.empty_like(t, device=dev) for t in host_in] for _ in range(2)]
    steps = [Step(tam, w, *d) for d in sets]
    for t_d, t_h in zip(sets[0], host_in):
        t_d.copy_(t_h)
    outs = steps[0].run()
    host_out = {n: torch.empty_like(t, device="cpu").pin_memory() for n, t in outs.items()}
    steps[1].ws = steps[0].ws                    # one workspace: the steps run in order
    for t_d, t_h in zip(sets[1], host_in):
        t_d.copy_(t_h)
    steps[1].run()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    # which outputs each row produces (copied back once that row is done)
    row_outs = {"pass1_lse": ["lse"], "pass2_mass_topk": ["s1_idx", "s1_len", "s1_mass"],
                "pass3_gather": ["o1"], "pass2_block_mass_topk": ["s2_idx", "s2_len", "s2_mass"],
                "pass3_block": ["o2"], "indexer_topk": ["s3_idx", "s3_len", "s3_score"],
                "pass3_indexer_support": ["o3"], "dense_prefill": ["od"]}
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = max(2, min(args.steps, 4))
    barrier(world, local_rank)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    in_ready = [torch.cuda.Event() for _ in range(n)]
    done = [None] * n                            # compute of step s finished reading its set
    for s in range(n):
        b = s % 2
        if s == 0:
            s_in.wait_stream(comp)
        if s >= 2:
            s_in.wait_event(done[s - 2])
        with torch.cuda.stream(s_in):
            for t_d, t_h in zip(sets[b], host_in):
                t_d.copy_(t_h, non_blocking=True)
        in_ready[s].record(s_in)
        comp.wait_event(in_ready[s])
        step = steps[b]
        ev = [torch.cuda.Event() for _ in range(len(step.rows) + 1)]
        outs = step.run(ev)
        done[s] = torch.cuda.Event()
        done[s].record(comp)
        for r, row in enumerate(step.rows):
            s_out.wait_event(ev[r + 1])
            with torch.cuda.stream(s_out):
                for name in row_outs[row]:
                    t = outs[name]
                    t.record_stream(s_out)
                    host_out[name].copy_(t, non_blocking=True)
    comp.wait_stream(s_out)
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world, local_rank)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n
    return {"value": job_value(world, w.N, ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "overlap": "inputs double-buffered on a copy stream; outputs copied per row on a second one"}


# ------------------------------------------------------------------ process group plumbing

def barrier(world, local_rank):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[local_rank])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    """The slowest rank's time: every replica's step is timed on its own device."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: query tokens of all replicas per second of the slowest one."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def support_quality(step):
    """Indexer support vs mass-oracle support (recall@k over rows with i+1 > k, when both
    use the same k) and each sparse output's max-abs distance from dense attention."""
    out, w = step.outputs, step.w
    res = {}
    od = out["od"].float()
    for key, name in (("o1", "per_query"), ("o2", "block_shared"), ("o3", "indexer")):
        if key in out:
            res[f"{name}_output_vs_dense_max_abs"] = float((out[key].float() - od).abs().max())
    if "s1_idx" in out and "s3_idx" in out and out["s1_idx"].shape == out["s3_idx"].shape:
        k = out["s1_idx"].shape[1]
        a, b = out["s1_idx"][k:].long(), out["s3_idx"][k:].long()       # rows i >= k are full
        if a.numel():
            pos = torch.searchsorted(a.contiguous(), b.contiguous()).clamp_(max=k - 1)
            hit = (torch.gather(a, 1, pos) == b).sum(dim=1).double() / k
            res["indexer_recall_at_k"] = float(hit.mean())
            res["recall_k"] = k
    return res


def workload_for(name: str):
    """The default step is the 32K layer with both supports (B_q = 64) and its indexer
    head (d_idx = 64, k = 1024 on the same tensors); other names are single workloads."""
    if name == WORKLOAD:
        base = tam_synth.WORKLOADS[WORKLOAD]
        return tam_synth.Workload(**{**base.__dict__, "d_idx": D_IDX})
    return tam_synth.WORKLOADS[name]


def sparse_pass_summary(w, row_ms):
    out = {}
    dense = row_ms["dense_prefill"]
    if "pass3_gather" in row_ms:
        out["per_query_q_tok_s"] = w.N / (row_ms["pass3_gather"] * 1e-3)
        out["speedup_vs_dense"] = dense / row_ms["pass3_gather"]
        out["oracle_pass12_plus3_q_tok_s"] = w.N / 1e-3 / (row_ms["pass1_lse"]
                                                           + row_ms["pass2_mass_topk"]
                                                           + row_ms["pass3_gather"])
    if "pass3_block" in row_ms:
        out["block_shared_q_tok_s"] = w.N / (row_ms["pass3_block"] * 1e-3)
        out["block_shared_speedup_vs_dense"] = dense / row_ms["pass3_block"]
        out["oracle_block_pass12_plus3_q_tok_s"] = w.N / 1e-3 / (
            row_ms["pass1_lse"] + row_ms["pass2_block_mass_topk"] + row_ms["pass3_block"])
    if "pass3_indexer_support" in row_ms:
        out["indexer_support_speedup_vs_dense"] = dense / row_ms["pass3_indexer_support"]
        out["indexer_path_speedup_vs_dense"] = dense / (row_ms["indexer_topk"]
                                                        + row_ms["pass3_indexer_support"])
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager library calls instead of a CUDA-graph replay of the step")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="gqa32k_2pct (default: every row), gqa4k_needles, longctx_<N>, indexer32k")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workload_for(args.workload)
    if args.impl == "reference":
        if rank != 0:
            return
        if w.name != WORKLOAD:
            print(json.dumps({"impl": "reference", "unavailable":
                              "the oracle arm is sampled on the default 32K workload only"}))
            return
        inp = tam_synth.make_inputs(w)
        run_reference(args, w, inp, rank, world)
        return
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    inp = tam_synth.make_inputs(w)
    try:
        run_ours(args, w, inp, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
