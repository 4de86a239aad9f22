#!/usr/bin/env python
"""Benchmark of the attention-mass top-k path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

The step (what `value` measures) is one call of the attention-mass oracle,
tam_mass_oracle_prefill, on one causal GQA prefill layer of the 32K workload
(N=32768, Hq=32, Hkv=8, d=128, bf16; sink at token 0, 64 planted needles) with
per-query support k=655: pass 1 (per-head LSE), pass 2 (head-averaged mass and its
top-k, streamed) and pass 3 (the sparse recompute on the support: the gathered
sparse attention).  value = query tokens of all ranks / step time (max over
ranks), i.e. the metric "query-tokens/s per GQA layer (mass oracle, sparse pass)".

Reported beside it (not part of value):
  rows            each pass of the step timed on its own entry point, with its roofline
                  (roofline = the longest of them);
  block_shared    the same call with block-shared support (B_q = 64), and its passes;
  all_rows_step   every row of the hot path in one CUDA graph: both oracles, the
                  indexer top-k (d_idx = 64, k = 1024) and pass 3 on its support, the
                  dense comparator;
  gather_out_of_l2  per-query pass 3 on a 262144-token layer whose K/V halves are four
                  times the L2 (random support, k = 2048), against HBM;
  support_quality the indexer's support against the mass oracle's at k = 1024
                  (recall@k, output difference), outputs against dense;
  next_rows       the fused block-shared indexer, the distillation target, the budget
                  sweep, a packed batch of eight sequences and a head-dim-256 layer.
With N > 1 GPUs every rank runs an independent replica of the workload (weak
scaling, no collective on the data path).  `--impl reference` times the fp64 CPU
oracle on a bounded sample of the step instead (rank 0 only).  `--workload` runs
another configuration (gqa4k_needles, longctx_<N>, indexer32k) as the step.
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
# per-query pass 3 with K/V far beyond the L2: 256K tokens (the longest context of the
# pages' TTFT figures), Hq 32 / Hkv 8, so that each half of the KV groups the gather walks
# (2 KB of K and V per key) is 537 MB against 126 MB of L2
GATHER_BIG = dict(N=262144, Hq=32, Hkv=8, d=128, k=2048)
# a head-dim-256 layer with the same bytes per token (q 16 x 256, k/v 8 x 256)
HEAD_DIM_256 = dict(N=32768, Hq=16, Hkv=8, d=256, k=655)
# L2 ceiling of this GPU as ncu states it (peak L2 sector rate x 32 B), read from the
# committed capture summarised in profiles/l2_sector_peak_b200.md
L2_PEAK_GBS = 34580.0
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


# ------------------------------------------------------------------ the calls

class Calls:
    """Device-resident inputs of one workload and the library calls of every row."""

    def __init__(self, tam, w, q, k, v, qx=None, kx=None):
        self.tam, self.w = tam, w
        self.q, self.k, self.v, self.qx, self.kx = q, k, v, qx, kx
        self.ws = tam.Workspace(q.device)
        self.out = {}

    @property
    def per_query(self):
        return 1 in self.w.block_q

    @property
    def block_q(self):
        return max(self.w.block_q)

    @property
    def indexer_k(self):
        return INDEXER_K if self.w.name == WORKLOAD else self.w.budget_k

    # the step: one oracle call (per query if the workload has it, else block-shared)
    def prefill(self, block_q=None):
        bq = block_q or (1 if self.per_query else self.block_q)
        r = self.tam.mass_oracle_prefill(self.q, self.k, self.v, self.w.budget_k, bq,
                                         workspace=self.ws, check=False)
        tag = "p1" if bq == 1 else "pb"
        self.out.update({f"{tag}_idx": r.idx, f"{tag}_len": r.length, f"{tag}_mass": r.value,
                         f"{tag}_lse": r.lse, f"{tag}_out": r.out})
        return r

    def row(self, name):
        t, w, ws, o = self.tam, self.w, self.ws, self.out
        if name == "pass1_lse":
            o["lse"] = t.attention_lse(self.q, self.k, workspace=ws, check=False)
        elif name == "pass2_mass_topk":
            s = t.mass_select(self.q, self.k, o["lse"], w.budget_k, 1, workspace=ws, check=False)
            o.update(s1_idx=s.idx, s1_len=s.length, s1_mass=s.value)
        elif name == "pass3_gather":
            o["o1"] = t.sparse_support_attention(self.q, self.k, self.v, o["s1_idx"], o["s1_len"],
                                                 1, workspace=ws, check=False)
        elif name == "pass2_block_mass_topk":
            s = t.mass_select(self.q, self.k, o["lse"], w.budget_k, self.block_q, workspace=ws,
                              check=False)
            o.update(s2_idx=s.idx, s2_len=s.length, s2_mass=s.value)
        elif name == "pass3_block":
            o["o2"] = t.sparse_support_attention(self.q, self.k, self.v, o["s2_idx"], o["s2_len"],
                                                 self.block_q, workspace=ws, check=False)
        elif name == "indexer_topk":
            s = t.indexer_topk(self.qx, self.kx, self.indexer_k, workspace=ws, check=False)
            o.update(s3_idx=s.idx, s3_len=s.length, s3_score=s.value)
        elif name == "pass3_indexer_support":
            o["o3"] = t.sparse_support_attention(self.q, self.k, self.v, o["s3_idx"], o["s3_len"],
                                                 1, workspace=ws, check=False)
        elif name == "dense_prefill":
            o["od"] = t.dense_gqa_prefill(self.q, self.k, self.v, workspace=ws, check=False)
        else:
            raise KeyError(name)

    def rows(self, names, events=None):
        for n, name in enumerate(names):
            if events is not None:
                events[n].record()
            self.row(name)
        if events is not None:
            events[len(names)].record()


def step_rows(w):
    """The passes of the step, each on its own entry point (per query, else block)."""
    if 1 in w.block_q:
        return ("pass1_lse", "pass2_mass_topk", "pass3_gather")
    return ("pass1_lse", "pass2_block_mass_topk", "pass3_block")


def all_rows(w):
    rows = ["pass1_lse"]
    if 1 in w.block_q:
        rows += ["pass2_mass_topk", "pass3_gather"]
    if any(b > 1 for b in w.block_q):
        rows += ["pass2_block_mass_topk", "pass3_block"]
    if w.d_idx:
        rows += ["indexer_topk", "pass3_indexer_support"]
    rows.append("dense_prefill")
    return tuple(rows)


def capture(tam, dev, fn):
    """fn's library launches captured once as a CUDA graph (after a warm-up on the
    capture's side stream); returns (graph, kernels launched per replay)."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = tam.kernel_launches()
    with torch.cuda.graph(g):
        fn()
    n = tam.kernel_launches() - n0
    g.replay()
    torch.cuda.synchronize()
    return g, n


def time_replays(graph, flush, steps, warm=False):
    """Per-replay device times (ms) of `graph`; the L2 is flushed before every replay
    (outside the timed events) unless warm."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s in range(steps):
        if not warm:
            flush.fill_(s & 0xff)
        ev[s][0].record()
        graph.replay()
        ev[s][1].record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def row_times(calls, names, flush, steps):
    """Eager per-row device times: CUDA events between the calls, L2 flushed first; one
    untimed round first, then the median over `steps` rounds (an eager call's events also
    see host-side gaps, which the median keeps out)."""
    calls.rows(names)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(steps)]
    for s in range(steps):
        flush.fill_(s & 0xff)
        calls.rows(names, ev[s])
    torch.cuda.synchronize()
    return {n: statistics.median(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps))
            for i, n in enumerate(names)}


# ------------------------------------------------------------------ rooflines

def algorithmic_work(calls, N):
    """Per-row algorithmic flops/bytes (what the method must do, not what it avoids)."""
    w, outs = calls.w, calls.out
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
    sp1 = support_pairs(N, w.budget_k)
    work["pass3_gather"] = {"bound": "l2", "bytes": float(gather(sp1) + qo + N * w.budget_k * 4 + N * 4)}
    kx = calls.indexer_k
    sp3 = support_pairs(N, kx)
    work["pass3_indexer_support"] = {"bound": "l2",
                                     "bytes": float(gather(sp3) + qo + N * kx * 4 + N * 4)}
    if "s2_len" in outs:
        bq = calls.block_q
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


def roofline_of(work, ms, pk, pk_kind, traffic=None):
    tf_peak = pk.get("bf16_tflops", pk.get("bf16_tflops_sustained"))
    if work["bound"] == "tensor":
        ach = work["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": ach / tf_peak, "traffic": traffic,
                "peak_kind": f"bf16 dense, burst, of {pk_kind}"}
    ach = work["bytes"] / (ms * 1e-3) / 1e9
    r = {"bound": work["bound"], "achieved": ach, "unit": "GB/s", "traffic": traffic,
         "frac_of_hbm": ach / pk["hbm_gbs"]}
    if work["bound"] == "l2":
        r.update(peak=L2_PEAK_GBS, frac=ach / L2_PEAK_GBS,
                 peak_kind="L2 sector ceiling per ncu (profiles/l2_sector_peak_b200.md); the "
                           "K/V gathered (134 MB, walked in two 67 MB halves) stays in L2")
    else:
        r.update(bound="hbm", peak=pk["hbm_gbs"], frac=ach / pk["hbm_gbs"],
                 peak_kind=f"HBM copy, of {pk_kind}")
    if "flops" in work:
        r["tflops"] = work["flops"] / (ms * 1e-3) / 1e12
    return r


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


# ------------------------------------------------------------------ oracle (CPU) arm

def oracle_sample_step(inp, w, n_rows: int):
    """The fp64 oracle on a bounded, stratified sample of the step (passes 1-3 for the
    step's support); returns the time it would take for the whole step, extrapolated
    by each part's per-row work ((i+1) for scoring, min(k, i+1) for the recompute)."""
    import oracle
    N = w.N
    rows = np.array([int((m + 0.5) * N / n_rows) for m in range(n_rows)], dtype=np.int64)
    wr = (rows + 1).astype(np.float64)
    w_all = float(causal_pairs(N))
    if 1 in w.block_q:
        kq = np.minimum(w.budget_k, rows + 1).astype(np.float64)
        kq_all = float(support_pairs(N, w.budget_k))
        t0 = time.perf_counter()
        idx, ln, _ = oracle.topk_rows(inp.q, inp.k, w.budget_k, rows)
        t1 = time.perf_counter()
        oracle.attn_rows(inp.q, inp.k, inp.v, rows, sup=idx, sup_len=ln)
        t2 = time.perf_counter()
        return (t1 - t0) * w_all / wr.sum() + (t2 - t1) * kq_all / kq.sum()
    bq = max(w.block_q)
    nb = -(-N // bq)
    blocks = np.unique(np.minimum(nb - 1, (rows // bq)))[: max(1, n_rows // 8)]
    brows = np.concatenate([np.arange(b * bq, min(N, (b + 1) * bq)) for b in blocks])
    t0 = time.perf_counter()
    bidx, bln, _ = oracle.block_topk(inp.q, inp.k, bq, w.budget_k, blocks)
    t1 = time.perf_counter()
    r, s, sl = oracle.block_rows_support(bidx, bln, bq, N, blocks)
    oracle.attn_rows(inp.q, inp.k, inp.v, r, sup=s, sup_len=sl)
    t2 = time.perf_counter()
    return (t1 - t0) * w_all / float((brows + 1).sum()) + (t2 - t1) * nb / len(blocks)


def calibrate_rows(inp, w, target_s: float):
    t0 = time.perf_counter()
    oracle_sample_step(inp, w, 4)
    dt = time.perf_counter() - t0
    return int(max(4, min(512, round(4 * target_s / max(dt, 1e-3)))))


def cpu_sample_desc(w, n_rows):
    what = ("query rows" if 1 in w.block_q else f"blocks of {max(w.block_q)} queries (about "
            f"{max(1, n_rows // 8)})")
    return (f"{n_rows} stratified {what} of the {w.name} workload through passes 1-3 of the "
            "step; time extrapolated to all rows by per-row work ((i+1) for scoring, "
            "min(k, i+1) for the sparse recompute)")


def run_reference(args, w, inp, rank, world):
    import oracle
    if rank != 0:
        return
    n_rows = calibrate_rows(inp, w, 3.0)
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
                         "sample": cpu_sample_desc(w, n_rows)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, world):
    bq = 1 if 1 in w.block_q else max(w.block_q)
    return {"workload": w.name, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "budget_k": w.budget_k, "block_q": bq,
            "step": (f"one tam_mass_oracle_prefill call: pass 1, pass 2 and its "
                     f"{'per-query' if bq == 1 else f'block-shared (B_q {bq})'} top-k, pass 3"),
            "rope": w.rope_base, "global_batch": world, "seq_len": w.N,
            "parallelism": f"replicas x{world} (independent layers, no collective)",
            "l2": "256 MB buffer written before every timed step (L2 is 126 MB)"}


# ------------------------------------------------------------------ our arm

def run_ours(args, w, inp, rank, world, local_rank):
    import top_attention_mass_b200 as tam
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    qx = inp.q_idx.to(dev) if inp.q_idx is not None else None
    kx = inp.k_idx.to(dev) if inp.k_idx is not None else None
    calls = Calls(tam, w, q, k, v, qx, kx)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    names = step_rows(w)
    block_q = 1 if calls.per_query else calls.block_q

    # warm-up: the step and its passes (the first launches load the kernels)
    for _ in range(args.warmup):
        calls.prefill()
        calls.rows(names)
    torch.cuda.synchronize()
    tam.check_status(calls.ws.get(256))
    fb_rows = (tam.mass_fallback_rows(q, k, w.budget_k, calls.ws) if calls.per_query else None)

    # the step as one CUDA graph (every launch of the call), replayed in the timed region
    graph, per_step_launches = capture(tam, dev, lambda: calls.prefill(block_q))
    tam.check_status(calls.ws.get(256))
    clocks = ClockSampler(local_rank)
    barrier(world, local_rank)
    torch.cuda.synchronize()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    times = time_replays(graph, flush, args.steps)
    t1.record()
    torch.cuda.synchronize()
    barrier(world, local_rank)
    clk = clocks.stop()
    tam.check_status(calls.ws.get(256))
    ms_step = max_over_ranks(statistics.mean(times), world, dev)
    region_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    warm_ms = statistics.mean(time_replays(graph, flush, args.steps, warm=True))
    launches = per_step_launches * args.steps
    del graph

    # the passes of the step, each on its own entry point
    pk, pk_kind = peaks()
    traffic = traffic_table()
    row_ms = row_times(calls, names, flush, args.steps)
    tam.check_status(calls.ws.get(256))
    # the dense comparator on the same layer (every workload), for the sparse-pass speedup
    dense_ms = row_times(calls, ("dense_prefill",), flush, args.steps)["dense_prefill"]
    tam.check_status(calls.ws.get(256))

    extra = {}
    if w.name == WORKLOAD and not args.no_extras:
        extra = measure_extras(args, tam, w, calls, flush, dev)
    work = algorithmic_work(calls, w.N)
    rows = {}
    for n in names:
        rows[n] = {"ms": row_ms[n], "q_tok_s": w.N / (row_ms[n] * 1e-3),
                   "roofline": roofline_of(work[n], row_ms[n], pk, pk_kind, traffic.get(n))}
    dominant = max(names, key=lambda n: row_ms[n])
    for key in ("block_shared", "all_rows_step"):
        for n, r in extra.get(key, {}).get("rows", {}).items():
            r["roofline"] = roofline_of(work[n], r["ms"], pk, pk_kind, traffic.get(n))

    e2e = measure_e2e(args, tam, w, inp, dev, world, local_rank, block_q)

    if rank != 0:
        return
    value = job_value(world, w.N, ms_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; stands in for the pages' 4K-100K long-context evaluations)",
        "config": config_dict(w, world),
        "roofline": {**rows[dominant]["roofline"], "kernel": dominant},
        "rows": rows,
        "dense_comparator": {
            "ms": dense_ms, "q_tok_s": w.N / (dense_ms * 1e-3),
            "roofline": roofline_of({"bound": "tensor", "flops": 4.0 * w.d * w.Hq * causal_pairs(w.N)},
                                    dense_ms, pk, pk_kind),
            "step_vs_dense": dense_ms / ms_step,
            "sparse_pass3_speedup_vs_dense": dense_ms / row_ms[names[-1]]},
        "timed_region_ms": region_ms,
        "warm_l2_ms_per_step": warm_ms,
        "fallback_rows": fb_rows,
        **extra,
        "sparsity_selfcheck": {
            "this_workload": 1.0 - support_pairs(w.N, w.budget_k) / causal_pairs(w.N),
            "N4096_k256": 1.0 - support_pairs(4096, 256) / causal_pairs(4096),
            "N102400_k2048": 1.0 - support_pairs(102400, 2048) / causal_pairs(102400),
        },
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        n_rows = calibrate_rows(inp, w, 15.0)
        t = oracle_sample_step(inp, w, n_rows)
        line["cpu_baseline"] = {"value": w.N / t, "unit": UNIT, "cores": oracle.threads(),
                                "kind": "oracle", "sample": cpu_sample_desc(w, n_rows)}
    print(json.dumps(line), flush=True)


def measure_extras(args, tam, w, calls, flush, dev):
    """Everything reported beside the step on the 32K workload (see the module doc)."""
    out = {}
    # block-shared oracle call (B_q = 64) and its passes
    g, _ = capture(tam, dev, lambda: calls.prefill(BLOCK_Q))
    ms_b = statistics.mean(time_replays(g, flush, args.steps))
    del g
    brows = ("pass1_lse", "pass2_block_mass_topk", "pass3_block")
    calls.rows(brows)
    bt = row_times(calls, brows, flush, args.steps)
    out["block_shared"] = {"block_q": BLOCK_Q, "ms": ms_b, "q_tok_s": w.N / (ms_b * 1e-3),
                           "rows": {n: {"ms": bt[n], "q_tok_s": w.N / (bt[n] * 1e-3)} for n in brows}}
    # every row of the hot path in one graph
    names = all_rows(w)
    g, _ = capture(tam, dev, lambda: calls.rows(names))
    ms_all = statistics.mean(time_replays(g, flush, args.steps))
    del g
    at = row_times(calls, names, flush, args.steps)
    tam.check_status(calls.ws.get(256))
    out["all_rows_step"] = {"rows_in_order": list(names), "ms": ms_all,
                            "q_tok_s": w.N / (ms_all * 1e-3),
                            "rows": {n: {"ms": at[n], "q_tok_s": w.N / (at[n] * 1e-3)} for n in names}}
    dense = at["dense_prefill"]
    out["sparse_pass"] = {
        "per_query_pass3_speedup_vs_dense": dense / at["pass3_gather"],
        "block_shared_pass3_speedup_vs_dense": dense / at["pass3_block"],
        "indexer_support_pass3_speedup_vs_dense": dense / at["pass3_indexer_support"],
        "indexer_path_speedup_vs_dense": dense / (at["indexer_topk"] + at["pass3_indexer_support"]),
        "per_query_oracle_passes_1_3_vs_dense": dense / (at["pass1_lse"] + at["pass2_mass_topk"]
                                                         + at["pass3_gather"]),
    }
    out["support_quality"] = support_quality(tam, w, calls, flush, args.steps)
    out["gather_out_of_l2"] = measure_gather_big(tam, dev, flush, args.steps)
    out["next_rows"] = measure_next_rows(args, tam, w, calls, flush)
    return out


def support_quality(tam, w, calls, flush, steps):
    """C5: the indexer's support (k = 1024) against the mass oracle's per-query support
    at the same k on the same tensors: recall@k over the rows with i+1 > k, and the
    max-abs difference of the two pass-3 outputs; each sparse output against dense;
    and the random-support stress row's pass-3 time at this k."""
    o = calls.out
    kx = calls.indexer_k
    m = tam.mass_select(calls.q, calls.k, o["lse"], kx, 1, workspace=calls.ws, check=False)
    om = tam.sparse_support_attention(calls.q, calls.k, calls.v, m.idx, m.length, 1,
                                      workspace=calls.ws, check=False)
    a, b = m.idx[kx:].long(), o["s3_idx"][kx:].long()          # rows i >= k hold k keys
    res = {"recall_k": kx}
    if a.numel():
        pos = torch.searchsorted(a.contiguous(), b.contiguous()).clamp_(max=kx - 1)
        hit = (torch.gather(a, 1, pos) == b).sum(dim=1).double() / kx
        res["indexer_recall_at_k"] = float(hit.mean())
    res["indexer_output_vs_mass_oracle_max_abs"] = float((o["o3"].float() - om.float()).abs().max())
    res["indexer_output_vs_mass_oracle_mean_abs"] = float((o["o3"].float() - om.float()).abs().mean())
    od = o["od"].float()
    for key, name in (("o1", "per_query"), ("o2", "block_shared"), ("o3", "indexer")):
        res[f"{name}_output_vs_dense_max_abs"] = float((o[key].float() - od).abs().max())
    # stress row: uniform-random support of the indexer's budget
    sidx, slen = tam_synth.stratified_support(w.N, kx, seed=7, device=calls.q.device)
    f = lambda: tam.sparse_support_attention(calls.q, calls.k, calls.v, sidx, slen, 1,  # noqa: E731
                                             workspace=calls.ws, check=False)
    f()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s in range(steps):
        flush.fill_(s & 0xff)
        ev[s][0].record()
        f()
        ev[s][1].record()
    torch.cuda.synchronize()
    res["stress_row_pass3_ms"] = statistics.mean(x.elapsed_time(y) for x, y in ev)
    res["stress_row_support"] = f"one uniform key per stratum of [0, i], k = {kx}"
    del m, om, sidx, slen
    return res


def measure_gather_big(tam, dev, flush, steps):
    """Per-query pass 3 with K/V far beyond the L2: 262144 tokens, Hq 32 / Hkv 8, d 128,
    random support of k = 2048 per query (one uniform key per stratum of [0, i]);
    inputs drawn on the device (the values do not matter to a gather's time)."""
    c = GATHER_BIG
    N, Hq, Hkv, d, kb = c["N"], c["Hq"], c["Hkv"], c["d"], c["k"]
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    q = torch.randn(N, Hq, d, generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn(N, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(N, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    idx, ln = tam_synth.stratified_support(N, kb, seed=9, device=dev)
    ws = tam.Workspace(dev)
    f = lambda: tam.sparse_support_attention(q, k, v, idx, ln, 1, workspace=ws, check=False)  # noqa: E731
    f()
    torch.cuda.synchronize()
    n = max(2, min(steps, 3))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for s in range(n):
        flush.fill_(s & 0xff)
        ev[s][0].record()
        f()
        ev[s][1].record()
    torch.cuda.synchronize()
    tam.check_status(ws.get(256))
    ms = statistics.mean(x.elapsed_time(y) for x, y in ev)
    gathered = support_pairs(N, kb) * Hkv * 2 * d * 2
    nbytes = gathered + 2 * N * Hq * d * 2 + N * kb * 4 + N * 4
    pk, pk_kind = peaks()
    ach = nbytes / (ms * 1e-3) / 1e9
    del q, k, v, idx, ln, ws
    torch.cuda.empty_cache()
    # DRAM bytes of this launch from the committed one-pass capture (None once the kernel
    # source has changed since): the L2 still serves part of the gathered rows here, so the
    # DRAM rate, not the algorithmic one, is the kernel's HBM fraction
    traffic = traffic_table().get("pass3_gather_stress256k")
    roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": traffic,
            "peak_kind": f"HBM copy, of {pk_kind}", "frac_of_8tbs_nominal": ach / 8000.0}
    if traffic:
        roof["dram_rate_gbs"] = traffic / (ms * 1e-3) / 1e9
        roof["dram_frac"] = roof["dram_rate_gbs"] / pk["hbm_gbs"]
    return {"N": N, "Hq": Hq, "Hkv": Hkv, "d": d, "budget_k": kb,
            "kv_bytes_per_half_of_the_groups": N * (Hkv // 2) * 2 * d * 2,
            "ms": ms, "q_tok_s": N / (ms * 1e-3), "bytes": nbytes, "roofline": roof}


def measure_next_rows(args, tam, w, calls, flush):
    """Rows beyond the step (reported, not part of `value`): the fused, selection-block-
    shared indexer (block sums of each query's softmax of its indexer scores, top-k per
    block of BLOCK_Q queries), pass 3 on that support, the indexer's distillation
    target (KL of the indexer's distribution from the head-averaged mass), a budget
    sweep (support mass at k = 256..2048 from one pass 2 at k = 2048) and a packed
    batch of eight sequences."""
    bq, kx = BLOCK_Q, INDEXER_K
    ws = calls.ws
    lse = tam.attention_lse(calls.q, calls.k, workspace=ws, check=False)

    def timed(fns):
        for _ in range(2):
            for fn in fns:
                fn()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
              for _ in range(args.steps)]
        for s in range(args.steps):
            flush.fill_(s & 0xff)
            for i, fn in enumerate(fns):
                ev[s][i].record()
                fn()
            ev[s][-1].record()
        torch.cuda.synchronize()
        tam.check_status(ws.get(256))
        return [statistics.median(e[i].elapsed_time(e[i + 1]) for e in ev) for i in range(len(fns))]

    box = {}

    def sel():
        box["sup"] = tam.indexer_topk(calls.qx, calls.kx, kx, bq, workspace=ws, check=False)

    def att():
        tam.sparse_support_attention(calls.q, calls.k, calls.v, box["sup"].idx,
                                     box["sup"].length, bq, workspace=ws, check=False)

    t_sel, t_att = timed([sel, att])
    n_sel = box["sup"].length.cpu().numpy().astype(np.int64)
    (t_kl,) = timed([lambda: tam.distill_kl(calls.q, calls.k, lse, calls.qx, calls.kx,
                                            workspace=ws, check=False)])
    budgets = [256, 512, 1024, 2048]

    def p2():
        box["s"] = tam.mass_select(calls.q, calls.k, lse, budgets[-1], 1, workspace=ws, check=False)

    def curve():
        box["c"] = tam.support_mass_curve(box["s"].value, box["s"].length, budgets)

    t_p2, t_cv = timed([p2, curve])
    mean_mass = box["c"].mean(dim=0).cpu().tolist()
    cu = [0]
    for n in VARLEN_SEQS:
        cu.append(cu[-1] + n)
    vl = None
    if cu[-1] == w.N:
        t_vo, t_vd = timed([
            lambda: tam.mass_oracle_prefill_varlen(calls.q, calls.k, calls.v, cu, VARLEN_K, 1,
                                                   workspace=ws, check=False),
            lambda: tam.dense_gqa_prefill_varlen(calls.q, calls.k, calls.v, cu, workspace=ws,
                                                 check=False)])
        vl = {"seq_lens": list(VARLEN_SEQS), "budget_k": VARLEN_K,
              "ms_oracle_passes_1_3": t_vo, "q_tok_s_oracle": w.N / (t_vo * 1e-3),
              "ms_dense": t_vd, "q_tok_s_dense": w.N / (t_vd * 1e-3)}
    hd = measure_head_dim_256(tam, calls.q.device, timed)
    return {
        "head_dim_256": hd,
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


def measure_head_dim_256(tam, dev, timed):
    """A d = 256 layer with the 32K layer's bytes per token (N 32768, Hq 16 / Hkv 8):
    the per-query oracle call (k = 655) and the dense comparator, inputs drawn on the
    device."""
    c = HEAD_DIM_256
    N, Hq, Hkv, d, kb = c["N"], c["Hq"], c["Hkv"], c["d"], c["k"]
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    q = torch.randn(N, Hq, d, generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn(N, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(N, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    ws = tam.Workspace(dev)
    t_or, t_de = timed([
        lambda: tam.mass_oracle_prefill(q, k, v, kb, 1, workspace=ws, check=False),
        lambda: tam.dense_gqa_prefill(q, k, v, workspace=ws, check=False)])
    fb = tam.mass_fallback_rows(q, k, kb, ws)
    pk, _ = peaks()
    dense_tf = 4.0 * d * Hq * causal_pairs(N) / (t_de * 1e-3) / 1e12
    del q, k, v, ws
    torch.cuda.empty_cache()
    return {**c, "ms_oracle_passes_1_3": t_or, "q_tok_s_oracle": N / (t_or * 1e-3),
            "fallback_rows": fb, "ms_dense": t_de, "q_tok_s_dense": N / (t_de * 1e-3),
            "dense_tflops": dense_tf,
            "dense_frac_of_burst": dense_tf / pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])}


def measure_e2e(args, tam, w, inp, dev, world, local_rank, block_q):
    """The step through the public API with pinned host inputs and results.

    Every step copies its inputs (Q, K, V) in from pinned host memory and every output
    (support indices, lengths, masses, lse, sparse output) back, on two copy streams
    next to the compute stream: inputs go to one of two device sets (the copy for step
    s+1 overlaps step s), and the outputs of step s go back once it is done.  The timed
    region runs from the first input copy to the last output copy."""
    if args.no_e2e:
        return None
    host_in = [inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()]
    sets = [[torch.empty_like(t, device=dev) for t in host_in] for _ in range(2)]
    ws = tam.Workspace(dev)

    def call(b):
        q, k, v = sets[b]
        r = tam.mass_oracle_prefill(q, k, v, w.budget_k, block_q, workspace=ws, check=False)
        return [r.idx, r.length, r.value, r.lse, r.out]

    for b in range(2):
        for t_d, t_h in zip(sets[b], host_in):
            t_d.copy_(t_h)
    outs = call(0)
    host_out = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = max(2, min(args.steps, 4))
    barrier(world, local_rank)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    done = [None] * n
    for s in range(n):
        b = s % 2
        if s == 0:
            s_in.wait_stream(comp)
        if s >= 2:
            s_in.wait_event(done[s - 2])
        with torch.cuda.stream(s_in):
            for t_d, t_h in zip(sets[b], host_in):
                t_d.copy_(t_h, non_blocking=True)
        ready = torch.cuda.Event()
        ready.record(s_in)
        comp.wait_event(ready)
        outs = call(b)
        done[s] = torch.cuda.Event()
        done[s].record(comp)
        s_out.wait_event(done[s])
        with torch.cuda.stream(s_out):
            for t, h in zip(outs, host_out):
                t.record_stream(s_out)
                h.copy_(t, non_blocking=True)
    comp.wait_stream(s_out)
    e1.record(comp)
    torch.cuda.synchronize()
    tam.check_status(ws.get(256))
    barrier(world, local_rank)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n
    return {"value": job_value(world, w.N, ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "call": "top_attention_mass_b200.mass_oracle_prefill (C ABI tam_mass_oracle_prefill)",
            "overlap": "inputs double-buffered on a copy stream; outputs copied back on a second one"}


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


def workload_for(name: str):
    """The default step is the 32K layer with both supports (B_q = 64) and its indexer
    head (d_idx = 64, k = 1024 on the same tensors); other names are single workloads."""
    if name == WORKLOAD:
        base = tam_synth.WORKLOADS[WORKLOAD]
        return tam_synth.Workload(**{**base.__dict__, "d_idx": D_IDX})
    return tam_synth.WORKLOADS[name]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the step and its passes only (no block-shared call, all-rows "
                         "step, out-of-L2 gather, support quality or next rows)")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="gqa32k_2pct (default), gqa4k_needles, longctx_<N>, indexer32k")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workload_for(args.workload)
    if args.impl == "reference":
        if rank != 0:
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
