"""The benchmark's roofline arithmetic on the host: per-unit work against closed forms,
the roofline fractions, and the committed DRAM-traffic table's staleness check (a row is
used only while its kernel sources hash to the recorded digests)."""
import json
import os
import shutil

import numpy as np

import bench


def test_pair_counts_match_closed_forms():
    for N in (1, 7, 4096, 32768):
        assert bench.causal_pairs(N) == N * (N + 1) // 2
    for N, k in ((4096, 256), (32768, 655), (102400, 2048), (10, 100)):
        # sum over i of min(k, i + 1): the first k rows grow, the rest hold k
        m = min(N, k)
        closed = m * (m + 1) // 2 + (N - m) * k
        assert bench.support_pairs(N, k) == closed
    # the pages' sparsity endpoints (technical report §3.1): 87.9 % and 96.0 %
    sp = lambda N, k: 1.0 - bench.support_pairs(N, k) / bench.causal_pairs(N)  # noqa: E731
    assert round(100 * sp(4096, 256), 1) == 87.9
    assert round(100 * sp(102400, 2048), 1) == 96.0


def test_roofline_fractions():
    pk = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    r = bench.roofline_of({"bound": "tensor", "flops": 8.0e12}, 10.0, pk, "test")
    assert abs(r["achieved"] - 800.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12
    r = bench.roofline_of({"bound": "hbm", "bytes": 3.2e10}, 10.0, pk, "test", traffic=1.0e9)
    assert abs(r["achieved"] - 3200.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12
    assert r["traffic"] == 1.0e9
    r = bench.roofline_of({"bound": "l2", "bytes": bench.L2_PEAK_GBS * 1e7}, 10.0, pk, "test")
    assert abs(r["frac"] - 1.0) < 1e-12 and abs(r["frac_of_hbm"] - bench.L2_PEAK_GBS / 6400.0) < 1e-9
    assert abs(bench.job_value(4, 32768, 20.0) - 4 * 32768 / 0.02) < 1e-6


def test_traffic_table_drops_rows_whose_sources_changed(tmp_path, monkeypatch):
    tab = bench.traffic_table()
    path = os.path.join(bench.ROOT, "profiles", "ncu_dram_traffic_gqa32k_step.json")
    rows = json.load(open(path))["rows"]
    assert set(tab) <= set(rows)
    for name, v in tab.items():
        assert v == rows[name]["dram_bytes_per_launch"] > 0
    # a copy of the tree where one kernel source differs: its rows, and only those, go
    root = tmp_path / "tree"
    (root / "profiles").mkdir(parents=True)
    shutil.copy(path, root / "profiles")
    srcs = {s for r in rows.values() for s in r["sources"]}
    for s in srcs:
        dst = root / s
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, s), dst)
    changed = "top_attention_mass_b200/csrc/attn_gather.cu"
    with open(root / changed, "a") as f:
        f.write("\n// edited\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    tab2 = bench.traffic_table()
    for name, r in rows.items():
        if changed in r["sources"]:
            assert name not in tab2
        elif name in tab:
            assert tab2[name] == tab[name]
