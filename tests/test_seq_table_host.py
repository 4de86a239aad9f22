"""The packed-batch tile order of csrc/launch.h, checked on the host: the table's
ordering and first-tile offsets, and the decoder every table-driven kernel runs per CTA,
compiled with g++ against the same header (tests/host/seq_table_check.cpp)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda_runtime.h")):
            return os.path.join(cand, "include")
    return None


def test_tile_order_is_a_bijection_longest_sequence_first(tmp_path):
    inc = _cuda_include()
    gxx = shutil.which("g++")
    if inc is None or gxx is None:
        pytest.skip("needs g++ and the CUDA headers")
    exe = str(tmp_path / "seq_table_check")
    src = os.path.join(ROOT, "tests", "host", "seq_table_check.cpp")
    csrc = os.path.join(ROOT, "top_attention_mass_b200", "csrc")
    r = subprocess.run([gxx, "-O2", "-std=c++17", "-I", csrc, "-I", inc, src, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
