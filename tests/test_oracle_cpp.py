"""The oracle's stand-alone C++ self-test (oracle/selftest.cpp), built with g++
against oracle.cpp and run as a binary: direct evaluation of the mass, the
support rule, nesting and monotonicity in k, block of one, k >= i+1 = dense, and
the Q = 0 closed form."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_selftest_binary(tmp_path):
    exe = str(tmp_path / "oracle_selftest")
    src = [os.path.join(ROOT, "oracle", "selftest.cpp"), os.path.join(ROOT, "oracle", "oracle.cpp")]
    subprocess.run(["g++", "-O2", "-std=c++17", "-fopenmp", *src, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all passed" in r.stdout
    # each planted mistake (dropped scale, interleaved head map, sum for mean, reversed
    # tie rule) makes the binary fail
    for m in (1, 2, 3, 4):
        r = subprocess.run([exe, str(m)], capture_output=True, text=True, timeout=120)
        assert r.returncode == 1 and "FAILED" in r.stdout, m
