"""The oracle's stand-alone C++ self-test (oracle/selftest.cpp), built with g++
against oracle.cpp and run as a binary: direct evaluation of the mass, the
support rule, nesting and monotonicity in k, block of one, k >= i+1 = dense, and
the Q = 0 closed form."""
import subprocess


def test_oracle_selftest_binary(tmp_path):
    import oracle
    exe = oracle.build_selftest(str(tmp_path))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all passed" in r.stdout
    # each planted mistake (dropped scale, interleaved head map, sum for mean, reversed
    # tie rule) makes the binary fail
    for m in (1, 2, 3, 4):
        r = subprocess.run([exe, str(m)], capture_output=True, text=True, timeout=120)
        assert r.returncode == 1 and "FAILED" in r.stdout, m
