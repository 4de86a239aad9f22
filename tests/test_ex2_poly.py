"""The FMA-pipe exponential of the kernels (csrc/tc_ptx.cuh, ex2_fma / ex2_fma2) against
the mathematics: its coefficients are read from the header and the same steps are
replayed in float32 (round to nearest integer by adding 1.5 * 2^23, degree-4 Horner
polynomial in f in [-0.5, 0.5], integer added to the exponent field, 0 below -125),
then compared with 2^x in float64.  The bound is the one the header states (2.7e-6
relative)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "top_attention_mass_b200", "csrc", "tc_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    val = {}
    for name in ("kEx2C0", "kEx2C1", "kEx2C2", "kEx2C3", "kEx2C4", "kRoundMagic"):
        m = re.search(name + r"\s*=\s*([0-9.]+)f", src)
        val[name] = float(m.group(1))
    assert val["kRoundMagic"] == 12582912.0
    return tuple(np.float32(val[f"kEx2C{i}"]) for i in range(5))


def _ex2_fma(x0):
    c0, c1, c2, c3, c4 = _coeffs()
    x0 = x0.astype(np.float32)
    x = np.maximum(x0, np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    p = (c4 * f + c3).astype(np.float32)
    p = (p * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    y = (p.view(np.int32) + (n << 23)).view(np.float32)
    return np.where(x0 < np.float32(-125.0), np.float32(0.0), y)


def test_relative_error_over_the_used_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001, dtype=np.float32),
                        -np.float32(2.0) ** -np.arange(1, 40, dtype=np.float32)])
    y = _ex2_fma(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2.8e-6


def test_exact_at_integers_within_the_bound_and_zero_below_the_clamp():
    x = np.arange(-125, 1, dtype=np.float32)
    y = _ex2_fma(x).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) < 2.8e-6)
    # a masked score (-inf) and anything below -125 give exactly 0, as ex2.approx.ftz does
    lo = _ex2_fma(np.array([-125.5, -126.0, -300.0, -np.inf], dtype=np.float32))
    assert np.all(lo == 0.0)
