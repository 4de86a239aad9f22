"""Comparison rules between the CUDA path and the fp64 oracle.

Rules (from the project's statement of the method's tolerances):
* support indices: identical, except that every index in the symmetric difference
  has oracle value within REL_TIE * m_k of m_k, the oracle's k-th largest value;
  rows are ascending and padded with -1; lengths identical (they are min(k, i+1));
* head-averaged mass: |gpu - oracle| <= 1e-4 absolute per selected entry (the
  oracle value is looked up at the GPU's index); block mass sums up to block_q
  rows, so its bound is 1e-4 per summed row;
* outputs: max-abs error <= 2e-2 for bf16 inputs, 1e-4 for fp32 inputs, against
  the oracle recomputed on the GPU's own support (pass 3 alone) - which equals the
  end-to-end comparison on every row whose support matches the oracle's exactly;
* per-head LSE: <= 1e-3 absolute (fp32 accumulation of up to 1e5 terms).
"""
import numpy as np

REL_TIE = 1e-3
MASS_ATOL = 1e-4
OUT_ATOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_ATOL = 1e-3
# KL per query: fp32 sums over up to 1e5 keys of P log P and P t, plus a log-sum-exp;
# the probabilities carry ~3e-6 relative error (exp2 approximations), which moves the
# sums by ~1e-5 per unit of entropy: 2e-3 absolute leaves an order of magnitude.
KL_ATOL = 2e-3


def check_support(gpu_idx, gpu_len, gpu_val, ora_idx, ora_len, ora_rows, val_atol=MASS_ATOL,
                  name="support"):
    """Compare supports row by row.  ora_rows[r] is the oracle's full value row (mass,
    block mass or indexer score) for the same row/block.  Returns the number of rows
    whose sets differ (all differences being near-ties)."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_len = np.asarray(gpu_len)
    gpu_val = np.asarray(gpu_val, dtype=np.float64)
    n_diff_rows = 0
    for r in range(len(ora_len)):
        n = int(ora_len[r])
        assert int(gpu_len[r]) == n, f"{name} row {r}: len {gpu_len[r]} != {n}"
        gi = gpu_idx[r, :n]
        assert np.all(gpu_idx[r, n:] == -1), f"{name} row {r}: padding"
        assert np.all(np.diff(gi) > 0), f"{name} row {r}: not strictly ascending"
        oi = ora_idx[r, :n]
        row = ora_rows[r]
        m_k = row[oi].min() if n else 0.0
        diff = set(gi.tolist()) ^ set(oi.tolist())
        if diff:
            n_diff_rows += 1
            for j in diff:
                assert abs(row[j] - m_k) <= REL_TIE * abs(m_k), (
                    f"{name} row {r}: index {j} value {row[j]!r} is not a near-tie of "
                    f"m_k={m_k!r}")
        err = np.abs(gpu_val[r, :n] - row[gi])
        assert err.max(initial=0.0) <= val_atol, f"{name} row {r}: value err {err.max()}"
        assert np.all(gpu_val[r, n:] == 0)
    return n_diff_rows


def check_close(gpu, ref, atol, name):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    finite = np.isfinite(ref)
    assert np.array_equal(np.isfinite(gpu), finite), f"{name}: non-finite pattern differs"
    err = np.abs(gpu[finite] - ref[finite])
    mx = float(err.max(initial=0.0))
    assert mx <= atol, f"{name}: max abs err {mx} > {atol}"
    return mx
