"""fp64 CPU oracle of the attention-mass top-k path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never touches it.  The arithmetic lives in ``oracle.cpp`` (plain C++,
double precision, OpenMP over independent rows); this file only builds it and
marshals numpy arrays.

Every function here follows the method as the sources on arXiv 2606.07703
state it ("How Much Dense Attention is Necessary?", Abstract; gist.science
technical report §2.1 and §2.2); the individual readings are listed in
``oracle.cpp``.  Pins that tie it to something other than itself live in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (g++, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def build_selftest(out_dir: str) -> str:
    """Compile the stand-alone C++ self-test (selftest.cpp + oracle.cpp) into out_dir."""
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "oracle_selftest")
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", os.path.join(_HERE, "selftest.cpp"), _SRC,
           "-o", exe]
    subprocess.run(cmd, check=True)
    return exe


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            L.orc_set_mutation.argtypes = [i32]
            L.orc_set_threads.argtypes = [i32]
            L.orc_get_threads.restype = i32
            L.orc_lse_rows.argtypes = [i64, i32, i32, i32, p, p, p, i64, p]
            L.orc_mass_rows.argtypes = [i64, i32, i32, i32, p, p, p, i64, p]
            L.orc_topk_rows.argtypes = [i64, i32, i32, i32, p, p, p, i64, i32, p, p, p]
            L.orc_block_mass.argtypes = [i64, i32, i32, i32, p, p, i32, p, i64, p]
            L.orc_block_topk.argtypes = [i64, i32, i32, i32, p, p, i32, p, i64, i32, p, p, p]
            L.orc_attn_rows.argtypes = [i64, i32, i32, i32, p, p, p, p, i64, p, p, i64, p, p]
            L.orc_indexer_topk_rows.argtypes = [i64, i32, p, p, p, i64, i32, p, p, p]
            L.orc_indexer_block_mass.argtypes = [i64, i32, p, p, i32, p, i64, p]
            L.orc_indexer_block_topk.argtypes = [i64, i32, p, p, i32, p, i64, i32, p, p, p]
            L.orc_distill_kl_rows.argtypes = [i64, i32, i32, i32, p, p, i32, p, p, p, i64, p]
            L.orc_support_mass_curve.argtypes = [i64, i32, i32, i32, p, p, p, i64, p, i32, p]
            _lib = L
    return _lib


def _f32(x) -> np.ndarray:
    """Exact fp32 copy of a bf16/fp32 tensor or array (widened to fp64 inside the C++)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _rows(rows, N) -> np.ndarray:
    r = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    if r.size and (r.min() < 0 or r.max() >= N):
        raise ValueError("row out of range")
    return r


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int):
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")


def set_mutation(m: int) -> None:
    """Plant a known mistake in the oracle (0 = none); only for the oracle's own tests."""
    lib().orc_set_mutation(int(m))


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def threads() -> int:
    return int(lib().orc_get_threads())


def lse_rows(q, k, rows=None) -> np.ndarray:
    """Per-head log-sum-exp of the causal scores, [nrows, Hq] fp64."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows, N)
    out = np.zeros((len(r), Hq), np.float64)
    _check(lib().orc_lse_rows(N, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(r), len(r), _ptr(out)))
    return out


def mass_rows(q, k, rows=None) -> np.ndarray:
    """Head-averaged token mass P_i[j], [nrows, N] fp64 (zero for j > i)."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows, N)
    out = np.zeros((len(r), N), np.float64)
    _check(lib().orc_mass_rows(N, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(r), len(r), _ptr(out)))
    return out


def topk_rows(q, k, budget: int, rows=None):
    """Per-query support: (idx [n,k] int32 ascending, -1 pad; len [n]; mass [n,k] fp64)."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows, N)
    idx = np.full((len(r), budget), -1, np.int32)
    ln = np.zeros(len(r), np.int32)
    ms = np.zeros((len(r), budget), np.float64)
    _check(lib().orc_topk_rows(N, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(r), len(r), budget,
                               _ptr(idx), _ptr(ln), _ptr(ms)))
    return idx, ln, ms


def block_mass(q, k, block_q: int, blocks=None) -> np.ndarray:
    """Block mass M_b[j], [nblocks, N] fp64 (zero beyond the block's last query)."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    nb = -(-N // block_q)
    b = _rows(blocks, nb)
    out = np.zeros((len(b), N), np.float64)
    _check(lib().orc_block_mass(N, Hq, Hkv, d, _ptr(q), _ptr(k), block_q, _ptr(b), len(b),
                                _ptr(out)))
    return out


def block_topk(q, k, block_q: int, budget: int, blocks=None):
    """Block-shared support S_b: (idx [nb,k], len [nb], block mass of idx [nb,k])."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    nb = -(-N // block_q)
    b = _rows(blocks, nb)
    idx = np.full((len(b), budget), -1, np.int32)
    ln = np.zeros(len(b), np.int32)
    ms = np.zeros((len(b), budget), np.float64)
    _check(lib().orc_block_topk(N, Hq, Hkv, d, _ptr(q), _ptr(k), block_q, _ptr(b), len(b), budget,
                                _ptr(idx), _ptr(ln), _ptr(ms)))
    return idx, ln, ms


def attn_rows(q, k, v, rows=None, sup=None, sup_len=None):
    """Attention on a support (None = dense causal): (out [n,Hq,d] fp64, lse [n,Hq] fp64).

    ``sup`` is [n, kmax] int32 (one row per listed query, entries outside [0, i] or -1 are
    ignored); ``sup_len`` [n] limits how many entries of each row are read.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows, N)
    out = np.zeros((len(r), Hq, d), np.float64)
    lse = np.zeros((len(r), Hq), np.float64)
    if sup is None:
        sp, lp, stride = None, None, 0
    else:
        s = np.ascontiguousarray(sup, np.int32)
        if s.shape[0] != len(r):
            raise ValueError("one support row per listed query")
        stride = s.shape[1]
        sp = _ptr(s)
        if sup_len is None:
            lp = None
        else:
            sl = np.ascontiguousarray(sup_len, np.int32)
            lp = _ptr(sl)
    _check(lib().orc_attn_rows(N, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(v), _ptr(r), len(r), sp, lp,
                               stride, _ptr(out), _ptr(lse)))
    return out, lse


def indexer_topk_rows(q_idx, k_idx, budget: int, rows=None):
    """Indexer support: (idx [n,k] int32 ascending, -1 pad; len [n]; score [n,k] fp64)."""
    qx, kx = _f32(q_idx), _f32(k_idx)
    N, dx = qx.shape
    r = _rows(rows, N)
    idx = np.full((len(r), budget), -1, np.int32)
    ln = np.zeros(len(r), np.int32)
    sc = np.zeros((len(r), budget), np.float64)
    _check(lib().orc_indexer_topk_rows(N, dx, _ptr(qx), _ptr(kx), _ptr(r), len(r), budget,
                                       _ptr(idx), _ptr(ln), _ptr(sc)))
    return idx, ln, sc


def _blocks(blocks, N, block_q):
    return _rows(blocks, -(-N // block_q))


def indexer_block_mass(q_idx, k_idx, block_q: int, blocks=None) -> np.ndarray:
    """Block sums of the per-query softmax of indexer scores: M [nblocks, N] fp64."""
    qx, kx = _f32(q_idx), _f32(k_idx)
    N, dx = qx.shape
    b = _blocks(blocks, N, block_q)
    M = np.zeros((len(b), N), np.float64)
    _check(lib().orc_indexer_block_mass(N, dx, _ptr(qx), _ptr(kx), block_q, _ptr(b), len(b),
                                        _ptr(M)))
    return M


def indexer_block_topk(q_idx, k_idx, block_q: int, budget: int, blocks=None):
    """Block-shared indexer support: (idx [nb,k] ascending, -1 pad; len [nb]; mass [nb,k])."""
    qx, kx = _f32(q_idx), _f32(k_idx)
    N, dx = qx.shape
    b = _blocks(blocks, N, block_q)
    idx = np.full((len(b), budget), -1, np.int32)
    ln = np.zeros(len(b), np.int32)
    ms = np.zeros((len(b), budget), np.float64)
    _check(lib().orc_indexer_block_topk(N, dx, _ptr(qx), _ptr(kx), block_q, _ptr(b), len(b),
                                        budget, _ptr(idx), _ptr(ln), _ptr(ms)))
    return idx, ln, ms


def distill_kl_rows(q, k, q_idx, k_idx, rows=None) -> np.ndarray:
    """KL(P_i || softmax(q_idx_i . k_idx)) per listed row (fp64)."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    qx, kx = _f32(q_idx), _f32(k_idx)
    r = _rows(rows, N)
    kl = np.zeros(len(r), np.float64)
    _check(lib().orc_distill_kl_rows(N, Hq, Hkv, d, _ptr(q), _ptr(k), qx.shape[1], _ptr(qx),
                                     _ptr(kx), _ptr(r), len(r), _ptr(kl)))
    return kl


def support_mass_curve(q, k, budgets, rows=None) -> np.ndarray:
    """Support mass of each listed query at each budget: [n, len(budgets)] fp64."""
    q, k = _f32(q), _f32(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows, N)
    ks = np.ascontiguousarray(budgets, np.int32)
    out = np.zeros((len(r), len(ks)), np.float64)
    _check(lib().orc_support_mass_curve(N, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(r), len(r), _ptr(ks),
                                        len(ks), _ptr(out)))
    return out


def block_rows_support(block_idx, block_len, block_q: int, N: int, blocks=None):
    """Expand block supports to one support row per query (query i uses its block's S_b).

    Returns (rows, sup [n,k], sup_len [n]); the causal cut j <= i happens in attn_rows.
    """
    nb = -(-N // block_q)
    b = _rows(blocks, nb)
    rows, sups, lens = [], [], []
    for r, bb in enumerate(b):
        for i in range(bb * block_q, min(N, (bb + 1) * block_q)):
            rows.append(i)
            sups.append(block_idx[r])
            lens.append(block_len[r])
    return (np.array(rows, np.int64), np.array(sups, np.int32).reshape(len(rows), -1),
            np.array(lens, np.int32))


def sparsity(sup_sizes_per_query, N: int) -> float:
    """1 - (selected causal pairs) / (all causal pairs)."""
    total = N * (N + 1) // 2
    return 1.0 - float(np.sum(sup_sizes_per_query)) / total


# ------------------------------------------------------------------ packed batches
# A packed batch holds independent causal sequences back to back along the token
# axis (sequence s owns tokens [cu[s], cu[s+1])); every quantity above is computed
# per sequence on its own slice, positions restarting at 0.


def seq_slices(cu_seqlens):
    cu = np.asarray(cu_seqlens, np.int64)
    if cu.ndim != 1 or cu.size < 2 or cu[0] != 0 or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens: [n_seq + 1], starts at 0, non-decreasing")
    return [(int(cu[s]), int(cu[s + 1])) for s in range(cu.size - 1)]


def varlen_mass_packed(q, k, cu_seqlens) -> np.ndarray:
    """Head-averaged mass of every packed query over the packed keys, [T, T] fp64
    (zero outside the query's own sequence and causal prefix)."""
    q, k = _f32(q), _f32(k)
    T = q.shape[0]
    P = np.zeros((T, T), np.float64)
    for t0, t1 in seq_slices(cu_seqlens):
        if t1 > t0:
            P[t0:t1, t0:t1] = mass_rows(q[t0:t1], k[t0:t1])
    return P


def varlen_support(q, k, cu_seqlens, budget: int, block_q: int = 1):
    """Support of every sequence (per query, or per block of block_q queries), rows
    packed in sequence order, key indices local to the sequence:
    (idx [n_sel, k] int32 ascending, -1 pad; len [n_sel]; value [n_sel, k] fp64)."""
    q, k = _f32(q), _f32(k)
    parts = []
    for t0, t1 in seq_slices(cu_seqlens):
        if t1 == t0:
            continue
        if block_q == 1:
            parts.append(topk_rows(q[t0:t1], k[t0:t1], budget))
        else:
            parts.append(block_topk(q[t0:t1], k[t0:t1], block_q, budget))
    if not parts:
        return (np.zeros((0, budget), np.int32), np.zeros(0, np.int32),
                np.zeros((0, budget), np.float64))
    return tuple(np.concatenate([p[c] for p in parts]) for c in range(3))


def varlen_attn(q, k, v, cu_seqlens, sup=None, sup_len=None, block_q: int = 1):
    """Attention of every packed query on its sequence (sup None: dense causal; else
    the packed support rows as varlen_support lays them out, block rows expanded to
    their queries): (out [T, Hq, d] fp64, lse [T, Hq] fp64)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    T, Hq, d = q.shape
    out = np.zeros((T, Hq, d), np.float64)
    lse = np.zeros((T, Hq), np.float64)
    sel0 = 0
    for t0, t1 in seq_slices(cu_seqlens):
        n = t1 - t0
        if n == 0:
            continue
        n_sel = n if block_q == 1 else -(-n // block_q)
        if sup is None:
            o, l = attn_rows(q[t0:t1], k[t0:t1], v[t0:t1])
        else:
            si = np.asarray(sup)[sel0:sel0 + n_sel]
            sl = np.asarray(sup_len)[sel0:sel0 + n_sel]
            if block_q == 1:
                o, l = attn_rows(q[t0:t1], k[t0:t1], v[t0:t1], sup=si, sup_len=sl)
            else:
                r, s, ln = block_rows_support(si, sl, block_q, n)
                o, l = attn_rows(q[t0:t1], k[t0:t1], v[t0:t1], r, sup=s, sup_len=ln)
        out[t0:t1], lse[t0:t1] = o, l
        sel0 += n_sel
    return out, lse


def varlen_indexer_support(q_idx, k_idx, cu_seqlens, budget: int, block_q: int = 1):
    """Indexer support of every sequence of a packed batch (per query, or block-shared
    over block_q queries), rows packed in sequence order, key indices local:
    (idx [n_sel, k] int32 ascending, -1 pad; len [n_sel]; value [n_sel, k] fp64)."""
    qx, kx = _f32(q_idx), _f32(k_idx)
    parts = []
    for t0, t1 in seq_slices(cu_seqlens):
        if t1 == t0:
            continue
        if block_q == 1:
            parts.append(indexer_topk_rows(qx[t0:t1], kx[t0:t1], budget))
        else:
            parts.append(indexer_block_topk(qx[t0:t1], kx[t0:t1], block_q, budget))
    if not parts:
        return (np.zeros((0, budget), np.int32), np.zeros(0, np.int32),
                np.zeros((0, budget), np.float64))
    return tuple(np.concatenate([p[c] for p in parts]) for c in range(3))
