"""Seeded synthetic inputs for the attention-mass top-k path.

This module only draws and shapes inputs: it holds none of the method's
arithmetic (no scores, no softmax, no mass, no selection).  Both the oracle
tests and the CUDA parity tests / benchmark take their inputs from here.

Workloads follow the configurations of the benchmark description:

* ``tiny_fp32``      N=512,  Hq=4,  Hkv=1, d=64,  fp32, k=32 per query; key 0 scaled x4 (sink)
* ``gqa4k_needles``  N=4096, Hq=32, Hkv=8, d=128, bf16, k=256 per query; 16 planted needles
* ``gqa32k_2pct``    N=32768, Hq=32, Hkv=8, d=128, bf16, k=655 per query and block-shared B_q=64;
                     sink at token 0, 64 planted needles
* ``longctx_<N>``    N in {4096,16384,32768,65536,102400}, Hq=16, Hkv=4, d=128, bf16, k=2048,
                     block-shared B_q=128; RoPE (base 1e6) on Q and K, sink, needles every N/32
* ``indexer32k``     the gqa32k_2pct tensors plus one head-collapsed indexer head (d_idx=64):
                     q_idx, k_idx = bf16(Q_flat W_q), bf16(K_flat W_k), W ~ N(0, 1/(128*32)); k=1024

The public evaluation suites the paper reports on (RULER, VideoMME,
MMLongBench-Doc, LongBench-v2) are not reproduced here; these synthetic
tensors only stand in for their shapes: 4K-100K contexts, ~2 % budgets and
retrieval-style "needle" structure.

Recipe (numpy ``default_rng(seed)``, seed 0 unless stated):
  1. draw fp32 N(0,1) Q [N,Hq,d], then K [N,Hkv,d], then V [N,Hkv,d];
  2. RoPE (rotate-half layout, theta_c = base^(-2c/d), positions 0..N-1) on Q and K, if asked;
  3. sink: K[0] *= 4, if asked;
  4. needles: positions drawn from the same generator after V (random needles), or on a fixed
     grid (grid needles); for every KV group g the needle key K[j*, g] gets
     3*sqrt(d)*qbar/|qbar| added, qbar = mean of Q[i*, h] over the query heads h of group g
     (consecutive query heads share a KV head);
  5. cast to the storage dtype (round-to-nearest-even for bf16).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    Hq: int
    Hkv: int
    d: int
    dtype: str                 # "bf16" or "f32"
    budget_k: int
    block_q: tuple             # supports to build: 1 = per query, >1 = block-shared
    sink: bool = False
    needles: int = 0           # random needles (count)
    grid_needles: bool = False # needles at j*_m = m*N/32, i*_m = j*_m + N/64
    rope_base: Optional[float] = None
    d_idx: int = 0             # indexer head width (0 = no indexer)
    seed: int = 0

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


LONGCTX_NS = (4096, 16384, 32768, 65536, 102400)

WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 512, 4, 1, 64, "f32", 32, (1,), sink=True),
    "gqa4k_needles": Workload("gqa4k_needles", 4096, 32, 8, 128, "bf16", 256, (1,), needles=16),
    "gqa32k_2pct": Workload("gqa32k_2pct", 32768, 32, 8, 128, "bf16", 655, (1, 64),
                            sink=True, needles=64),
    "indexer32k": Workload("indexer32k", 32768, 32, 8, 128, "bf16", 1024, (1,),
                           sink=True, needles=64, d_idx=64),
}
for _n in LONGCTX_NS:
    WORKLOADS[f"longctx_{_n}"] = Workload(f"longctx_{_n}", _n, 16, 4, 128, "bf16", 2048, (128,),
                                          sink=True, grid_needles=True, rope_base=1e6)


def custom(name: str, N: int, Hq: int, Hkv: int, d: int, dtype: str = "bf16", budget_k: int = 8,
           block_q: tuple = (1,), seed: int = 0, **kw) -> Workload:
    """A workload of arbitrary small shape (parity and edge-case tests)."""
    return Workload(name, N, Hq, Hkv, d, dtype, budget_k, block_q, seed=seed, **kw)


@dataclass
class Inputs:
    w: Workload
    q: torch.Tensor            # [N,Hq,d] storage dtype, CPU
    k: torch.Tensor            # [N,Hkv,d]
    v: torch.Tensor            # [N,Hkv,d]
    needle_j: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    needle_i: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    q_idx: Optional[torch.Tensor] = None   # [N,d_idx] bf16
    k_idx: Optional[torch.Tensor] = None   # [N,d_idx] bf16


def _rope_rotate_half(x: np.ndarray, base: float) -> np.ndarray:
    """Rotary position embedding, rotate-half layout, positions 0..N-1 (fp32)."""
    N, _, d = x.shape
    half = d // 2
    c = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * c / d)
    ang = np.arange(N, dtype=np.float64)[:, None] * theta[None, :]
    cos = np.cos(ang).astype(np.float32)[:, None, :]
    sin = np.sin(ang).astype(np.float32)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1).astype(np.float32)


def _plant(q: np.ndarray, k: np.ndarray, js, is_, G: int) -> None:
    d = q.shape[2]
    Hkv = k.shape[1]
    for j, i in zip(js, is_):
        for g in range(Hkv):
            qbar = q[i, g * G:(g + 1) * G, :].astype(np.float64).mean(axis=0)
            nrm = np.linalg.norm(qbar)
            if nrm > 0:
                k[j, g, :] += (3.0 * math.sqrt(d) * qbar / nrm).astype(np.float32)


def _to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


def make_inputs(w: Workload, N: Optional[int] = None) -> Inputs:
    """Draw the seeded tensors of workload ``w`` (optionally overriding N)."""
    if N is not None and N != w.N:
        w = Workload(**{**w.__dict__, "N": N})
    rng = np.random.default_rng(w.seed)
    N, Hq, Hkv, d = w.N, w.Hq, w.Hkv, w.d
    q = rng.standard_normal((N, Hq, d), dtype=np.float32)
    k = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    v = rng.standard_normal((N, Hkv, d), dtype=np.float32)
    if w.rope_base is not None:
        q = _rope_rotate_half(q, w.rope_base)
        k = _rope_rotate_half(k, w.rope_base)
    if w.sink:
        k[0] *= 4.0
    nj = np.zeros(0, np.int64)
    ni = np.zeros(0, np.int64)
    if w.needles and N >= 4:
        m = min(w.needles, N - 2)
        nj = np.sort(rng.choice(np.arange(1, N - 1), size=m, replace=False)).astype(np.int64)
        ni = np.array([rng.integers(j + 1, N) for j in nj], dtype=np.int64)
    elif w.grid_needles and N >= 64:
        nj = np.array([m * N // 32 for m in range(1, 32)], dtype=np.int64)
        ni = np.minimum(nj + N // 64, N - 1)
    if len(nj):
        _plant(q, k, nj, ni, w.group)
    inp = Inputs(w, _to_storage(q, w.dtype), _to_storage(k, w.dtype), _to_storage(v, w.dtype),
                 nj, ni)
    if w.d_idx:
        inp.q_idx, inp.k_idx = indexer_projections(inp, w.d_idx, seed=w.seed + 1)
    return inp


def indexer_projections(inp: Inputs, d_idx: int, seed: int = 1):
    """Random Gaussian head-collapsed projections of the head-concatenated Q and K.

    W_q [Hq*d, d_idx] and W_k [Hkv*d, d_idx] are drawn N(0, std=1/sqrt(128*32)) from
    ``default_rng(seed)`` in that order; the products run in fp32 and are rounded to bf16.
    """
    N, Hq, d = inp.q.shape
    Hkv = inp.k.shape[1]
    rng = np.random.default_rng(seed)
    std = 1.0 / math.sqrt(128 * 32)
    wq = torch.from_numpy(rng.standard_normal((Hq * d, d_idx), dtype=np.float32) * np.float32(std))
    wk = torch.from_numpy(rng.standard_normal((Hkv * d, d_idx), dtype=np.float32) * np.float32(std))
    qf = inp.q.float().reshape(N, Hq * d)
    kf = inp.k.float().reshape(N, Hkv * d)
    return (qf @ wq).to(torch.bfloat16).contiguous(), (kf @ wk).to(torch.bfloat16).contiguous()


def stress_support(N: int, budget_k: int, seed: int = 7, rows=None):
    """Uniform-random support: min(k, i+1) distinct indices from [0, i], sorted ascending.

    Returns (idx [n,k] int32, -1 padded; len [n] int32) for the given rows (default all).
    """
    rng = np.random.default_rng(seed)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    idx = np.full((len(rows), budget_k), -1, np.int32)
    ln = np.zeros(len(rows), np.int32)
    for r, i in enumerate(rows):
        n = min(budget_k, int(i) + 1)
        if n == int(i) + 1:
            sel = np.arange(n)
        else:
            sel = np.sort(rng.choice(int(i) + 1, size=n, replace=False))
        idx[r, :n] = sel
        ln[r] = n
    return idx, ln


def stratified_support(N: int, budget_k: int, seed: int = 7, device="cpu"):
    """A random support for timing runs at large N, drawn in bulk with torch: row i keeps
    every key when i + 1 <= k, else one uniform key from each of the k strata
    [floor(t (i+1) / k), floor((t+1) (i+1) / k)), t = 0..k-1 (distinct, ascending).
    Returns (idx [N,k] int32, -1 padded; len [N] int32) on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    idx = torch.empty(N, budget_k, dtype=torch.int32, device=device)
    ln = torch.clamp(torch.arange(1, N + 1, device=device), max=budget_k).to(torch.int32)
    t = torch.arange(budget_k, device=device, dtype=torch.int64)
    chunk = max(1, (1 << 24) // budget_k)
    for r0 in range(0, N, chunk):
        i = torch.arange(r0, min(N, r0 + chunk), device=device, dtype=torch.int64)[:, None]
        n = i + 1
        lo = (t[None, :] * n) // budget_k
        hi = ((t[None, :] + 1) * n) // budget_k
        u = torch.rand(lo.shape, generator=g, device=device, dtype=torch.float64)
        sel = lo + torch.floor(u * (hi - lo)).to(torch.int64)
        full = n <= budget_k
        sel = torch.where(full, t[None, :].expand_as(sel), sel)
        sel = torch.where(t[None, :] < n, sel, torch.full_like(sel, -1))
        idx[r0:r0 + len(i)] = sel.to(torch.int32)
    return idx, ln


def sample_rows(N: int, needle_i=(), n_random: int = 256, seed: int = 11) -> np.ndarray:
    """Rows checked at large N: first and last 64, every needle's query, seeded random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(64, N))) | set(range(max(0, N - 64), N)) | {int(i) for i in needle_i}
    rows |= {int(x) for x in rng.integers(0, N, size=min(n_random, N))}
    return np.array(sorted(rows), dtype=np.int64)


def sample_blocks(n_blocks: int, n: int = 16, seed: int = 13) -> np.ndarray:
    """Blocks checked at large N: first, last and seeded random ones (n in total)."""
    rng = np.random.default_rng(seed)
    s = {0, n_blocks - 1}
    while len(s) < min(n, n_blocks):
        s.add(int(rng.integers(0, n_blocks)))
    return np.array(sorted(s), dtype=np.int64)
