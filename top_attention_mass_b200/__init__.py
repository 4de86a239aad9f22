"""Python binding of libtam.so: the B200 attention-mass top-k path.

Thin ctypes marshalling over the C ABI declared in ``include/tam.h``; every
step of the path runs in the library's CUDA kernels.  PyTorch only provides
device memory (output tensors, the workspace) and the current CUDA stream.
There is no CPU path: if ``libtam.so`` has not been built, or there is no CUDA
device, every call raises.

Functions (same names as the C entry points, without the ``tam_`` prefix):

* ``mass_oracle_prefill``      passes 1-3 of the attention-mass top-k oracle
* ``attention_lse``            pass 1 alone (per-head log-sum-exp)
* ``mass_select``              pass 2 alone (mass + top-k support, given pass 1's lse)
* ``indexer_topk``             head-collapsed indexer support
* ``sparse_support_attention`` pass 3 alone (attention on a given support)
* ``dense_gqa_prefill``        dense causal GQA attention (comparator)
* ``mass_oracle_prefill_varlen``, ``dense_gqa_prefill_varlen``, ``indexer_topk_varlen``,
  ``sparse_support_attention_varlen``
                               the same over a packed batch of sequences

Inputs may be CUDA tensors, or CPU tensors (ideally pinned): then they are
copied to ``device``, the call runs there, and the results come back to the CPU.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# TAM_LIBRARY=debug loads the debug-checks build (pass-2 stores checked against their
# extents; see tam.h, TAM_ERR_OVERFLOW) instead of the release library
LIB_PATH = os.path.join(_HERE, "libtam_debug.so" if os.environ.get("TAM_LIBRARY") == "debug"
                        else "libtam.so")

TAM_OK, TAM_ERR_INVALID_ARG, TAM_ERR_UNSUPPORTED, TAM_ERR_WORKSPACE = 0, 1, 2, 3
TAM_ERR_CUDA, TAM_ERR_TIMEOUT, TAM_ERR_OVERFLOW = 4, 5, 6
TAM_BF16, TAM_F32 = 0, 1

EXPORTED = (
    "tam_version", "tam_status_string", "tam_mass_oracle_workspace", "tam_mass_workspace_min",
    "tam_mass_oracle_prefill", "tam_attention_lse_workspace", "tam_attention_lse",
    "tam_mass_select_workspace", "tam_mass_select", "tam_mass_select_noalloc",
    "tam_indexer_workspace", "tam_indexer_workspace_min", "tam_indexer_topk",
    "tam_distill_kl_workspace", "tam_distill_kl_workspace_min", "tam_distill_kl",
    "tam_support_mass_curve", "tam_sparse_attention_workspace", "tam_sparse_support_attention",
    "tam_dense_workspace", "tam_dense_gqa_prefill", "tam_kernel_launches", "tam_check_status",
    "tam_mass_oracle_workspace_varlen", "tam_mass_oracle_prefill_varlen",
    "tam_dense_gqa_prefill_varlen", "tam_indexer_workspace_varlen", "tam_indexer_topk_varlen",
    "tam_sparse_support_attention_varlen", "tam_mass_fallback_rows", "tam_indexer_fallback_rows",
)


class TamError(RuntimeError):
    def __init__(self, code: int, where: str, detail=None):
        self.code = code
        self.detail = detail
        msg = f"{where}: {status_string(code)} ({code})"
        if detail is not None:
            msg += f" detail={list(detail)}"
        super().__init__(msg)


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libtam.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m top_attention_mass_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, sz, p = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        L.tam_version.restype = i32
        L.tam_status_string.restype = ctypes.c_char_p
        L.tam_status_string.argtypes = [i32]
        L.tam_mass_oracle_workspace.restype = sz
        L.tam_mass_oracle_workspace.argtypes = [i64, i32, i32, i32, i32, i32, i32]
        L.tam_mass_workspace_min.restype = sz
        L.tam_mass_workspace_min.argtypes = [i64, i32, i32, i32, i32, i32, i32]
        L.tam_mass_oracle_prefill.restype = i32
        L.tam_mass_oracle_prefill.argtypes = [i64, i32, i32, i32, i32, p, p, p, i32, i32, p, p, p,
                                              p, p, p, sz, p]
        L.tam_attention_lse_workspace.restype = sz
        L.tam_attention_lse_workspace.argtypes = [i64, i32, i32, i32, i32]
        L.tam_attention_lse.restype = i32
        L.tam_attention_lse.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, sz, p]
        L.tam_mass_select_workspace.restype = sz
        L.tam_mass_select_workspace.argtypes = [i64, i32, i32, i32, i32, i32, i32]
        L.tam_mass_select.restype = i32
        L.tam_mass_select.argtypes = [i64, i32, i32, i32, i32, p, p, p, i32, i32, p, p, p, p, sz,
                                      p]
        L.tam_mass_select_noalloc.restype = i32
        L.tam_mass_select_noalloc.argtypes = [i64, i32, i32, i32, i32, p, p, p, i32, i32, p, p, p,
                                              p]
        L.tam_indexer_workspace.restype = sz
        L.tam_indexer_workspace.argtypes = [i64, i32, i32, i32, i32]
        L.tam_indexer_workspace_min.restype = sz
        L.tam_indexer_workspace_min.argtypes = [i64, i32, i32, i32, i32]
        L.tam_indexer_topk.restype = i32
        L.tam_indexer_topk.argtypes = [i64, i32, i32, p, p, i32, i32, p, p, p, p, sz, p]
        L.tam_distill_kl_workspace.restype = sz
        L.tam_distill_kl_workspace.argtypes = [i64, i32, i32, i32, i32, i32]
        L.tam_distill_kl_workspace_min.restype = sz
        L.tam_distill_kl_workspace_min.argtypes = [i64, i32, i32, i32, i32, i32]
        L.tam_distill_kl.restype = i32
        L.tam_distill_kl.argtypes = [i64, i32, i32, i32, i32, p, p, p, i32, p, p, p, p, sz, p]
        L.tam_support_mass_curve.restype = i32
        L.tam_support_mass_curve.argtypes = [i64, i32, p, p, p, i32, p, p]
        L.tam_sparse_attention_workspace.restype = sz
        L.tam_sparse_attention_workspace.argtypes = [i64, i32, i32, i32, i32]
        L.tam_sparse_support_attention.restype = i32
        L.tam_sparse_support_attention.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, i32,
                                                   i32, p, p, p, sz, p]
        L.tam_dense_workspace.restype = sz
        L.tam_dense_workspace.argtypes = [i64, i32, i32, i32, i32]
        L.tam_dense_gqa_prefill.restype = i32
        L.tam_dense_gqa_prefill.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, sz, p]
        L.tam_mass_oracle_workspace_varlen.restype = sz
        L.tam_mass_oracle_workspace_varlen.argtypes = [i32, p, i32, i32, i32, i32, i32, i32]
        L.tam_mass_oracle_prefill_varlen.restype = i32
        L.tam_mass_oracle_prefill_varlen.argtypes = [i32, p, i32, i32, i32, i32, p, p, p, i32, i32,
                                                     p, p, p, p, p, p, sz, p]
        L.tam_dense_gqa_prefill_varlen.restype = i32
        L.tam_dense_gqa_prefill_varlen.argtypes = [i32, p, i32, i32, i32, i32, p, p, p, p, p, p,
                                                   sz, p]
        L.tam_indexer_workspace_varlen.restype = sz
        L.tam_indexer_workspace_varlen.argtypes = [i32, p, i32, i32, i32, i32]
        L.tam_indexer_topk_varlen.restype = i32
        L.tam_indexer_topk_varlen.argtypes = [i32, p, i32, i32, p, p, i32, i32, p, p, p, p, sz, p]
        L.tam_sparse_support_attention_varlen.restype = i32
        L.tam_sparse_support_attention_varlen.argtypes = [i32, p, i32, i32, i32, i32, p, p, p, p, p,
                                                          i32, i32, p, p, p, sz, p]
        L.tam_mass_fallback_rows.restype = i64
        L.tam_mass_fallback_rows.argtypes = [i64, i32, i32, i32, i32, i32, p, p]
        L.tam_indexer_fallback_rows.restype = i64
        L.tam_indexer_fallback_rows.argtypes = [i64, i32, i32, i32, p, p]
        L.tam_kernel_launches.restype = ctypes.c_uint64
        L.tam_check_status.restype = i32
        L.tam_check_status.argtypes = [p, p, p]
        _lib = L
        return _lib


def status_string(code: int) -> str:
    try:
        return lib().tam_status_string(int(code)).decode()
    except Exception:
        return "status"


def version() -> int:
    return int(lib().tam_version())


def kernel_launches() -> int:
    """Kernels this library has launched in this process (all entry points)."""
    return int(lib().tam_kernel_launches())


def mass_fallback_rows(q, k, budget_k: int, workspace, stream=None) -> int:
    """Rows of the last per-query mass selection in `workspace` (a Workspace or the
    uint8 tensor a call used) that went to the fallback path; -1 if it does not stream."""
    N, Hq, Hkv, d = _shape(q, k)
    t = workspace.get(256) if isinstance(workspace, Workspace) else workspace
    return int(lib().tam_mass_fallback_rows(N, Hq, Hkv, d, _dtype_code(q), budget_k, _ptr(t),
                                            _stream(t.device, stream)))


def indexer_fallback_rows(q_idx, budget_k: int, workspace, stream=None) -> int:
    """As mass_fallback_rows, for the last per-query indexer selection."""
    N, dx = q_idx.shape
    t = workspace.get(256) if isinstance(workspace, Workspace) else workspace
    return int(lib().tam_indexer_fallback_rows(N, dx, _dtype_code(q_idx), budget_k, _ptr(t),
                                               _stream(t.device, stream)))


# ------------------------------------------------------------------ marshalling helpers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TAM_BF16
    if t.dtype == torch.float32:
        return TAM_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


class Workspace:
    """A reusable device workspace (uint8 tensor) that grows on demand.

    A call that gets no workspace uses one default workspace per device.  Calls are
    ordered on their stream, so that is safe for one stream at a time; calls that run
    concurrently on several streams need one Workspace each (the status block and the
    scratch would otherwise be shared)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = {}


def _workspace(device: torch.device, nbytes: int, ws: Optional[Workspace]) -> torch.Tensor:
    if ws is None:
        key = (device.type, device.index)
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(device)
    return ws.get(nbytes)


def _raise(rc: int, where: str):
    if rc != TAM_OK:
        raise TamError(rc, where)


def check_status(workspace: torch.Tensor, stream=None):
    """Wait for the stream and raise if the last call on this workspace flagged an error."""
    detail = (ctypes.c_int32 * 8)()
    rc = lib().tam_check_status(_ptr(workspace), _stream(workspace.device, stream), detail)
    if rc != TAM_OK:
        raise TamError(rc, "device status", list(detail))


def _to_device(ts, device):
    """Move CPU inputs to `device` (non-blocking from pinned memory); CUDA inputs pass through."""
    out, host = [], False
    for t in ts:
        if t is None:
            out.append(None)
        elif t.is_cuda:
            out.append(t.contiguous())
        else:
            host = True
            out.append(t.contiguous().to(device, non_blocking=t.is_pinned()))
    return out, host


def _dev_of(t: torch.Tensor, device) -> torch.device:
    if t.is_cuda:
        return t.device
    return torch.device(device or "cuda")


def _shape(q: torch.Tensor, k: torch.Tensor):
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q is [N, Hq, d] and k, v are [N, Hkv, d]")
    N, Hq, d = q.shape
    if k.shape[0] != N or k.shape[2] != d or k.dtype != q.dtype:
        raise ValueError("k must be [N, Hkv, d] with q's N, d and dtype")
    return N, Hq, k.shape[1], d


# ------------------------------------------------------------------ entry points

@dataclass
class Support:
    idx: torch.Tensor             # [n_sel, k] int32 ascending, -1 padded
    length: torch.Tensor          # [n_sel] int32
    value: torch.Tensor           # [n_sel, k] fp32: mass (oracle) or score (indexer)
    lse: Optional[torch.Tensor] = None    # [Hq, N] fp32
    out: Optional[torch.Tensor] = None    # [N, Hq, d]


def mass_oracle_prefill(q, k, v=None, budget_k: int = 1, block_q: int = 1, *,
                        compute_out: bool = True, return_lse: bool = True,
                        workspace: Optional[Workspace] = None, stream=None, check: bool = True,
                        device=None, workspace_bytes: Optional[int] = None) -> Support:
    """Attention-mass top-k oracle (passes 1-3) for one causal GQA prefill layer.

    workspace_bytes: pass this many workspace bytes instead of the preferred size
    (at least tam_mass_workspace_min; a smaller workspace only means more chunks)."""
    dev = _dev_of(q, device)
    (q, k, v), host = _to_device([q, k, v], dev)
    N, Hq, Hkv, d = _shape(q, k)
    if compute_out and v is None:
        raise ValueError("v is needed for the recomputed output")
    dt = _dtype_code(q)
    n_sel = N if block_q == 1 else -(-N // block_q)
    sup_idx = torch.empty(n_sel, budget_k, dtype=torch.int32, device=dev)
    sup_len = torch.empty(n_sel, dtype=torch.int32, device=dev)
    sup_mass = torch.empty(n_sel, budget_k, dtype=torch.float32, device=dev)
    lse = torch.empty(Hq, N, dtype=torch.float32, device=dev) if return_lse else None
    out = torch.empty_like(q) if compute_out else None
    L = lib()
    nbytes = L.tam_mass_oracle_workspace(N, Hq, Hkv, d, dt, budget_k, block_q)
    if nbytes == 0:
        _raise(L.tam_mass_oracle_prefill(N, Hq, Hkv, d, dt, None, None, None, budget_k, block_q,
                                         None, None, None, None, None, None, 0, None),
               "mass_oracle_prefill")
    if workspace_bytes is not None:
        nbytes = int(workspace_bytes)
    ws = _workspace(dev, nbytes, workspace)
    rc = L.tam_mass_oracle_prefill(N, Hq, Hkv, d, dt, _ptr(q), _ptr(k), _ptr(v), budget_k, block_q,
                                   _ptr(sup_idx), _ptr(sup_len), _ptr(sup_mass), _ptr(lse),
                                   _ptr(out), _ptr(ws), min(ws.numel(), nbytes),
                                   _stream(dev, stream))
    _raise(rc, "mass_oracle_prefill")
    if check:
        check_status(ws, stream)
    res = Support(sup_idx, sup_len, sup_mass, lse, out)
    if host:
        res = Support(*[None if t is None else t.cpu() for t in
                        (res.idx, res.length, res.value, res.lse, res.out)])
    return res


def attention_lse(q, k, *, workspace: Optional[Workspace] = None, stream=None,
                  check: bool = True) -> torch.Tensor:
    """Pass 1: per-head log-sum-exp of the causal scores, [Hq, N] fp32."""
    dev = q.device
    N, Hq, Hkv, d = _shape(q, k)
    dt = _dtype_code(q)
    lse = torch.empty(Hq, N, dtype=torch.float32, device=dev)
    L = lib()
    nbytes = L.tam_attention_lse_workspace(N, Hq, Hkv, d, dt)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_attention_lse(N, Hq, Hkv, d, dt, _ptr(q.contiguous()), _ptr(k.contiguous()),
                             _ptr(lse), _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise(rc, "attention_lse")
    if check:
        check_status(ws, stream)
    return lse


def mass_select(q, k, lse, budget_k: int, block_q: int = 1, *,
                workspace: Optional[Workspace] = None, stream=None, check: bool = True,
                workspace_bytes: Optional[int] = None) -> Support:
    """Pass 2: head-averaged mass and its top-k support, given pass 1's lse [Hq, N].

    workspace_bytes: as in mass_oracle_prefill."""
    dev = q.device
    N, Hq, Hkv, d = _shape(q, k)
    dt = _dtype_code(q)
    if lse.shape != (Hq, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be [Hq, N] fp32")
    n_sel = N if block_q == 1 else -(-N // block_q)
    sup_idx = torch.empty(n_sel, budget_k, dtype=torch.int32, device=dev)
    sup_len = torch.empty(n_sel, dtype=torch.int32, device=dev)
    sup_mass = torch.empty(n_sel, budget_k, dtype=torch.float32, device=dev)
    L = lib()
    nbytes = L.tam_mass_select_workspace(N, Hq, Hkv, d, dt, budget_k, block_q)
    if workspace_bytes is not None and nbytes:
        nbytes = int(workspace_bytes)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_mass_select(N, Hq, Hkv, d, dt, _ptr(q.contiguous()), _ptr(k.contiguous()),
                           _ptr(lse.contiguous()), budget_k, block_q, _ptr(sup_idx), _ptr(sup_len),
                           _ptr(sup_mass), _ptr(ws), min(ws.numel(), nbytes) if nbytes else 0,
                           _stream(dev, stream))
    _raise(rc, "mass_select")
    if check:
        check_status(ws, stream)
    return Support(sup_idx, sup_len, sup_mass)


def indexer_topk(q_idx, k_idx, budget_k: int, block_q: int = 1, *,
                 workspace: Optional[Workspace] = None, stream=None, check: bool = True,
                 device=None, workspace_bytes: Optional[int] = None) -> Support:
    """Head-collapsed indexer support: top-k of q_idx . k_idx per query (block_q = 1), or
    per block of block_q queries the top-k of the block's summed per-query softmax of
    those scores (block_q > 1; values are the block sums).

    workspace_bytes: at least tam_indexer_workspace_min (more chunks below the
    preferred size)."""
    dev = _dev_of(q_idx, device)
    (q_idx, k_idx), host = _to_device([q_idx, k_idx], dev)
    N, dx = q_idx.shape
    if k_idx.shape != q_idx.shape or k_idx.dtype != q_idx.dtype:
        raise ValueError("q_idx and k_idx must both be [N, d_idx] of one dtype")
    dt = _dtype_code(q_idx)
    n_sel = N if block_q == 1 else -(-N // block_q)
    sup_idx = torch.empty(n_sel, budget_k, dtype=torch.int32, device=dev)
    sup_len = torch.empty(n_sel, dtype=torch.int32, device=dev)
    sup_score = torch.empty(n_sel, budget_k, dtype=torch.float32, device=dev)
    L = lib()
    nbytes = L.tam_indexer_workspace(N, dx, dt, budget_k, block_q)
    if workspace_bytes is not None and nbytes:
        nbytes = int(workspace_bytes)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_indexer_topk(N, dx, dt, _ptr(q_idx), _ptr(k_idx), budget_k, block_q,
                            _ptr(sup_idx), _ptr(sup_len), _ptr(sup_score), _ptr(ws),
                            min(ws.numel(), nbytes) if nbytes else 0, _stream(dev, stream))
    _raise(rc, "indexer_topk")
    if check:
        check_status(ws, stream)
    res = Support(sup_idx, sup_len, sup_score)
    if host:
        res = Support(res.idx.cpu(), res.length.cpu(), res.value.cpu())
    return res


def distill_kl(q, k, lse, q_idx, k_idx, *, workspace: Optional[Workspace] = None, stream=None,
               check: bool = True, workspace_bytes: Optional[int] = None) -> torch.Tensor:
    """The indexer's distillation target per query: KL(P_i || softmax(q_idx_i . k_idx)),
    P_i the head-averaged mass of pass 2 (given pass 1's lse [Hq, N]).  Returns [N] fp32."""
    dev = q.device
    N, Hq, Hkv, d = _shape(q, k)
    dt = _dtype_code(q)
    if lse.shape != (Hq, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be [Hq, N] fp32")
    if q_idx.shape != k_idx.shape or q_idx.shape[0] != N or q_idx.dtype != q.dtype:
        raise ValueError("q_idx and k_idx must be [N, d_idx] in q's dtype")
    dx = q_idx.shape[1]
    kl = torch.empty(N, dtype=torch.float32, device=dev)
    L = lib()
    nbytes = L.tam_distill_kl_workspace(N, Hq, Hkv, d, dt, dx)
    if workspace_bytes is not None and nbytes:
        nbytes = int(workspace_bytes)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_distill_kl(N, Hq, Hkv, d, dt, _ptr(q.contiguous()), _ptr(k.contiguous()),
                          _ptr(lse.contiguous()), dx, _ptr(q_idx.contiguous()),
                          _ptr(k_idx.contiguous()), _ptr(kl), _ptr(ws),
                          min(ws.numel(), nbytes) if nbytes else 0, _stream(dev, stream))
    _raise(rc, "distill_kl")
    if check:
        check_status(ws, stream)
    return kl


def support_mass_curve(sup_val, sup_len, budgets, *, stream=None) -> torch.Tensor:
    """Budget sweep: [rows, len(budgets)] fp32, the sum of the k largest values of each
    support row for every budget k (rows of a top-kmax support, e.g. Support.value)."""
    dev = sup_val.device
    if sup_val.dim() != 2 or sup_val.dtype != torch.float32 or sup_len.dtype != torch.int32:
        raise TypeError("sup_val [rows, kmax] fp32 and sup_len [rows] int32")
    rows, kmax = sup_val.shape
    ks = (ctypes.c_int32 * len(budgets))(*[int(b) for b in budgets])
    out = torch.empty(rows, len(budgets), dtype=torch.float32, device=dev)
    rc = lib().tam_support_mass_curve(rows, kmax, _ptr(sup_val.contiguous()),
                                      _ptr(sup_len.contiguous()), ks, len(budgets), _ptr(out),
                                      _stream(dev, stream))
    _raise(rc, "support_mass_curve")
    return out


def sparse_support_attention(q, k, v, sup_idx, sup_len, block_q: int = 1, *,
                             return_lse: bool = False, workspace: Optional[Workspace] = None,
                             stream=None, check: bool = True, device=None):
    """Pass 3: attention recomputed on a given support. Returns out (and lse)."""
    dev = _dev_of(q, device)
    (q, k, v, sup_idx, sup_len), host = _to_device([q, k, v, sup_idx, sup_len], dev)
    N, Hq, Hkv, d = _shape(q, k)
    dt = _dtype_code(q)
    if sup_idx.dtype != torch.int32 or sup_len.dtype != torch.int32:
        raise TypeError("sup_idx and sup_len are int32")
    kmax = sup_idx.shape[1]
    out = torch.empty_like(q)
    lse = torch.empty(Hq, N, dtype=torch.float32, device=dev) if return_lse else None
    L = lib()
    nbytes = L.tam_sparse_attention_workspace(N, Hq, Hkv, d, dt)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_sparse_support_attention(N, Hq, Hkv, d, dt, _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(sup_idx), _ptr(sup_len), kmax, block_q, _ptr(out),
                                        _ptr(lse), _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise(rc, "sparse_support_attention")
    if check:
        check_status(ws, stream)
    if host:
        out = out.cpu()
        lse = None if lse is None else lse.cpu()
    return (out, lse) if return_lse else out


def dense_gqa_prefill(q, k, v, *, return_lse: bool = False,
                      workspace: Optional[Workspace] = None, stream=None, check: bool = True,
                      device=None):
    """Dense causal GQA attention. Returns out (and lse)."""
    dev = _dev_of(q, device)
    (q, k, v), host = _to_device([q, k, v], dev)
    N, Hq, Hkv, d = _shape(q, k)
    dt = _dtype_code(q)
    out = torch.empty_like(q)
    lse = torch.empty(Hq, N, dtype=torch.float32, device=dev) if return_lse else None
    L = lib()
    nbytes = L.tam_dense_workspace(N, Hq, Hkv, d, dt)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_dense_gqa_prefill(N, Hq, Hkv, d, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                 _ptr(lse), _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise(rc, "dense_gqa_prefill")
    if check:
        check_status(ws, stream)
    if host:
        out = out.cpu()
        lse = None if lse is None else lse.cpu()
    return (out, lse) if return_lse else out


# ------------------------------------------------------------------ packed batches

def _cu_host(cu_seqlens) -> torch.Tensor:
    """cu_seqlens as a contiguous host int64 tensor (the library reads it on the host)."""
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int64, device="cpu").contiguous()
    if cu.dim() != 1 or cu.numel() < 2:
        raise ValueError("cu_seqlens is [n_seq + 1] int64")
    return cu


def selection_offsets(cu_seqlens, block_q: int = 1) -> torch.Tensor:
    """First selection row of every sequence of a packed batch ([n_seq + 1] int64)."""
    cu = _cu_host(cu_seqlens)
    n = cu[1:] - cu[:-1]
    n_sel = n if block_q == 1 else (n + block_q - 1) // block_q
    return torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n_sel, 0)])


def lse_block(lse: torch.Tensor, cu_seqlens, s: int) -> torch.Tensor:
    """The [Hq, N_s] lse block of sequence s inside a packed varlen lse."""
    cu = _cu_host(cu_seqlens)
    t0, t1 = int(cu[s]), int(cu[s + 1])
    Hq = lse.numel() // int(cu[-1]) if int(cu[-1]) else 0
    return lse[Hq * t0:Hq * t1].view(Hq, t1 - t0)


def mass_oracle_prefill_varlen(q, k, v, cu_seqlens, budget_k: int, block_q: int = 1, *,
                               compute_out: bool = True, return_lse: bool = True,
                               workspace: Optional[Workspace] = None, stream=None,
                               check: bool = True, device=None) -> Support:
    """mass_oracle_prefill over a packed batch: q [T, Hq, d], k/v [T, Hkv, d], sequence s
    owning tokens [cu_seqlens[s], cu_seqlens[s+1]).  Support rows are packed in sequence
    order (see ``selection_offsets``), key indices are positions within the sequence,
    and ``lse`` is flat (one [Hq, N_s] block per sequence, see ``lse_block``)."""
    cu = _cu_host(cu_seqlens)
    n_seq = cu.numel() - 1
    dev = _dev_of(q, device)
    (q, k, v), host = _to_device([q, k, v], dev)
    T, Hq, Hkv, d = _shape(q, k)
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    if compute_out and v is None:
        raise ValueError("v is needed for the recomputed output")
    dt = _dtype_code(q)
    n_sel = int(selection_offsets(cu, block_q)[-1])
    sup_idx = torch.empty(n_sel, budget_k, dtype=torch.int32, device=dev)
    sup_len = torch.empty(n_sel, dtype=torch.int32, device=dev)
    sup_mass = torch.empty(n_sel, budget_k, dtype=torch.float32, device=dev)
    lse = torch.empty(Hq * T, dtype=torch.float32, device=dev) if return_lse else None
    out = torch.empty_like(q) if compute_out else None
    L = lib()
    cu_p = ctypes.c_void_p(cu.data_ptr())
    nbytes = L.tam_mass_oracle_workspace_varlen(n_seq, cu_p, Hq, Hkv, d, dt, budget_k, block_q)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_mass_oracle_prefill_varlen(n_seq, cu_p, Hq, Hkv, d, dt, _ptr(q), _ptr(k), _ptr(v),
                                          budget_k, block_q, _ptr(sup_idx), _ptr(sup_len),
                                          _ptr(sup_mass), _ptr(lse), _ptr(out), _ptr(ws),
                                          ws.numel() if nbytes else 0, _stream(dev, stream))
    _raise(rc, "mass_oracle_prefill_varlen")
    if check:
        check_status(ws, stream)
    res = Support(sup_idx, sup_len, sup_mass, lse, out)
    if host:
        res = Support(*[None if t is None else t.cpu() for t in
                        (res.idx, res.length, res.value, res.lse, res.out)])
    return res


def dense_gqa_prefill_varlen(q, k, v, cu_seqlens, *, return_lse: bool = False,
                             workspace: Optional[Workspace] = None, stream=None,
                             check: bool = True, device=None):
    """dense_gqa_prefill over a packed batch (layout as mass_oracle_prefill_varlen)."""
    cu = _cu_host(cu_seqlens)
    n_seq = cu.numel() - 1
    dev = _dev_of(q, device)
    (q, k, v), host = _to_device([q, k, v], dev)
    T, Hq, Hkv, d = _shape(q, k)
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    dt = _dtype_code(q)
    out = torch.empty_like(q)
    lse = torch.empty(Hq * T, dtype=torch.float32, device=dev) if return_lse else None
    L = lib()
    ws = _workspace(dev, 256, workspace)
    rc = L.tam_dense_gqa_prefill_varlen(n_seq, ctypes.c_void_p(cu.data_ptr()), Hq, Hkv, d, dt,
                                        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(ws),
                                        ws.numel(), _stream(dev, stream))
    _raise(rc, "dense_gqa_prefill_varlen")
    if check:
        check_status(ws, stream)
    if host:
        out = out.cpu()
        lse = None if lse is None else lse.cpu()
    return (out, lse) if return_lse else out


def indexer_topk_varlen(q_idx, k_idx, cu_seqlens, budget_k: int, block_q: int = 1, *,
                        workspace: Optional[Workspace] = None, stream=None, check: bool = True,
                        device=None) -> Support:
    """indexer_topk over a packed batch: q_idx, k_idx [T, d_idx]; support rows packed in
    sequence order (see ``selection_offsets``), positions local to each sequence."""
    cu = _cu_host(cu_seqlens)
    n_seq = cu.numel() - 1
    dev = _dev_of(q_idx, device)
    (q_idx, k_idx), host = _to_device([q_idx, k_idx], dev)
    if q_idx.dim() != 2 or k_idx.shape != q_idx.shape or k_idx.dtype != q_idx.dtype:
        raise ValueError("q_idx and k_idx are [T, d_idx] of one dtype")
    T, dx = q_idx.shape
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    dt = _dtype_code(q_idx)
    n_sel = int(selection_offsets(cu, block_q)[-1])
    sup_idx = torch.empty(n_sel, budget_k, dtype=torch.int32, device=dev)
    sup_len = torch.empty(n_sel, dtype=torch.int32, device=dev)
    sup_score = torch.empty(n_sel, budget_k, dtype=torch.float32, device=dev)
    L = lib()
    cu_p = ctypes.c_void_p(cu.data_ptr())
    nbytes = L.tam_indexer_workspace_varlen(n_seq, cu_p, dx, dt, budget_k, block_q)
    ws = _workspace(dev, max(nbytes, 256), workspace)
    rc = L.tam_indexer_topk_varlen(n_seq, cu_p, dx, dt, _ptr(q_idx), _ptr(k_idx), budget_k,
                                   block_q, _ptr(sup_idx), _ptr(sup_len), _ptr(sup_score),
                                   _ptr(ws), ws.numel() if nbytes else 0, _stream(dev, stream))
    _raise(rc, "indexer_topk_varlen")
    if check:
        check_status(ws, stream)
    res = Support(sup_idx, sup_len, sup_score)
    if host:
        res = Support(res.idx.cpu(), res.length.cpu(), res.value.cpu())
    return res


def sparse_support_attention_varlen(q, k, v, sup_idx, sup_len, cu_seqlens, block_q: int = 1, *,
                                    return_lse: bool = False,
                                    workspace: Optional[Workspace] = None, stream=None,
                                    check: bool = True, device=None):
    """sparse_support_attention over a packed batch; support rows as the varlen selection
    calls lay them out.  Returns out [T, Hq, d] (and the flat per-sequence lse blocks)."""
    cu = _cu_host(cu_seqlens)
    n_seq = cu.numel() - 1
    dev = _dev_of(q, device)
    (q, k, v, sup_idx, sup_len), host = _to_device([q, k, v, sup_idx, sup_len], dev)
    T, Hq, Hkv, d = _shape(q, k)
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    if sup_idx.dtype != torch.int32 or sup_len.dtype != torch.int32:
        raise TypeError("sup_idx and sup_len are int32")
    dt = _dtype_code(q)
    out = torch.empty_like(q)
    lse = torch.empty(Hq * T, dtype=torch.float32, device=dev) if return_lse else None
    L = lib()
    ws = _workspace(dev, 256, workspace)
    rc = L.tam_sparse_support_attention_varlen(n_seq, ctypes.c_void_p(cu.data_ptr()), Hq, Hkv, d,
                                               dt, _ptr(q), _ptr(k), _ptr(v), _ptr(sup_idx),
                                               _ptr(sup_len), sup_idx.shape[1], block_q, _ptr(out),
                                               _ptr(lse), _ptr(ws), ws.numel(),
                                               _stream(dev, stream))
    _raise(rc, "sparse_support_attention_varlen")
    if check:
        check_status(ws, stream)
    if host:
        out = out.cpu()
        lse = None if lse is None else lse.cpu()
    return (out, lse) if return_lse else out
