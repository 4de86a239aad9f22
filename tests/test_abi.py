"""The C-ABI library loads, exports every symbol tam.h declares, and rejects bad
arguments on the host before touching the GPU (no compute call runs here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tam.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tam_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(tam_lib):
    L = tam_lib.lib()
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(tam_lib.EXPORTED)


def test_debug_checks_build_exports_the_same_symbols(tam_lib):
    """libtam_debug.so (the pass-2 stores checked against their extents) is built beside
    libtam.so and exports every declared symbol too."""
    path = os.path.join(ROOT, "top_attention_mass_b200", "libtam_debug.so")
    assert os.path.exists(path), "build() builds the debug-checks library"
    D = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(D, n), n


def test_version_and_status_strings(tam_lib):
    assert tam_lib.version() >= 100
    for code in range(7):
        assert tam_lib.status_string(code) != "unknown status"
    assert tam_lib.status_string(99) == "unknown status"


def test_workspace_queries(tam_lib):
    L = tam_lib.lib()
    ws = L.tam_mass_oracle_workspace(4096, 32, 8, 128, tam_lib.TAM_BF16, 256, 1)
    assert ws > 0 and ws % 256 == 0
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 128, tam_lib.TAM_BF16, 256, 64) > 0
    # rejected arguments give 0
    assert L.tam_mass_oracle_workspace(4096, 30, 8, 128, 0, 256, 1) == 0      # Hq % Hkv
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 96, 0, 256, 1) == 0       # d
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 128, 0, 0, 1) == 0        # k < 1
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 128, 0, 5000, 1) == 0     # k > 4096
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 128, 0, 256, 0) == 0      # block_q < 1
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 128, 7, 256, 1) == 0      # dtype
    lo = L.tam_mass_workspace_min(4096, 32, 8, 128, tam_lib.TAM_BF16, 256, 1)
    assert 0 < lo <= ws
    assert L.tam_mass_workspace_min(4096, 32, 8, 128, 0, 0, 1) == 0          # k < 1
    assert L.tam_indexer_workspace(4096, 64, 0, 1024, 1) > 0
    assert 0 < L.tam_indexer_workspace_min(4096, 64, 0, 1024, 1) <= L.tam_indexer_workspace(
        4096, 64, 0, 1024, 1)
    assert L.tam_indexer_workspace(4096, 48, 0, 1024, 1) == 0
    for f in ("tam_attention_lse_workspace", "tam_sparse_attention_workspace",
              "tam_dense_workspace"):
        assert getattr(L, f)(4096, 32, 8, 128, 0) >= 256


def _fake(addr=1 << 20):
    return ctypes.c_void_p(addr)        # aligned, never dereferenced: calls fail validation first


def test_host_side_argument_errors(tam_lib):
    L = tam_lib.lib()
    T = tam_lib
    f = _fake()
    # null pointers
    rc = L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, None, f, f, 8, 1, f, f, f, None, None, f,
                                   1 << 30, None)
    assert rc == T.TAM_ERR_INVALID_ARG
    # misaligned pointer
    rc = L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, ctypes.c_void_p((1 << 20) + 2), f, f, 8, 1,
                                   f, f, f, None, None, f, 1 << 30, None)
    assert rc == T.TAM_ERR_INVALID_ARG
    # bad shapes / budgets
    assert L.tam_mass_oracle_prefill(64, 6, 4, 64, 0, f, f, f, 8, 1, f, f, f, None, None, f,
                                     1 << 30, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_mass_oracle_prefill(64, 4, 1, 80, 0, f, f, f, 8, 1, f, f, f, None, None, f,
                                     1 << 30, None) == T.TAM_ERR_UNSUPPORTED
    assert L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, f, f, f, 0, 1, f, f, f, None, None, f,
                                     1 << 30, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, f, f, f, 8192, 1, f, f, f, None, None, f,
                                     1 << 30, None) == T.TAM_ERR_UNSUPPORTED
    assert L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, f, f, f, 8, 0, f, f, f, None, None, f,
                                     1 << 30, None) == T.TAM_ERR_INVALID_ARG
    # N * k >= 2^31
    assert L.tam_mass_oracle_prefill(1 << 21, 4, 1, 64, 0, f, f, f, 1024, 1, f, f, f, None, None,
                                     f, 1 << 40, None) == T.TAM_ERR_UNSUPPORTED
    # workspace too small
    assert L.tam_mass_oracle_prefill(64, 4, 1, 64, 0, f, f, f, 8, 1, f, f, f, None, None, f, 16,
                                     None) == T.TAM_ERR_WORKSPACE
    assert L.tam_indexer_topk(64, 32, 0, f, f, 8, 2, f, f, f, f, 1 << 30,
                              None) == T.TAM_ERR_UNSUPPORTED          # block-shared: d_idx 64/128
    assert L.tam_indexer_topk(64, 64, 0, f, f, 8, 2, f, f, f, f, 16,
                              None) == T.TAM_ERR_WORKSPACE            # block-shared indexer
    assert L.tam_indexer_topk(64, 40, 0, f, f, 8, 1, f, f, f, f, 1 << 30,
                              None) == T.TAM_ERR_UNSUPPORTED
    assert L.tam_sparse_support_attention(64, 4, 1, 64, 0, f, f, f, None, f, 8, 1, f, None, f,
                                          1 << 20, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_dense_gqa_prefill(64, 4, 1, 64, 0, f, f, f, f, None, f, 8,
                                   None) == T.TAM_ERR_WORKSPACE
    assert L.tam_attention_lse(64, 4, 1, 64, 0, f, f, None, f, 256, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_check_status(None, None, None) == T.TAM_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """With libtam.so absent the binding raises instead of computing anything elsewhere."""
    import top_attention_mass_b200 as tam
    monkeypatch.setattr(tam, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(tam, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        tam.lib()


def test_product_does_not_import_the_oracle():
    """Nothing in the package refers to the oracle."""
    pkg = os.path.join(ROOT, "top_attention_mass_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "liboracle" not in txt and "orc_" not in txt, fn


def test_varlen_and_head_dim_host_checks(tam_lib):
    """Packed-batch offsets and head dims are validated on the host (no launch here)."""
    import numpy as np
    L = tam_lib.lib()
    T = tam_lib
    f = _fake()

    def cu_ptr(a):
        arr = np.ascontiguousarray(a, np.int64)
        return arr, arr.ctypes.data_as(ctypes.c_void_p)

    good, gp = cu_ptr([0, 100, 100, 4096])
    ws = L.tam_mass_oracle_workspace_varlen(3, gp, 32, 8, 128, T.TAM_BF16, 256, 1)
    assert ws > 0 and ws % 256 == 0
    # the largest sequence sets the size (the single-sequence query for it), plus the packed
    # LSE of the whole batch (Hq x T floats, rounded up to 256 bytes, and 256 bytes of slack)
    lse_bytes = (32 * 4096 * 4 + 255) // 256 * 256 + 256
    assert ws == L.tam_mass_oracle_workspace(3996, 32, 8, 128, T.TAM_BF16, 256, 1) + lse_bytes
    assert L.tam_mass_oracle_workspace_varlen(3, gp, 32, 8, 256, T.TAM_BF16, 256, 1) > 0
    assert L.tam_mass_oracle_workspace_varlen(3, gp, 32, 8, 96, T.TAM_BF16, 256, 1) == 0
    for bad in ([1, 100], [0, 50, 40], [0, 1 << 31]):
        arr, bp = cu_ptr(bad)
        n = len(bad) - 1
        assert L.tam_mass_oracle_workspace_varlen(n, bp, 32, 8, 128, 0, 8, 1) == 0
        assert L.tam_mass_oracle_prefill_varlen(n, bp, 32, 8, 128, 0, f, f, f, 8, 1, f, f, f, None,
                                                None, f, 1 << 30, None) != T.TAM_OK
        assert L.tam_dense_gqa_prefill_varlen(n, bp, 32, 8, 128, 0, f, f, f, f, None, f, 1 << 20,
                                              None) != T.TAM_OK
    assert L.tam_mass_oracle_prefill_varlen(0, gp, 32, 8, 128, 0, f, f, f, 8, 1, f, f, f, None,
                                            None, f, 1 << 30, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_mass_oracle_prefill_varlen(3, None, 32, 8, 128, 0, f, f, f, 8, 1, f, f, f, None,
                                            None, f, 1 << 30, None) == T.TAM_ERR_INVALID_ARG
    # workspace below the largest sequence's minimum
    assert L.tam_mass_oracle_prefill_varlen(3, gp, 32, 8, 128, 0, f, f, f, 8, 1, f, f, f, None,
                                            None, f, 4096, None) == T.TAM_ERR_WORKSPACE
    assert L.tam_dense_gqa_prefill_varlen(3, gp, 32, 8, 128, 0, f, f, f, f, None, f, 16,
                                          None) == T.TAM_ERR_WORKSPACE
    assert L.tam_dense_gqa_prefill_varlen(3, gp, 32, 8, 80, 0, f, f, f, f, None, f, 1 << 20,
                                          None) == T.TAM_ERR_UNSUPPORTED
    # head dim 256 is accepted by the single-sequence queries too
    assert L.tam_mass_oracle_workspace(4096, 32, 8, 256, T.TAM_BF16, 256, 1) > 0
    assert L.tam_dense_workspace(4096, 32, 8, 256, T.TAM_F32) > 0


def test_varlen_indexer_and_pass3_host_checks(tam_lib):
    import numpy as np
    L = tam_lib.lib()
    T = tam_lib
    f = _fake()
    good = np.array([0, 64, 64, 4096], np.int64)
    gp = good.ctypes.data_as(ctypes.c_void_p)
    assert L.tam_indexer_workspace_varlen(3, gp, 64, T.TAM_BF16, 1024, 1) == \
        L.tam_indexer_workspace(4032, 64, T.TAM_BF16, 1024, 1)
    assert L.tam_indexer_workspace_varlen(3, gp, 40, T.TAM_BF16, 1024, 1) == 0
    bad = np.array([0, 50, 40], np.int64)
    bp = bad.ctypes.data_as(ctypes.c_void_p)
    assert L.tam_indexer_workspace_varlen(2, bp, 64, T.TAM_BF16, 8, 1) == 0
    assert L.tam_indexer_topk_varlen(2, bp, 64, 0, f, f, 8, 1, f, f, f, f, 1 << 30,
                                     None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_indexer_topk_varlen(3, gp, 32, 0, f, f, 8, 2, f, f, f, f, 1 << 30,
                                     None) == T.TAM_ERR_UNSUPPORTED       # block-shared: d_idx 64/128
    assert L.tam_indexer_topk_varlen(3, gp, 64, 0, f, f, 8, 1, f, f, f, f, 64,
                                     None) == T.TAM_ERR_WORKSPACE
    assert L.tam_sparse_support_attention_varlen(2, bp, 32, 8, 128, 0, f, f, f, f, f, 8, 1, f, None,
                                                 f, 1 << 20, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_sparse_support_attention_varlen(3, gp, 32, 8, 128, 0, f, f, f, None, f, 8, 1, f,
                                                 None, f, 1 << 20, None) == T.TAM_ERR_INVALID_ARG
    assert L.tam_sparse_support_attention_varlen(3, gp, 32, 8, 128, 0, f, f, f, f, f, 8, 1, f, None,
                                                 f, 16, None) == T.TAM_ERR_WORKSPACE


def test_packed_batch_helpers():
    """Host-side helpers of the varlen binding (no device involved)."""
    import torch
    import top_attention_mass_b200 as tam
    cu = [0, 1, 130, 130, 393]
    assert tam.selection_offsets(cu, 1).tolist() == [0, 1, 130, 130, 393]
    # blocks of 64: 1 -> 1, 129 -> 3, 0 -> 0, 263 -> 5
    assert tam.selection_offsets(cu, 64).tolist() == [0, 1, 4, 4, 9]
    Hq = 3
    flat = torch.arange(Hq * 393, dtype=torch.float32)
    blk = tam.lse_block(flat, cu, 3)
    assert blk.shape == (Hq, 263)
    assert blk[0, 0].item() == Hq * 130 and blk[2, 262].item() == Hq * 393 - 1
    assert tam.lse_block(flat, cu, 2).shape == (Hq, 0)
    with pytest.raises(ValueError):
        tam.selection_offsets([0], 1)


def _stream_layout(N, k, nseg, head):
    """The streamed per-query selection's workspace after `head` bytes, as include/tam.h
    documents it: sample stride S (the smallest prime of at least 17 leaving at most
    4096 sampled keys per row), segment capacity from the threshold rank, then tau, the
    fallback list, the counts and a region that holds the sample rows, the candidates
    or the fallback scratch; returns (preferred, minimum) sizes."""
    import math
    a256 = lambda x: (x + 255) // 256 * 256              # noqa: E731
    S = max(17, -(-N // 4096))
    while any(S % f == 0 for f in range(2, int(math.isqrt(S)) + 1)) or (N - 1) // S + 1 > 4096:
        S += 1
    mu = k / S
    r = math.ceil(mu + 5.0 * math.sqrt(mu) + 4.0)
    per = math.ceil(1.5 * S * (r + 1.0) / nseg) + 32
    seg_cap = (per + 31) // 32 * 32
    cap = nseg * seg_cap
    off_region = head + a256(N * 4) + a256((N + 1) * 4) + a256(N * nseg * 4)

    def sample_offset(i):
        a, b = i // S, i % S
        return i + S * (a * (a - 1) // 2) + a * b

    tri = N * (N + 1) // 2
    pref = max(sample_offset(N) * 4, N * cap * 8, min(N, 148) * N * 4)
    s_max = (N - 1) // S + 1
    lo = max(min(N, 64) * s_max * 4, min(N, 64) * cap * 8, min(tri, 64 * N) * 4)
    return off_region + a256(pref), off_region + a256(lo)


@pytest.mark.parametrize("N", [1, 64, 65, 1000, 4096, 32768, 65536])
def test_workspace_sizes_follow_the_documented_layout(tam_lib, N):
    """Per query on the tensor cores: status block (256 B), lse (Hq*N floats), then the
    streamed selection (thresholds, fallback list, candidate counts and a region sized
    for every row's candidates at once, at least 64 rows of them)."""
    L = tam_lib.lib()
    Hq, Hkv, d, k = 32, 8, 128, 16
    a256 = lambda x: (x + 255) // 256 * 256              # noqa: E731
    head = 256 + a256(Hq * N * 4)
    pref = L.tam_mass_oracle_workspace(N, Hq, Hkv, d, tam_lib.TAM_BF16, k, 1)
    lo = L.tam_mass_workspace_min(N, Hq, Hkv, d, tam_lib.TAM_BF16, k, 1)
    want_pref, want_lo = _stream_layout(N, k, 8, head)     # CTA pairs: 8 segments per row
    assert pref == want_pref
    assert lo == want_lo
    # the mass-select and no-lse variants share the layout
    assert L.tam_mass_select_workspace(N, Hq, Hkv, d, tam_lib.TAM_BF16, k, 1) == pref
