"""tam_mass_select_noalloc: pass 2 for callers that cannot allocate device memory.

Such callers (a plugin whose host engine owns all device memory, a process that
must not cudaMalloc while serving) get the scratch from a static device array in
the library.  The test calls the entry point through the C ABI twice in a row and
compares each result with the regular workspace-based entry point, within the
support/mass tolerance the other parity tests use.  One case per query fits the
static scratch whole, one is block-shared, and one (N = 8192, k = 1024) prefers
about 200 MB of workspace, so that inside the 64 MiB it runs in several chunks.  It
also checks that a problem larger than the static scratch is refused before anything
runs.  The file sorts
last so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import tam_synth
from parity_util import MASS_ATOL

pytestmark = pytest.mark.gpu


def _noalloc(L, q, k, lse, kb, bq, out):
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    idx, ln, ms = out
    return L.tam_mass_select_noalloc(N, Hq, Hkv, d, 0, q.data_ptr(), k.data_ptr(), lse.data_ptr(),
                                     kb, bq, idx.data_ptr(), ln.data_ptr(), ms.data_ptr(),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("N,Hq,Hkv,kb,bq", [(2048, 32, 8, 128, 1), (3000, 32, 8, 200, 64),
                                             (8192, 8, 2, 1024, 1)])
def test_noalloc_matches_workspace_entry_point(tam_lib, N, Hq, Hkv, kb, bq):
    w = tam_synth.custom("noalloc", N, Hq, Hkv, 128, dtype="bf16", seed=21, sink=True, needles=8)
    inp = tam_synth.make_inputs(w)
    q, k = inp.q.cuda(), inp.k.cuda()
    lse = tam_lib.attention_lse(q, k)
    ref = tam_lib.mass_select(q, k, lse, kb, bq)
    n_sel = N if bq == 1 else -(-N // bq)
    L = tam_lib.lib()
    if N == 8192:
        # the regular call's preferred workspace is well above the static scratch, the
        # smallest one well below it: the no-alloc call runs in chunks
        assert L.tam_mass_oracle_workspace(N, Hq, Hkv, 128, 0, kb, bq) > 2 * (64 << 20)
        assert L.tam_mass_workspace_min(N, Hq, Hkv, 128, 0, kb, bq) < (16 << 20)
    for _ in range(2):
        out = (torch.full((n_sel, kb), 7, dtype=torch.int32, device="cuda"),
               torch.full((n_sel,), 7, dtype=torch.int32, device="cuda"),
               torch.full((n_sel, kb), 7.0, dtype=torch.float32, device="cuda"))
        rc = _noalloc(L, q, k, lse, kb, bq, out)
        assert rc == tam_lib.TAM_OK, tam_lib.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(out[1], ref.length)
        assert torch.equal(out[0], ref.idx)
        err = (out[2] - ref.value).abs().max().item()
        assert err <= MASS_ATOL * bq


def test_noalloc_rejects_problems_beyond_the_static_scratch(tam_lib):
    L = tam_lib.lib()
    N, kb = 262144, 4096                   # lse + 64 mass rows alone need ~96 MiB
    need = L.tam_mass_workspace_min(N, 32, 8, 128, 0, kb, 1)
    assert need > (64 << 20)
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    rc = L.tam_mass_select_noalloc(N, 32, 8, 128, 0, p, p, p, kb, 1, p, p, p, None)
    assert rc == tam_lib.TAM_ERR_WORKSPACE
