"""The debug-checks build (libtam_debug.so): the pass-2 kernels check every slab-row,
candidate and block-mass store against the extent the host planned for the launch and,
instead of an out-of-range store, record TAM_ERR_OVERFLOW in the status block.

Each case runs in a child process (the library is chosen once per process, with
TAM_LIBRARY=debug).  With the planned extents the results equal the release library's
bit for bit and the status stays clear; with TAM_DEBUG_SHRINK_EXTENTS the host plans
extents of 64 entries while the buffers keep their size, so the checks fire (and skip
the stores) without any access outside a buffer."""
import json
import os
import subprocess
import sys

import pytest
import torch

import tam_synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys, torch
sys.path.insert(0, {root!r})
import tam_synth
import top_attention_mass_b200 as tam
assert tam.LIB_PATH.endswith("libtam_debug.so"), tam.LIB_PATH
w = tam_synth.custom("dbg", 3000, 16, 4, 128, dtype="bf16", seed=5, sink=True, needles=3)
inp = tam_synth.make_inputs(w)
q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
qx, kx = q[:, 0, :64].contiguous(), k[:, 0, :64].contiguous()
lse = tam.attention_lse(q, k)
res = {{}}
for name in ("perquery", "block", "indexer", "distill"):
    ws = tam.Workspace(q.device)
    if name == "indexer":
        out = tam.indexer_topk(qx, kx, 50, workspace=ws, check=False)
        saved = {{"idx": out.idx.cpu(), "value": out.value.cpu()}}
    elif name == "distill":
        saved = {{"kl": tam.distill_kl(q, k, lse, qx, kx, workspace=ws, check=False).cpu()}}
    else:
        out = tam.mass_oracle_prefill(q, k, v, 40, 1 if name == "perquery" else 64,
                                      workspace=ws, check=False)
        saved = {{"idx": out.idx.cpu(), "value": out.value.cpu()}}
    try:
        tam.check_status(ws.get(256))
        res[name] = {{"code": 0}}
    except tam.TamError as e:
        res[name] = {{"code": e.code, "detail": list(e.detail)}}
    torch.save(saved, {out!r} + "_" + name + ".pt")
print(json.dumps(res))
"""


def _child(tmp_path, shrink):
    env = dict(os.environ, TAM_LIBRARY="debug")
    if shrink:
        env["TAM_DEBUG_SHRINK_EXTENTS"] = "1"
    else:
        env.pop("TAM_DEBUG_SHRINK_EXTENTS", None)
    out = str(tmp_path / ("shrunk" if shrink else "planned"))
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, out=out)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1]), out


def test_debug_build_planned_extents_match_release(tam_lib, tmp_path):
    res, out = _child(tmp_path, shrink=False)
    assert all(r["code"] == 0 for r in res.values()), res
    w = tam_synth.custom("dbg", 3000, 16, 4, 128, dtype="bf16", seed=5, sink=True, needles=3)
    inp = tam_synth.make_inputs(w)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    qx, kx = q[:, 0, :64].contiguous(), k[:, 0, :64].contiguous()
    ref = {"perquery": tam_lib.mass_oracle_prefill(q, k, v, 40, 1),
           "block": tam_lib.mass_oracle_prefill(q, k, v, 40, 64),
           "indexer": tam_lib.indexer_topk(qx, kx, 50)}
    for name, r in ref.items():
        got = torch.load(out + "_" + name + ".pt")
        assert torch.equal(got["idx"], r.idx.cpu()), name
        assert torch.equal(got["value"], r.value.cpu()), name
    kl = tam_lib.distill_kl(q, k, tam_lib.attention_lse(q, k), qx, kx)
    assert torch.equal(torch.load(out + "_distill.pt")["kl"], kl.cpu())


def test_debug_build_flags_out_of_extent_stores(tam_lib, tmp_path):
    res, _ = _child(tmp_path, shrink=True)
    sites = {"perquery": (1, 2), "block": (3,), "indexer": (1, 2), "distill": (1,)}
    for name, r in res.items():
        assert r["code"] == tam_lib.TAM_ERR_OVERFLOW, (name, r)
        assert r["detail"][2] in sites[name], (name, r)       # the store site
        assert r["detail"][3] >= r["detail"][4] == 64, (name, r)   # index >= extent
