"""GPU parity of the one-launch front end (vsa_tile_coarse): tiling, block
means, selection and compression branch, bit for bit equal to the separate
launches and to the oracle ("FastVideo VSA", introduction and section
"Choose top-k"; section "Checkpoint behavior" for the compression branch)."""
import numpy as np
import pytest
import torch

import block_sparse_video_gather_b200 as vsa
import oracle
from block_sparse_video_gather_b200 import build as vsa_build
from block_sparse_video_gather_b200 import workloads
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()


def _dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TDT[dtype])


def _host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _bits(t):
    return t.cpu().numpy().view(np.uint32)


def _separate(plan, q, k, v, topk, gated):
    qt, qb = vsa.tile(plan, q, pooled=True)
    kt, kb = vsa.tile(plan, k, pooled=True)
    vt, vb = vsa.tile(plan, v, pooled=True) if gated else (vsa.tile(plan, v), None)
    out = dict(qt=qt, kt=kt, vt=vt, qbar=qb, kbar=kb)
    if gated:
        out["vbar"] = vb
        r = vsa.coarse_compress(plan, qb, kb, vb, topk)
        if topk > 0:
            out["oc"], out["idx"], out["num"] = r
        else:
            out["oc"] = r
    elif topk > 0:
        out["idx"], out["num"] = vsa.coarse_topk(plan, qb, kb, topk)
    return out


CASES = [
    # (name, workload kwargs, topk, gated, dtype)
    ("tiny", None, 4, False, "bf16"),
    ("tiny-gated", None, 4, True, "bf16"),
    ("fastwan", None, 64, False, "bf16"),
    ("fastwan-gated-f16", None, 64, True, "f16"),
    ("long", None, 59, False, "bf16"),
    ("one-block", dict(T=3, Hg=5, Wg=7, B=2, H=3), 1, True, "bf16"),
    ("ragged", dict(T=9, Hg=17, Wg=23, B=2, H=2), 5, False, "f16"),
    ("tile64-prefix", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 7, True, "bf16"),
    ("tiles-only", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 0, False, "bf16"),
    # 7 blocks: the last tile item of four 64-token blocks holds three
    ("tile64-odd", dict(T=5, Hg=9, Wg=4, block=(4, 4, 4), n_prefix=10, B=2, H=2), 3, True, "f16"),
    ("compress-only", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 0, True, "f16"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_one_launch_equals_separate_launches_and_oracle(case):
    name, kw, topk, gated, dtype = case
    wl = workloads.WORKLOADS[name.split("-")[0]] if kw is None else workloads.custom(topk=max(topk, 1), **kw)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype=dtype)
    plan = vsa.Plan.of(wl)
    q, k, v = (_dev(inp[n], dtype) for n in ("q", "k", "v"))
    ws = vsa.workspace(wl.B, wl.H)
    fused = vsa.tile_coarse(plan, q, k, v, topk, ws, gated)
    sep = _separate(plan, q, k, v, topk, gated)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    assert int(ws.abs().sum()) == 0, "workspace must be zero again after the launch"
    assert sorted(fused) == sorted(sep)
    for n in fused:
        a, b = fused[n], sep[n]
        if a.dtype in (torch.bfloat16, torch.float16):
            assert np.array_equal(_host(a), _host(b)), n
        elif a.dtype == torch.float32:
            assert np.array_equal(_bits(a), _bits(b)), n
        else:
            assert torch.equal(a, b), n
    # and against the oracle
    for n, t in (("q", "qt"), ("k", "kt"), ("v", "vt")):
        ref = oracle.tile(g, inp[n])
        assert np.array_equal(_host(fused[t]), ref), t
        if t != "vt" or gated:
            assert np.array_equal(_bits(fused[t[0] + "bar"]), oracle.pool(g, ref, dtype).view(np.uint32))
    if topk > 0:
        qb, kb = oracle.pool(g, oracle.tile(g, inp["q"]), dtype), oracle.pool(g, oracle.tile(g, inp["k"]), dtype)
        ridx, rnum = oracle.topk(oracle.score(qb, kb), topk)
        assert np.array_equal(fused["idx"].cpu().numpy(), ridx)
        assert np.array_equal(fused["num"].cpu().numpy(), rnum)


def test_repeated_calls_and_forward_paths_agree():
    """Two fused calls in a row (workspace reused) and the separate-launch
    Forward give identical results on the benchmark workload, gated."""
    wl = workloads.WORKLOADS["fastwan"]
    inp = workloads.make_inputs(wl, gate=True)
    plan = vsa.Plan.of(wl)
    args = [H.to_dev(inp[n]) for n in ("q", "k", "v")]
    gate = H.to_dev(inp["gate"])
    f1 = vsa.Forward(plan, wl.B, wl.H, wl.topk, gated=True, fused=True)
    f0 = vsa.Forward(plan, wl.B, wl.H, wl.topk, gated=True, fused=False)
    o1 = f1(*args, gate=gate)[0].clone()
    o1b = f1(*args, gate=gate)[0].clone()
    o0 = f0(*args, gate=gate)[0].clone()
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    assert torch.equal(o1.view(torch.int16), o1b.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o0.view(torch.int16))
    assert torch.equal(f1.idx, f0.idx) and torch.equal(f1.oc.view(torch.int32), f0.oc.view(torch.int32))
    assert int(f1.ws.abs().sum()) == 0
