"""vsa_tile_coarse_static (the one-launch front end on the library's own
static counters) against vsa_tile_coarse with a caller workspace: identical
outputs on two calls in a row of each.  Kept in its own file, collected
last, so it runs after every other test as well as alone."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_video_gather_b200 as vsa
from block_sparse_video_gather_b200 import build as vsa_build
from block_sparse_video_gather_b200 import workloads


def test_rejects_more_heads_than_the_static_counters_hold():
    """B*H above 4096 is refused before any device work (runs without a GPU too)."""
    vsa_build.build()
    L = vsa.lib()
    p = vsa.Plan(4, 8, 8)
    F = ctypes.c_void_p(0x100000)
    rc = L.vsa_tile_coarse_static(p.handle, vsa.VSA_BF16, F, F, F, 2, 2049, 128, 1, F, F, F, F, F, None, F, F,
                                  None, None)
    assert rc == vsa.VSA_ERR_UNSUPPORTED


def _dev(bits, dtype):
    t = torch.float16 if dtype == "f16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(t)


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def _same(a: dict, b: dict):
    assert sorted(a) == sorted(b)
    for n in a:
        assert torch.equal(_bits(a[n]), _bits(b[n])), n


CASES = [
    ("fastwan", None, 64, False, "bf16"),
    ("gated-ragged", dict(T=9, Hg=17, Wg=23, B=2, H=3), 5, True, "f16"),
    ("tile64-prefix", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 7, True, "bf16"),
    ("compress-only", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 0, True, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_counters_match_caller_workspace(case):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    name, kw, topk, gated, dtype = case
    wl = workloads.WORKLOADS[name] if kw is None else workloads.custom(topk=max(topk, 1), **kw)
    inp = workloads.make_inputs(wl, dtype=dtype)
    plan = vsa.Plan.of(wl)
    q, k, v = (_dev(inp[n], dtype) for n in ("q", "k", "v"))
    ws = vsa.workspace(wl.B, wl.H)
    ref = [vsa.tile_coarse(plan, q, k, v, topk, ws, gated) for _ in range(2)]
    got = [vsa.tile_coarse(plan, q, k, v, topk, None, gated) for _ in range(2)]
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    for r in ref + got[1:]:
        _same(got[0], r)
    assert int(ws.abs().sum()) == 0
