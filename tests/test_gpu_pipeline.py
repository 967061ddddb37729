"""vsa.HostPipeline: steps on pinned host tensors with copies overlapped across
steps give, bit for bit, the outputs of the same steps run one at a time."""
import numpy as np
import pytest
import torch

import block_sparse_video_gather_b200 as vsa
from block_sparse_video_gather_b200 import build as vsa_build
from block_sparse_video_gather_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()


def _host(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("gated", [False, True])
def test_pipelined_steps_match_sequential_steps(gated):
    base = workloads.WORKLOADS["wan81"]
    fields = {k: v for k, v in base.__dict__.items() if k != "name"}
    wls = [workloads.custom(name=f"s{i}", **{**fields, "seed": 40 + i}) for i in range(4)]
    plan = vsa.Plan.of(base)
    fwd = vsa.Forward(plan, base.B, base.H, base.topk, gated=gated)
    inputs = [workloads.make_inputs(w, gate=gated) for w in wls]
    host = [{n: _host(x[n]) for n in (("q", "k", "v", "gate") if gated else ("q", "k", "v"))} for x in inputs]
    outs = [torch.empty(fwd.o.shape, dtype=torch.bfloat16).pin_memory() for _ in wls]
    pipe = vsa.HostPipeline(fwd)
    for h, o in zip(host, outs):
        pipe.submit(h["q"], h["k"], h["v"], o, gate=h.get("gate"))
    pipe.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    for h, o in zip(host, outs):
        ref, _ = fwd(*(h[n].cuda() for n in ("q", "k", "v")), gate=h["gate"].cuda() if gated else None)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16))
    assert not torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
