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


@pytest.mark.parametrize("name", ["tiny", "tile64", "tile64map"])
def test_graph_replay_matches_eager_steps(name):
    """vsa.Forward.graph: a CUDA graph of one step, replayed after the inputs
    change in place, gives bit for bit what an eager step gives (the one-launch
    front end's counters are back at zero after each replay)."""
    wl = workloads.WORKLOADS[name]
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, prefix_dense=wl.prefix_dense)
    dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).cuda().view(torch.bfloat16)
    inp = workloads.make_inputs(wl)
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    keep = torch.from_numpy(inp["row_keep"]).cuda() if inp["row_keep"] is not None else None
    g = fwd.graph(q, k, v, bmap, row_keep=keep)
    fields = {f: getattr(wl, f) for f in wl.__dataclass_fields__ if f != "name"}
    other = workloads.make_inputs(workloads.custom(name="other", **{**fields, "seed": 7}))
    for src in (other, inp):
        q.copy_(dev(src["q"])), k.copy_(dev(src["k"])), v.copy_(dev(src["v"]))
        g.replay()
        torch.cuda.synchronize()
        got_o, got_lse, got_idx = fwd.o.clone(), fwd.lse.clone(), fwd.idx.clone()
        ref_o, ref_lse = fwd(q, k, v, bmap, row_keep=keep)
        torch.cuda.synchronize()
        assert vsa.get_status() == vsa.VSA_OK
        assert torch.equal(got_idx, fwd.idx)
        assert torch.equal(got_o.view(torch.int16), ref_o.view(torch.int16))
        assert torch.equal(got_lse.view(torch.int32), ref_lse.view(torch.int32))
        assert int(fwd.ws.abs().sum()) == 0
