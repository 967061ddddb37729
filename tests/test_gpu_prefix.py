"""GPU parity of the tile-64 selection (vsa_coarse_topk_prefix and the
one-launch vsa_tile_coarse_prefix) against the oracle, bit for bit.

FastVideo commit log, examples/inference/basic/README.md: in the tile-64
layout the prefix query tiles attend every tile, a video query tile attends
the prefix plus a top-k of the video tiles, and some rows select nothing.
"""
import numpy as np
import pytest
import torch

import block_sparse_video_gather_b200 as vsa
import oracle
from block_sparse_video_gather_b200 import build as vsa_build
from block_sparse_video_gather_b200 import workloads
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()
    assert vsa.get_status() == vsa.VSA_OK


def _check(plan, qbar, kbar, k, keep, max_k, n_pre):
    """Standalone call and oracle on the same block means; returns the GPU index."""
    dq, dk = torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda()
    dkeep = torch.from_numpy(keep).cuda() if keep is not None else None
    idx, num = vsa.coarse_topk_prefix(plan, dq, dk, k, dkeep, max_k)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    ridx, rnum = oracle.topk_prefix(oracle.score(qbar, kbar), n_pre, k, keep, max_k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(num.cpu().numpy(), rnum)
    return idx, num


@pytest.mark.parametrize("fused", [False, True])
def test_tile64_workload_bit_exact(fused):
    """The full tile64 workload: tiling, means, index and counts equal the oracle's."""
    wl = workloads.WORKLOADS["tile64"]
    ref = H.oracle_front(wl)
    inp = H.inputs(wl)
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, prefix_dense=True, fused=fused)
    fwd.front(H.to_dev(inp["q"]), H.to_dev(inp["k"]), H.to_dev(inp["v"]),
              row_keep=torch.from_numpy(inp["row_keep"]).cuda())
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    np.testing.assert_array_equal(H.from_dev(fwd.qt), ref["qt"])
    np.testing.assert_array_equal(H.from_dev(fwd.vt), ref["vt"])
    np.testing.assert_array_equal(fwd.idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(fwd.num.cpu().numpy(), ref["num"])
    num = ref["num"]
    assert set(np.unique(num).tolist()) == {0, 40, 264}
    assert int((num == 0).sum()) == 317
    if fused:
        assert int(fwd.ws.abs().sum()) == 0


@pytest.mark.parametrize("n_prefix,k", [(100, 1), (100, 7), (128, 40), (100, 58), (0, 5)])
def test_prefix_rule_on_edge_grids(n_prefix, k):
    """A partial prefix tile, k = 1, k = every video tile (dense rows), no prefix
    at all, forced-empty rows, B = 2 and a row stride above the longest row."""
    wl = workloads.custom(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=n_prefix, H=3, B=2, topk=k)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qbar = oracle.pool(g, oracle.tile(g, inp["q"]))
    kbar = oracle.pool(g, oracle.tile(g, inp["k"]))
    keep = (np.random.default_rng(40).random((2, 3, g.NB)) > 0.15).astype(np.uint8)
    max_k = (g.NB if g.n_pre else k) + 3
    k = min(k, g.NB - g.n_pre)
    _check(vsa.Plan.of(wl), qbar, kbar, k, keep, max_k, g.n_pre)


@pytest.mark.parametrize("k", [1, 4, 9])
def test_prefix_rule_with_ties(k):
    """Integer-valued block means give many exact score ties: lower index wins."""
    rng = np.random.default_rng(41)
    plan = vsa.Plan(4, 8, 12, (4, 4, 4), n_prefix=130)  # 3 prefix tiles + 6 video tiles
    NB = plan.NB
    qbar = rng.integers(-2, 3, size=(1, 2, NB, 128)).astype(np.float32)
    kbar = rng.integers(-2, 3, size=(1, 2, NB, 128)).astype(np.float32)
    kbar[0, 1] = 0.0
    k = min(k, NB - 3)
    _check(plan, qbar, kbar, k, None, NB, 3)


def test_fused_equals_separate_on_an_edge_grid():
    wl = workloads.custom(T=5, Hg=9, Wg=11, block=(4, 4, 4), n_prefix=70, H=2, topk=6)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    plan = vsa.Plan.of(wl)
    keep = torch.from_numpy((np.random.default_rng(42).random((1, 2, g.NB)) > 0.1).astype(np.uint8)).cuda()
    q, k, v = (H.to_dev(inp[n]) for n in ("q", "k", "v"))
    ws = vsa.workspace(1, 2)
    fused = vsa.tile_coarse_prefix(plan, q, k, v, 6, ws, keep)
    qt, qb = vsa.tile(plan, q, pooled=True)
    kt, kb = vsa.tile(plan, k, pooled=True)
    idx, num = vsa.coarse_topk_prefix(plan, qb, kb, 6, keep)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    assert torch.equal(fused["idx"], idx) and torch.equal(fused["num"], num)
    assert torch.equal(fused["qbar"].view(torch.int32), qb.view(torch.int32))
    assert torch.equal(fused["qt"].view(torch.int16), qt.view(torch.int16))
    assert int(ws.abs().sum()) == 0
    ridx, rnum = oracle.topk_prefix(oracle.score(oracle.pool(g, oracle.tile(g, inp["q"])),
                                                 oracle.pool(g, oracle.tile(g, inp["k"]))), g.n_pre, 6,
                                    keep.cpu().numpy())
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
