"""Failure detection without a GPU fault: a bounded wait that runs out.

The one-launch front end's score items wait (at most 2 s) for the tile items
of their head to announce their block means on a counter in the caller's
workspace.  A counter preset far below zero never reaches its target, so the
wait runs out: the kernel records VSA_ERR_TIMEOUT, the waiting items return,
every other item finishes, and the host reads the status.  The context stays
usable: the next calls give the normal results.
"""
import numpy as np
import pytest
import torch

import block_sparse_video_gather_b200 as vsa
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


def test_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable():
    wl = workloads.WORKLOADS["tiny"]  # B1 H2, 8 blocks: one score item per head
    inp = H.inputs(wl)
    plan = vsa.Plan.of(wl)
    q, k, v = (H.to_dev(inp[n]) for n in ("q", "k", "v"))
    assert vsa.get_status() == vsa.VSA_OK
    ws = vsa.workspace(wl.B, wl.H)
    ws[0] = -(1 << 30)  # head 0's arrivals can never reach their target
    vsa.tile_coarse(plan, q, k, v, wl.topk, ws)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_ERR_TIMEOUT
    assert vsa.get_status() == vsa.VSA_OK  # read and cleared
    # the context is intact: a fresh workspace gives the oracle's selection again
    ref = H.oracle_front(wl)
    ws2 = vsa.workspace(wl.B, wl.H)
    out = vsa.tile_coarse(plan, q, k, v, wl.topk, ws2)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    np.testing.assert_array_equal(out["idx"].cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(H.from_dev(out["qt"]), ref["qt"])
    assert int(ws2.abs().sum()) == 0
