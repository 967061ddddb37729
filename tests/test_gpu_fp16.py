"""GPU parity of the fp16 path ("FastVideo VSA", section "Verify routing and
fallback": FP16 or BF16 tensors): tiling and pooled means bit-exact, indices
bit-exact, attention within the same tolerances as bf16."""
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


def _dev16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.float16)


def _host16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("shape", [((5, 9, 9), (4, 8, 8), 0), ((8, 8, 8), (4, 4, 4), 128)])
def test_fp16_tile_pool_bit_exact(shape):
    (T, Hg, Wg), block, npre = shape
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, H=3, B=2)
    g = oracle.geometry_of(wl)
    x = workloads.make_inputs(wl, dtype="f16")["q"]
    plan = vsa.Plan.of(wl)
    xt, pooled = vsa.tile(plan, _dev16(x), pooled=True)
    ref = oracle.tile(g, x)
    np.testing.assert_array_equal(_host16(xt), ref)
    np.testing.assert_array_equal(pooled.cpu().numpy().view(np.uint32), oracle.pool(g, ref, "f16").view(np.uint32))
    np.testing.assert_array_equal(_host16(vsa.untile(plan, xt)), x)


@pytest.mark.parametrize("name", ["tiny", "wan81", "fastwan", "long"])
def test_fp16_full_path(name):
    wl = workloads.WORKLOADS[name]
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype="f16")
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    (idx, num), _ = oracle.coarse(g, qt, kt, wl.topk, "f16")
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, dtype=torch.float16)
    o, lse = fwd(_dev16(inp["q"]), _dev16(inp["k"]), _dev16(inp["v"]))
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    np.testing.assert_array_equal(fwd.idx.cpu().numpy(), idx)
    np.testing.assert_array_equal(fwd.num.cpu().numpy(), num)
    real = np.flatnonzero(H.real_rows(wl))
    rng = np.random.default_rng(21)
    rows = np.concatenate([bh * g.Sp + rng.choice(real, min(300, len(real)), replace=False)
                           for bh in range(wl.B * wl.H)])
    o_ref, lse_ref = oracle.attn_rows(g, qt, kt, vt, idx, num, rows, "f16")
    o_gpu = _host16(fwd.ot).reshape(-1, 128)[rows].view(np.float16).astype(np.float64)
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= H.O_MAX_ABS and err.mean() <= H.O_MEAN_ABS, (err.max(), err.mean())
    lerr = np.abs(lse.cpu().numpy().reshape(-1)[rows] - lse_ref).max()
    assert lerr <= H.LSE_ABS, lerr
    np.testing.assert_array_equal(_host16(o), oracle.untile(g, _host16(fwd.ot)))
