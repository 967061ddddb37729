"""GPU parity of the gate-compress branch ("FastVideo VSA", section "Checkpoint
behavior"; FastVideo commit log: the gate-compress branch pools per tile).

Reading under test: o_compress[r] = sum_c softmax_c(D^-1/2 qbar_r . kbar_c) vbar_c
over all blocks of the head, and o = o_fine + gate * o_compress[block(token)].

Tolerances:
* o_compress (fp32 weights and sums against fp64): 2e-4 absolute.  The
  fp32 score of a block pair carries a rounding error of order
  D * 2^-24 * |qbar| |kbar| (~2e-4 for |qbar| |kbar| ~ 32), which moves a
  weight by ~scale * 2e-4 relative; times |vbar| <= ~3 this stays below 1e-4.
* the gated output keeps the fine stage's tolerances (o max-abs 2e-2,
  mean-abs 2e-3 against fp64), its values being a bf16/fp16 rounding of
  o_fine + gate * o_compress.
* untile_gate alone: one fp32 fused multiply-add then one rounding to the
  16-bit format, so each result lies within 0.5 ulp of the exact value plus
  the fp32 rounding (< 2^-13 ulp of the 16-bit format).
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

OC_ABS = 2e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()


TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def _dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TDT[dtype])


def _host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _oracle_means(wl, dtype="bf16"):
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype=dtype, gate=True)
    tiled = [oracle.tile(g, inp[n]) for n in ("q", "k", "v")]
    means = [oracle.pool(g, t, dtype) for t in tiled]
    return g, inp, tiled, means


@pytest.mark.parametrize("name", ["tiny", "fastwan", "long"])
def test_compress_and_selection_from_oracle_means(name):
    """Oracle block means in, GPU branch out: o_compress within tolerance and the
    fused selection bit-identical to the oracle's top-k."""
    wl = workloads.WORKLOADS[name]
    g, _, _, (qb, kb, vb) = _oracle_means(wl)
    plan = vsa.Plan.of(wl)
    oc, idx, num = vsa.coarse_compress(plan, torch.from_numpy(qb).cuda(), torch.from_numpy(kb).cuda(),
                                       torch.from_numpy(vb).cuda(), wl.topk)
    torch.cuda.synchronize()
    ref_idx, ref_num = oracle.topk(oracle.score(qb, kb), wl.topk)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(num.cpu().numpy(), ref_num)
    ref = oracle.compress(qb, kb, vb)
    err = np.abs(oc.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= OC_ABS, err


def test_compress_alone_matches_fused_launch():
    """topk = 0 (selection from a block map) gives the same o_compress bit for bit."""
    wl = workloads.WORKLOADS["tile64"]
    g, _, _, means = _oracle_means(wl)
    plan = vsa.Plan.of(wl)
    qb, kb, vb = (torch.from_numpy(m).cuda() for m in means)
    alone = vsa.coarse_compress(plan, qb, kb, vb, 0)
    fused, _, _ = vsa.coarse_compress(plan, qb, kb, vb, 16)
    torch.cuda.synchronize()
    assert torch.equal(alone, fused)
    err = np.abs(alone.cpu().numpy().astype(np.float64) - oracle.compress(*means)).max()
    assert err <= OC_ABS, err


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("shape", [((5, 9, 11), (4, 8, 8), 0), ((6, 5, 7), (4, 4, 4), 70)])
def test_untile_gate_rounds_once(shape, dtype):
    (T, Hg, Wg), block, npre = shape
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, B=2, H=3)
    g = oracle.geometry_of(wl)
    rng = np.random.default_rng(30)
    to16 = workloads.f32_to_f16_bits if dtype == "f16" else workloads.f32_to_bf16_bits
    ot = to16(rng.standard_normal((2, 3, g.Sp, 128)).astype(np.float32))
    gate = to16(rng.standard_normal((2, g.S, 3, 128)).astype(np.float32) * 2)
    oc = rng.standard_normal((2, 3, g.NB, 128)).astype(np.float32)
    plan = vsa.Plan.of(wl)
    o = vsa.untile_gate(plan, _dev(ot, dtype), torch.from_numpy(oc).cuda(), _dev(gate, dtype))
    torch.cuda.synchronize()
    got_t = oracle.tile(g, _host(o))  # back to tiled rows through the oracle's tiling
    real = np.flatnonzero(H.real_rows(wl))
    rows = np.concatenate([bh * g.Sp + real for bh in range(6)])
    o_fine = oracle.half_to_f32(ot, dtype).reshape(-1, 128)[rows].astype(np.float64)
    exact = oracle.gate_rows(g, rows, o_fine, gate, oc.astype(np.float64), dtype)
    got = oracle.half_to_f32(got_t, dtype).reshape(-1, 128)[rows].astype(np.float64)
    mant = 8 if dtype == "bf16" else 11
    # ulp of the 16-bit format at the exact value (normal range; fp16 subnormals share 2^-24)
    e = np.floor(np.log2(np.maximum(np.abs(exact), 1e-30)))
    ulp = np.exp2(e - (mant - 1))
    if dtype == "f16":
        ulp = np.maximum(ulp, 2.0 ** -24)
    ratio = np.abs(got - exact) / ulp
    assert ratio.max() <= 0.5 + 2.0 ** -13, ratio.max()
    # padded slots of the tiled input never reach the output: rows of o are exactly the real tokens
    assert _host(o).shape == (2, g.S, 3, 128)


@pytest.mark.parametrize("name,dtype", [("tiny", "bf16"), ("fastwan", "bf16"), ("wan81", "f16"), ("tile64", "bf16")])
def test_gated_forward_full_size(name, dtype):
    """vsa.Forward(gated=True) against the oracle: fine stage on sampled real rows
    (every row for tiny) plus gate * o_compress of the row's block."""
    wl = workloads.WORKLOADS[name]
    g, inp, (qt, kt, vt), (qb, kb, vb) = _oracle_means(wl, dtype)
    if wl.map_driven:
        idx, num = oracle.map_to_index(inp["map"])
    else:
        idx, num = oracle.topk(oracle.score(qb, kb), wl.topk)
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, dtype=TDT[dtype], gated=True)
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    o, lse = fwd(_dev(inp["q"], dtype), _dev(inp["k"], dtype), _dev(inp["v"], dtype), bmap,
                 gate=_dev(inp["gate"], dtype))
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    np.testing.assert_array_equal(fwd.idx.cpu().numpy(), idx)
    np.testing.assert_array_equal(fwd.num.cpu().numpy(), num)
    np.testing.assert_array_equal(fwd.vbar.cpu().numpy().view(np.uint32), vb.view(np.uint32))
    oc_ref = oracle.compress(qb, kb, vb)
    assert np.abs(fwd.oc.cpu().numpy() - oc_ref).max() <= OC_ABS
    real = np.flatnonzero(H.real_rows(wl))
    if name == "tiny":
        rows = np.concatenate([bh * g.Sp + real for bh in range(wl.B * wl.H)])
    else:
        rng = np.random.default_rng(31)
        rows = np.concatenate([bh * g.Sp + np.unique(np.concatenate(
            [rng.choice(real, 40, replace=False), real[:2], real[-2:]])) for bh in range(wl.B * wl.H)])
    o_fine, _ = oracle.attn_rows(g, qt, kt, vt, idx, num, rows, dtype)
    expect = oracle.gate_rows(g, rows, o_fine, inp["gate"], oc_ref, dtype)
    got = oracle.half_to_f32(oracle.tile(g, _host(o)), dtype).reshape(-1, 128)[rows].astype(np.float64)
    err = np.abs(got - expect)
    assert err.max() <= H.O_MAX_ABS and err.mean() <= H.O_MEAN_ABS, (err.max(), err.mean())
