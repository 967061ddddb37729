"""Pins of the oracle's fp16 path ("FastVideo VSA", section "Verify routing and
fallback": the kernel takes FP16 or BF16 tensors)."""
import numpy as np
import torch

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import block_mask, dense_masked_attention, tile_by_reshape, valid_slots_by_reshape


def test_fp16_conversion_exhaustive():
    """Every one of the 65536 fp16 patterns converts like numpy's float16 (nan as nan)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_f32(bits, "f16")
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_conversion_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_f32(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_fp16_rounding_of_the_generator():
    x = np.array([1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, -2.5, 0.0, 65504.0], dtype=np.float32)
    np.testing.assert_array_equal(workloads.f32_to_f16_bits(x).view(np.float16),
                                  torch.from_numpy(x).half().numpy())


def test_fp16_pool_matches_fp64_mean():
    wl = workloads.custom(T=7, Hg=13, Wg=11, H=2, D=32)
    inp = workloads.make_inputs(wl, threads=1, dtype="f16")
    g = oracle.geometry_of(wl)
    p = oracle.pool(g, oracle.tile(g, inp["q"]), "f16").astype(np.float64)
    xf = inp["q"].view(np.float16).astype(np.float64)
    t = tile_by_reshape(xf, wl.T, wl.Hg, wl.Wg, wl.block).reshape(1, 2, g.NB, g.bs, 32)
    valid = valid_slots_by_reshape(wl.T, wl.Hg, wl.Wg, wl.block).reshape(g.NB, g.bs)
    ref = (t * valid[None, None, :, :, None]).sum(axis=3) / valid.sum(axis=1)[None, None, :, None]
    bound = 256 * 2.0 ** -24 * np.abs(t).sum(axis=3).max() + 1e-7
    assert np.abs(p - ref).max() <= bound


def test_fp16_attention_matches_dense_masked():
    wl = workloads.custom(T=5, Hg=9, Wg=9, H=1, D=64)
    inp = workloads.make_inputs(wl, threads=1, dtype="f16")
    g = oracle.geometry_of(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(20)
    num = rng.integers(0, 4, size=(1, 1, g.NB)).astype(np.int32)
    idx = np.full((1, 1, g.NB, 3), -1, dtype=np.int32)
    for r in range(g.NB):
        idx[0, 0, r, :num[0, 0, r]] = np.sort(rng.permutation(g.NB)[:num[0, 0, r]])
    o, lse = oracle.attn(g, qt, kt, vt, idx, num, "f16")
    f = lambda a: a[0, 0].view(np.float16).astype(np.float64)
    valid = valid_slots_by_reshape(5, 9, 9, (4, 8, 8))
    ro, rl = dense_masked_attention(f(qt), f(kt), f(vt), block_mask(idx[0, 0], num[0, 0], g.NB, g.bs, valid))
    np.testing.assert_allclose(o[0, 0], ro, rtol=0, atol=1e-12)
    fin = np.isfinite(rl)
    np.testing.assert_array_equal(np.isfinite(lse[0, 0]), fin)
    np.testing.assert_allclose(lse[0, 0][fin], rl[fin], rtol=0, atol=1e-12)
