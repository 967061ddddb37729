"""Pins of the oracle's fine stage (attention on selected blocks).

Sources: "FastVideo VSA" (vLLM-Omni user guide): introduction (each query
block attends only to its selected key/value blocks), section "Choose top-k"
(topk == num_blocks keeps every block, i.e. dense attention) and section
"Verify routing and fallback" (non-causal, equal lengths, scale
head_size^-1/2); FastVideo commit log, examples/inference/basic/README.md
(rows with zero count; "every tile selected" is exactly dense attention).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import block_mask, dense_masked_attention, valid_slots_by_reshape

f32 = workloads.bf16_bits_to_f32


def _tiled_inputs(wl):
    inp = workloads.make_inputs(wl, threads=1)
    g = oracle.geometry_of(wl)
    return g, inp, [oracle.tile(g, inp[n]) for n in ("q", "k", "v")]


def _random_selection(rng, B, H, NB, max_k, zero_rows=True):
    num = rng.integers(0 if zero_rows else 1, max_k + 1, size=(B, H, NB)).astype(np.int32)
    idx = np.full((B, H, NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(B, H, NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(NB)[:num[pos]])
    return idx, num


@pytest.mark.parametrize("shape", [((5, 9, 9), (4, 8, 8), 0), ((8, 8, 8), (4, 4, 4), 100)])
def test_matches_dense_attention_with_explicit_block_mask(shape):
    (T, Hg, Wg), block, npre = shape
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, H=2, D=64)
    g, inp, (qt, kt, vt) = _tiled_inputs(wl)
    rng = np.random.default_rng(10)
    idx, num = _random_selection(rng, 1, 2, g.NB, min(3, g.NB))
    o, lse = oracle.attn(g, qt, kt, vt, idx, num)
    valid = valid_slots_by_reshape(T, Hg, Wg, block, npre)
    for h in range(2):
        allowed = block_mask(idx[0, h], num[0, h], g.NB, g.bs, valid)
        ro, rl = dense_masked_attention(f32(qt[0, h]).astype(np.float64), f32(kt[0, h]).astype(np.float64),
                                        f32(vt[0, h]).astype(np.float64), allowed)
        np.testing.assert_allclose(o[0, h], ro, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse[0, h]), np.isinf(rl))
        fin = np.isfinite(rl)
        np.testing.assert_allclose(lse[0, h][fin], rl[fin], rtol=0, atol=1e-12)


def test_all_blocks_equals_torch_sdpa():
    """topk == NB: every block kept, so the result is dense attention over the real tokens;
    torch's scaled_dot_product_attention in fp64 on the untiled tokens is the reference."""
    wl = workloads.custom(T=5, Hg=9, Wg=9, H=2, D=128)
    g, inp, (qt, kt, vt) = _tiled_inputs(wl)
    idx = np.broadcast_to(np.arange(g.NB, dtype=np.int32), (1, 2, g.NB, g.NB)).copy()
    num = np.full((1, 2, g.NB), g.NB, dtype=np.int32)
    o, lse = oracle.attn(g, qt, kt, vt, idx, num)
    # pick the real rows with the reshape-form validity mask (not the oracle's untile)
    valid = valid_slots_by_reshape(5, 9, 9, (4, 8, 8))
    q = torch.from_numpy(f32(qt[0][:, valid]).astype(np.float64))
    k = torch.from_numpy(f32(kt[0][:, valid]).astype(np.float64))
    v = torch.from_numpy(f32(vt[0][:, valid]).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
    np.testing.assert_allclose(o[0][:, valid], ref, rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp((q @ k.transpose(-1, -2)) / np.sqrt(128), dim=-1).numpy()
    np.testing.assert_allclose(lse[0][:, valid], ref_lse, rtol=0, atol=1e-12)


def test_zero_count_rows():
    wl = workloads.custom(T=8, Hg=8, Wg=8, H=1, D=32)
    g, inp, (qt, kt, vt) = _tiled_inputs(wl)
    idx = np.array([[[[1], [-1]]]], dtype=np.int32)
    num = np.array([[[1, 0]]], dtype=np.int32)
    o, lse = oracle.attn(g, qt, kt, vt, idx, num)
    assert (o[0, 0, 256:] == 0).all() and np.isneginf(lse[0, 0, 256:]).all()
    assert np.isfinite(lse[0, 0, :256]).all()


def test_rows_of_softmax_sum_to_one():
    """With v = 1 everywhere, o = sum_j p_j = 1 for every non-empty row."""
    wl = workloads.custom(T=5, Hg=9, Wg=9, H=1, D=64)
    g, inp, (qt, kt, _) = _tiled_inputs(wl)
    ones = np.full(qt.shape, workloads.f32_to_bf16_bits(np.float32(1.0)), dtype=np.uint16)
    rng = np.random.default_rng(11)
    idx, num = _random_selection(rng, 1, 1, g.NB, 3, zero_rows=False)
    o, _ = oracle.attn(g, qt, kt, ones, idx, num)
    assert np.abs(o - 1.0).max() < 1e-12


def test_single_valid_key():
    """(5,9,9) has a corner block with one real token: selecting only it gives o = v of
    that token and lse = scale * q . k."""
    wl = workloads.custom(T=5, Hg=9, Wg=9, H=1, D=64)
    g, inp, (qt, kt, vt) = _tiled_inputs(wl)
    last = g.NB - 1
    assert oracle.block_valid_counts(g)[last] == 1
    idx = np.full((1, 1, g.NB, 1), last, dtype=np.int32)
    num = np.ones((1, 1, g.NB), dtype=np.int32)
    o, lse = oracle.attn(g, qt, kt, vt, idx, num)
    j = last * g.bs  # slot 0 of the corner block is its only real token
    vj = f32(vt[0, 0, j]).astype(np.float64)
    kj = f32(kt[0, 0, j]).astype(np.float64)
    q = f32(qt[0, 0]).astype(np.float64)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(vj, o[0, 0].shape), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], q @ kj / 8.0, rtol=0, atol=1e-12)


def test_identical_keys_average_values():
    """All real keys equal: every logit is the same, so o is the plain mean of the
    selected real values."""
    wl = workloads.custom(T=8, Hg=8, Wg=12, H=1, D=32)
    g, inp, (qt, kt, vt) = _tiled_inputs(wl)
    valid = valid_slots_by_reshape(8, 8, 12, (4, 8, 8))
    same = np.zeros_like(kt)
    same[0, 0, valid] = kt[0, 0, 0]
    idx = np.array([[[[0, 1], [0, 1], [1, 3], [2, 3]]]], dtype=np.int32)
    num = np.full((1, 1, 4), 2, dtype=np.int32)
    o, lse = oracle.attn(g, qt, same, vt, idx, num)
    v = f32(vt[0, 0]).astype(np.float64).reshape(g.NB, g.bs, 32)
    vm = valid.reshape(g.NB, g.bs)
    for r in range(g.NB):
        sel = idx[0, 0, r]
        mean = np.concatenate([v[b][vm[b]] for b in sel]).mean(axis=0)
        np.testing.assert_allclose(o[0, 0, r * g.bs:(r + 1) * g.bs], np.broadcast_to(mean, (g.bs, 32)),
                                   rtol=0, atol=1e-12)
