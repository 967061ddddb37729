"""Pins of the oracle's gate-compress (coarse) branch.

Sources: "FastVideo VSA" (vLLM-Omni user guide), section "Checkpoint
behavior" (checkpoints carry a learned gate_compress projection) and the
FastVideo commit log, examples/inference/basic/README.md (the gate-compress
branch pools per tile).  The pages print no formula; the reading pinned here
is dense attention among the block means of a head (scale D^-1/2), broadcast
to every token of the query block, times the caller's gate, added to the
sparse branch.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import tile_by_reshape, valid_slots_by_reshape


def _means(rng, B, H, NB, D, scale=1.0):
    return [(rng.standard_normal((B, H, NB, D)) * scale).astype(np.float32) for _ in range(3)]


def test_equals_library_attention_among_block_means():
    """The branch is softmax attention over NB 'tokens': torch's fp64 SDPA on CPU."""
    rng = np.random.default_rng(0)
    for B, H, NB, D in [(1, 2, 8, 128), (2, 3, 37, 64), (1, 1, 300, 128)]:
        qb, kb, vb = _means(rng, B, H, NB, D, scale=2.0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qb).double(), torch.from_numpy(kb).double(), torch.from_numpy(vb).double())
        np.testing.assert_allclose(oracle.compress(qb, kb, vb), ref.numpy(), rtol=0, atol=1e-12)


def test_single_block_returns_its_mean():
    rng = np.random.default_rng(1)
    qb, kb, vb = _means(rng, 2, 2, 1, 128)
    assert np.array_equal(oracle.compress(qb, kb, vb), vb.astype(np.float64))


@pytest.mark.parametrize("case", ["zero_query", "equal_keys"])
def test_uniform_weights_give_the_mean_of_v(case):
    rng = np.random.default_rng(2)
    qb, kb, vb = _means(rng, 1, 2, 24, 128)
    if case == "zero_query":
        qb[:] = 0.0
    else:
        kb[:] = kb[:, :, :1]
    expect = np.broadcast_to(vb.astype(np.float64).mean(axis=2, keepdims=True), vb.shape)
    np.testing.assert_allclose(oracle.compress(qb, kb, vb), expect, rtol=0, atol=1e-12)


def test_dominant_block_is_selected():
    """Block j's key is a large multiple of row r's query: o[r] -> vbar[j]."""
    rng = np.random.default_rng(3)
    qb, kb, vb = _means(rng, 1, 1, 16, 128, scale=0.01)
    for r, j in [(0, 5), (7, 0), (15, 15)]:
        kb[0, 0, j] = qb[0, 0, r] * (1e4 / float(qb[0, 0, r] @ qb[0, 0, r]))
    out = oracle.compress(qb, kb, vb)
    for r, j in [(0, 5), (7, 0), (15, 15)]:
        np.testing.assert_allclose(out[0, 0, r], vb[0, 0, j], rtol=0, atol=1e-9)


def test_scale_is_inverse_sqrt_head_size():
    """Two blocks with logit gap g: weight of the first = 1 / (1 + exp(-g / sqrt(D)))."""
    D = 64
    qb = np.zeros((1, 1, 2, D), np.float32)
    kb = np.zeros((1, 1, 2, D), np.float32)
    vb = np.zeros((1, 1, 2, D), np.float32)
    qb[0, 0, :, 0] = 3.0
    kb[0, 0, 0, 0] = 2.0   # logit 6 / 8
    vb[0, 0, 0, 1] = 1.0   # channel 1 reads the first block's weight
    out = oracle.compress(qb, kb, vb)
    w = 1.0 / (1.0 + np.exp(-6.0 / np.sqrt(D)))
    np.testing.assert_allclose(out[0, 0, :, 1], [w, w], rtol=0, atol=1e-15)


def test_permutation_equivariance():
    rng = np.random.default_rng(4)
    qb, kb, vb = _means(rng, 1, 2, 20, 128)
    base = oracle.compress(qb, kb, vb)
    pk = rng.permutation(20)
    np.testing.assert_allclose(oracle.compress(qb, kb[:, :, pk], vb[:, :, pk]), base, rtol=0, atol=1e-12)
    pq = rng.permutation(20)
    np.testing.assert_allclose(oracle.compress(qb[:, :, pq], kb, vb), base[:, :, pq], rtol=0, atol=1e-12)


def test_heads_are_independent():
    rng = np.random.default_rng(5)
    qb, kb, vb = _means(rng, 2, 3, 10, 128)
    full = oracle.compress(qb, kb, vb)
    for b in range(2):
        for h in range(3):
            one = oracle.compress(qb[b:b + 1, h:h + 1], kb[b:b + 1, h:h + 1], vb[b:b + 1, h:h + 1])
            assert np.array_equal(one[0, 0], full[b, h])


BF16_ONE = 0x3F80
F16_ONE = 0x3C00


@pytest.mark.parametrize("shape", [((5, 9, 11), (4, 8, 8), 0), ((6, 5, 7), (4, 4, 4), 70)])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_gate_broadcasts_each_blocks_branch_to_its_tokens(shape, dtype):
    """o_compress[b,h,r,:] = (r+1) + 1000 h + 1e5 b in channel 0 and gate = 1:
    the gated term of a token names its block, head and batch; the block of
    every token comes from the reshape form of the tiling."""
    (T, Hg, Wg), block, npre = shape
    B, H, D = 2, 3, 8
    g = oracle.geometry(T, Hg, Wg, block, npre)
    oc = np.zeros((B, H, g.NB, D))
    for b in range(B):
        for h in range(H):
            oc[b, h, :, 0] = np.arange(1, g.NB + 1) + 1000 * h + 1e5 * b
    gate = np.full((B, g.S, H, D), BF16_ONE if dtype == "bf16" else F16_ONE, np.uint16)
    valid = valid_slots_by_reshape(T, Hg, Wg, block, npre)
    rows = np.array([bh * g.Sp + i for bh in range(B * H) for i in np.flatnonzero(valid)], np.int64)
    o_fine = np.zeros((len(rows), D))
    out = oracle.gate_rows(g, rows, o_fine, gate, oc, dtype)
    expect = oc.reshape(B * H * g.NB, D)[(rows // g.Sp) * g.NB + (rows % g.Sp) // g.bs]
    assert np.array_equal(out, expect)
    # and the token the gate is read from: a gate that encodes the token index
    S = g.S
    tok = np.arange(S, dtype=np.float32)[None, :, None, None] * np.ones((B, 1, H, 1), np.float32)
    gate2 = (workloads.f32_to_f16_bits if dtype == "f16" else workloads.f32_to_bf16_bits)(
        np.broadcast_to(tok % 64, (B, S, H, D)))
    tiled_tok = tile_by_reshape(np.broadcast_to(tok % 64, (B, S, H, D)).copy(), T, Hg, Wg, block, npre)
    oc1 = np.ones((B, H, g.NB, D))
    out2 = oracle.gate_rows(g, rows, o_fine, gate2, oc1, dtype)
    expect2 = tiled_tok.reshape(B * H * g.Sp, D)[rows].astype(np.float64)
    assert np.array_equal(out2, expect2)


def test_zero_gate_leaves_the_sparse_branch():
    g = oracle.geometry(4, 8, 8)
    rng = np.random.default_rng(6)
    rows = np.arange(g.Sp, dtype=np.int64)
    o_fine = rng.standard_normal((g.Sp, 16))
    out = oracle.gate_rows(g, rows, o_fine, np.zeros((1, g.S, 1, 16), np.uint16), rng.standard_normal((1, 1, 1, 16)))
    assert np.array_equal(out, o_fine)


def test_padded_row_is_rejected():
    g = oracle.geometry(3, 8, 8)  # the last temporal slot of the block is padding
    rows = np.array([g.Sp - 1], np.int64)
    with pytest.raises(ValueError):
        oracle.gate_rows(g, rows, np.zeros((1, 4)), np.zeros((1, g.S, 1, 4), np.uint16), np.zeros((1, 1, 1, 4)))
