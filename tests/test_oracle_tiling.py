"""Pins of the oracle's geometry, tile, untile and pool steps.

Sources: "FastVideo VSA" (vLLM-Omni user guide), introduction (blocks of the
post-patch latent grid) and section "Choose top-k" (block size (4, 8, 8), the
zero-padded block count and its worked example).
"""
import math
import os

import numpy as np
import pytest

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import tile_by_reshape, valid_slots_by_reshape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fastwan_route.txt")

SHAPES = [
    # (T, Hg, Wg, block, n_prefix): full blocks, partial blocks on each axis,
    # a one-token corner block, a single block, and prefix tiles.
    (8, 16, 16, (4, 8, 8), 0),
    (5, 9, 9, (4, 8, 8), 0),
    (7, 8, 16, (4, 8, 8), 0),
    (4, 13, 8, (4, 8, 8), 0),
    (4, 8, 11, (4, 8, 8), 0),
    (4, 8, 8, (4, 8, 8), 0),
    (1, 1, 1, (4, 8, 8), 0),
    (8, 8, 8, (4, 4, 4), 128),
    (5, 6, 7, (4, 4, 4), 100),
]


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            key, *rest = line.split()
            vals[key] = [float(x) if "." in x else int(x) for x in rest]
    return vals


def test_worked_example_route_log():
    """The page prints num_blocks=120 and keep_ratio=53.3% for (31,22,40), (4,8,8), topk 64."""
    gv = _golden()
    T, Hg, Wg = gv["dit_seq_shape"]
    g = oracle.geometry(T, Hg, Wg, tuple(gv["block_size"]))
    assert g.S == gv["seq_len"][0]
    assert g.NB == gv["num_blocks"][0]
    keep = round(100.0 * gv["topk"][0] / g.NB, 1)
    assert keep == gv["keep_ratio_percent"][0]


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_block_count_by_enumeration(name):
    """Every block of the padded grid holds at least one real token, so NB equals the
    number of distinct (t//bt, y//bh, x//bw) triples, plus the prefix tiles."""
    wl = workloads.WORKLOADS[name]
    g = oracle.geometry_of(wl)
    bt, bh, bw = wl.block
    t, y, x = np.meshgrid(np.arange(wl.T) // bt, np.arange(wl.Hg) // bh, np.arange(wl.Wg) // bw,
                          indexing="ij")
    distinct = len(set(zip(t.ravel().tolist(), y.ravel().tolist(), x.ravel().tolist())))
    pre = len(set((np.arange(wl.n_prefix) // (bt * bh * bw)).tolist()))
    assert g.NB == distinct + pre == wl.num_blocks
    assert g.S == wl.seq_len and g.Sp == g.NB * g.bs


def test_config_block_counts():
    """NB for the workloads as stated with them: 8, 120, 168, 264 tiles, 588."""
    got = {n: oracle.geometry_of(w).NB for n, w in workloads.WORKLOADS.items()}
    assert got == {"tiny": 8, "fastwan": 120, "wan81": 168, "tile64": 264, "tile64map": 264, "long": 588}


@pytest.mark.parametrize("shape", SHAPES)
def test_valid_counts_match_reshape(shape):
    T, Hg, Wg, block, npre = shape
    g = oracle.geometry(T, Hg, Wg, block, npre)
    counts = oracle.block_valid_counts(g)
    valid = valid_slots_by_reshape(T, Hg, Wg, block, npre)
    assert counts.sum() == g.S
    assert (counts >= 1).all()
    np.testing.assert_array_equal(counts, valid.reshape(g.NB, g.bs).sum(axis=1))


@pytest.mark.parametrize("shape", SHAPES)
def test_tile_matches_reshape_form(shape):
    T, Hg, Wg, block, npre = shape
    g = oracle.geometry(T, Hg, Wg, block, npre)
    rng = np.random.default_rng(1)
    B, H, D = 2, 3, 16
    x = rng.integers(1, 65535, size=(B, g.S, H, D), dtype=np.uint16)
    xt = oracle.tile(g, x)
    np.testing.assert_array_equal(xt, tile_by_reshape(x, T, Hg, Wg, block, npre))
    # padded rows are zero, real rows are never zero here (inputs are >= 1)
    valid = valid_slots_by_reshape(T, Hg, Wg, block, npre)
    assert (xt[:, :, ~valid] == 0).all()
    assert (xt[:, :, valid] != 0).all()


@pytest.mark.parametrize("shape", SHAPES)
def test_untile_inverts_tile(shape):
    T, Hg, Wg, block, npre = shape
    g = oracle.geometry(T, Hg, Wg, block, npre)
    rng = np.random.default_rng(2)
    x = rng.integers(0, 65536, size=(1, g.S, 2, 8), dtype=np.uint16)
    np.testing.assert_array_equal(oracle.untile(g, oracle.tile(g, x)), x)


def test_tile_is_token_bijection():
    """Tag each token with its own id; each id lands in exactly one slot."""
    g = oracle.geometry(5, 9, 9, (4, 8, 8))
    ids = np.arange(1, g.S + 1, dtype=np.uint16)
    x = ids.reshape(1, g.S, 1, 1)
    xt = oracle.tile(g, x)[0, 0, :, 0]
    nz = xt[xt != 0]
    assert len(nz) == g.S and len(set(nz.tolist())) == g.S


def test_block_order_and_slot_order():
    """Block (bT,bH,bW) sits at ((bT*nH + bH)*nW + bW); token (lt,lh,lw) at (lt*bh + lh)*bw + lw."""
    g = oracle.geometry(8, 16, 24, (4, 8, 8))  # nT=2, nH=2, nW=3
    T, Hg, Wg = 8, 16, 24
    ids = np.arange(g.S, dtype=np.uint16).reshape(1, g.S, 1, 1)
    xt = oracle.tile(g, ids + 1)[0, 0, :, 0].astype(np.int64) - 1
    for (t, y, x) in [(0, 0, 0), (5, 9, 17), (7, 15, 23), (3, 8, 7), (4, 0, 8)]:
        blk = ((t // 4) * 2 + y // 8) * 3 + x // 8
        slot = ((t % 4) * 8 + y % 8) * 8 + x % 8
        assert xt[blk * 256 + slot] == (t * Hg + y) * Wg + x


def _bf16(v):
    return workloads.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))


def test_pool_constant_block_is_exact():
    g = oracle.geometry(5, 9, 9, (4, 8, 8))
    x = np.broadcast_to(_bf16(0.75), (1, g.S, 1, 4)).copy()
    np.testing.assert_array_equal(oracle.pool(g, oracle.tile(g, x)), np.full((1, 1, g.NB, 4), 0.75, np.float32))


def test_pool_one_hot_divides_by_valid_count():
    g = oracle.geometry(5, 9, 9, (4, 8, 8))
    counts = oracle.block_valid_counts(g)
    x = np.zeros((1, g.S, 1, 1), dtype=np.uint16)
    x[0, g.S - 1, 0, 0] = _bf16(3.0).item()  # last token: the one-token corner block
    p = oracle.pool(g, oracle.tile(g, x))[0, 0, :, 0]
    last = g.NB - 1
    assert counts[last] == 1 and p[last] == np.float32(3.0)
    x[0, 0, 0, 0] = _bf16(3.0).item()  # first token: a full block of 256
    p = oracle.pool(g, oracle.tile(g, x))[0, 0, :, 0]
    assert p[0] == np.float32(3.0) / np.float32(counts[0])


def test_pool_sums_in_slot_order_in_fp32():
    """A block holding 2^24, then 254 ones, then -2^24 in slot order: the fp32 running sum
    absorbs every 1 (2^24 + 1 rounds back to 2^24), so the mean is exactly 0.  Any other
    order or a wider accumulator gives 254/256."""
    g = oracle.geometry(4, 8, 8, (4, 8, 8))
    vals = np.ones(256, dtype=np.float32)
    vals[0], vals[255] = 2.0 ** 24, -(2.0 ** 24)
    x = _bf16(vals).reshape(1, 256, 1, 1)  # one block; slot order == token order here
    p = oracle.pool(g, oracle.tile(g, x))
    assert p[0, 0, 0, 0] == 0.0


def test_pool_matches_fp64_mean():
    wl = workloads.custom(T=7, Hg=13, Wg=11, H=2, D=32)
    inp = workloads.make_inputs(wl, threads=1)
    g = oracle.geometry_of(wl)
    p = oracle.pool(g, oracle.tile(g, inp["q"])).astype(np.float64)
    xf = workloads.bf16_bits_to_f32(inp["q"]).astype(np.float64)
    tiled = tile_by_reshape(xf, wl.T, wl.Hg, wl.Wg, wl.block)
    valid = valid_slots_by_reshape(wl.T, wl.Hg, wl.Wg, wl.block).reshape(g.NB, g.bs)
    t = tiled.reshape(1, 2, g.NB, g.bs, 32)
    ref = (t * valid[None, None, :, :, None]).sum(axis=3) / valid.sum(axis=1)[None, None, :, None]
    # sequential fp32 sum of n terms: error <= n * 2^-24 * sum|x| (+ one division)
    bound = 256 * 2.0 ** -24 * np.abs(t).sum(axis=3).max() + 1e-7
    assert np.abs(p - ref).max() <= bound


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(10000) * 10).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0]  # ties to even
    ours = workloads.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
