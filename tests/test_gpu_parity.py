"""GPU parity of every step of the forward path against the CPU oracle.

Bit-exact: tile, pooled means, untile, q2k_idx/q2k_num (coarse top-k and the
bool-map compaction).  Attention: o within max-abs 2e-2 and mean-abs 2e-3 of
the fp64 oracle, lse within 1e-3, on the same seeded inputs; the fine stage is
also run on oracle-supplied indices.  Small cases compare every row; the
full-size workloads compare the whole index and sampled rows of o / lse.
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

EDGE_SHAPES = [
    # (T, Hg, Wg, block, n_prefix): partial blocks on every axis, a one-token
    # corner block, a single block, tiles of 64 after a prefix.
    (8, 16, 16, (4, 8, 8), 0),
    (5, 9, 9, (4, 8, 8), 0),
    (7, 8, 16, (4, 8, 8), 0),
    (12, 20, 20, (4, 8, 8), 0),
    (4, 8, 8, (4, 8, 8), 0),
    (1, 1, 1, (4, 8, 8), 0),
    (8, 8, 8, (4, 4, 4), 128),
    (5, 6, 7, (4, 4, 4), 100),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()
    assert vsa.get_status() == vsa.VSA_OK


def _wl(shape, H_=2, **kw):
    T, Hg, Wg, block, npre = shape
    return workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, H=H_, **kw)


def _bits32(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


@pytest.mark.parametrize("shape", EDGE_SHAPES)
def test_tile_pool_untile_bit_exact(shape):
    wl = _wl(shape, H_=3, B=2)
    g = oracle.geometry_of(wl)
    plan = vsa.Plan.of(wl)
    x = H.inputs(wl)["q"]
    xt, pooled = vsa.tile(plan, H.to_dev(x), pooled=True)
    ref_t = oracle.tile(g, x)
    np.testing.assert_array_equal(H.from_dev(xt), ref_t)
    np.testing.assert_array_equal(_bits32(pooled.cpu().numpy()), _bits32(oracle.pool(g, ref_t)))
    xt_plain = vsa.tile(plan, H.to_dev(x))
    np.testing.assert_array_equal(H.from_dev(xt_plain), ref_t)
    # untile: padded rows hold garbage on purpose; they must be dropped
    rng = np.random.default_rng(5)
    junk = rng.integers(0, 0x7F00, size=ref_t.shape, dtype=np.uint16)
    back = vsa.untile(plan, H.to_dev(junk))
    np.testing.assert_array_equal(H.from_dev(back), oracle.untile(g, junk))
    np.testing.assert_array_equal(H.from_dev(vsa.untile(plan, xt)), x)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK


@pytest.mark.parametrize("name", ["tiny", "fastwan", "wan81", "long"])
def test_coarse_topk_bit_exact(name):
    wl = workloads.WORKLOADS[name]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    inp = H.inputs(wl)
    qt, qbar = vsa.tile(plan, H.to_dev(inp["q"]), pooled=True)
    kt, kbar = vsa.tile(plan, H.to_dev(inp["k"]), pooled=True)
    np.testing.assert_array_equal(_bits32(qbar.cpu().numpy()), _bits32(ref["qbar"]))
    np.testing.assert_array_equal(_bits32(kbar.cpu().numpy()), _bits32(ref["kbar"]))
    idx, num = vsa.coarse_topk(plan, qbar, kbar, wl.topk)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(num.cpu().numpy(), ref["num"])


@pytest.mark.parametrize("k", [1, 3, 8])
def test_coarse_topk_ties_and_extremes(k):
    """Scores with many exact ties (integer-valued pooled means) and k = 1 / NB."""
    rng = np.random.default_rng(12)
    plan = vsa.Plan(8, 16, 16)  # NB = 8
    qbar = rng.integers(-2, 3, size=(1, 3, 8, 128)).astype(np.float32)
    kbar = rng.integers(-2, 3, size=(1, 3, 8, 128)).astype(np.float32)
    kbar[0, 0] = 0.0  # a whole head of zero scores (also -0.0 products)
    qbar[0, 1, :, :] = -qbar[0, 1, :, :] * 0.0
    idx, num = vsa.coarse_topk(plan, torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), k)
    ref_idx, ref_num = oracle.topk(oracle.score(qbar, kbar), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(num.cpu().numpy(), ref_num)


def test_coarse_topk_large_random_many_rows():
    rng = np.random.default_rng(13)
    plan = vsa.Plan(81, 30, 52)  # NB = 588
    qbar = rng.standard_normal((1, 2, 588, 128)).astype(np.float32)
    kbar = rng.standard_normal((1, 2, 588, 128)).astype(np.float32)
    for k in (1, 59, 300, 588):
        idx, num = vsa.coarse_topk(plan, torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), k)
        ref_idx, ref_num = oracle.topk(oracle.score(qbar, kbar), k)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)


@pytest.mark.parametrize("shape", [(1, 1, 4, 4), (2, 3, 11, 13), (1, 2, 40, 100)])
def test_map_to_index_bit_exact(shape):
    rng = np.random.default_rng(14)
    m = rng.random(shape) < 0.3
    m[0, 0, 0] = False
    m[0, 0, -1] = True
    idx, num = vsa.map_to_index(torch.from_numpy(m).cuda())
    ref_idx, ref_num = oracle.map_to_index(m)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(num.cpu().numpy(), ref_num)


def test_map_to_index_tile64_workload():
    wl = workloads.WORKLOADS["tile64map"]
    m = H.inputs(wl)["map"]
    idx, num = vsa.map_to_index(torch.from_numpy(m).cuda())
    ref_idx, ref_num = oracle.map_to_index(m)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(num.cpu().numpy(), ref_num)


def _attn_vs_oracle(wl, idx, num, rows=None, what=""):
    """Fine stage on the oracle's tiled inputs and the given index; compare rows."""
    ref = H.oracle_front(wl)
    g = ref["g"]
    plan = vsa.Plan.of(wl)
    q, k, v = (H.to_dev(ref[n]) for n in ("qt", "kt", "vt"))
    o, lse = vsa.sparse_attn_fwd(plan, q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(num).cuda())
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    B, Hh = wl.B, wl.H
    real = H.real_rows(wl)
    if rows is None:
        rows = np.flatnonzero(np.tile(real, B * Hh))
    o_ref, lse_ref = oracle.attn_rows(g, ref["qt"], ref["kt"], ref["vt"], idx, num, rows)
    o_bits = H.from_dev(o).reshape(-1, 128)[rows]
    lse_gpu = lse.cpu().numpy().reshape(-1)[rows]
    return H.compare_o_lse(o_bits, lse_gpu, o_ref, lse_ref, what)


def test_attention_tiny_every_row():
    wl = workloads.WORKLOADS["tiny"]
    ref = H.oracle_front(wl)
    _attn_vs_oracle(wl, ref["idx"], ref["num"], what="tiny")


@pytest.mark.parametrize("shape", EDGE_SHAPES)
def test_attention_oracle_indices_nonuniform_rows(shape):
    """Random selections with per-row counts 0..max_k (zero rows included), on grids
    with partial blocks along every axis."""
    wl = _wl(shape, H_=2)
    g = oracle.geometry_of(wl)
    rng = np.random.default_rng(15)
    max_k = min(5, g.NB)
    num = rng.integers(0, max_k + 1, size=(1, 2, g.NB)).astype(np.int32)
    num.reshape(-1)[0] = max_k
    idx = np.full((1, 2, g.NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(1, 2, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    _attn_vs_oracle(wl, idx, num, what=str(shape))


def test_attention_all_blocks_is_dense():
    """topk == NB: the oracle here equals dense attention (pinned to fp64 SDPA)."""
    wl = _wl((12, 20, 20, (4, 8, 8), 0), H_=2)
    g = oracle.geometry_of(wl)
    idx = np.broadcast_to(np.arange(g.NB, dtype=np.int32), (1, 2, g.NB, g.NB)).copy()
    num = np.full((1, 2, g.NB), g.NB, dtype=np.int32)
    _attn_vs_oracle(wl, idx, num, what="all blocks")


def test_attention_unsorted_and_repeated_ids_follow_the_list():
    """The fine stage takes the list as given (order free); results match the oracle."""
    wl = _wl((8, 16, 16, (4, 8, 8), 0), H_=1)
    idx = np.array([[[[7, 0, 3], [2, 5, 1], [6, 6, 4], [0, 1, 2], [3, 2, 1], [4, 5, 6], [7, 3, 0], [1, 0, 5]]]],
                   dtype=np.int32)
    num = np.full((1, 1, 8), 3, dtype=np.int32)
    _attn_vs_oracle(wl, idx, num, what="unsorted")


def test_zero_count_rows_give_zero_and_neg_inf():
    wl = workloads.WORKLOADS["tiny"]
    ref = H.oracle_front(wl)
    num = ref["num"].copy()
    num[0, 0, ::2] = 0
    _attn_vs_oracle(wl, ref["idx"], num, what="zero rows")


def test_bad_index_is_reported_and_skipped():
    wl = workloads.WORKLOADS["tiny"]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    idx = ref["idx"].copy()
    idx[0, 1, 3, 0] = 99   # out of range: skipped
    q, k, v = (H.to_dev(ref[n]) for n in ("qt", "kt", "vt"))
    o, lse = vsa.sparse_attn_fwd(plan, q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(ref["num"]).cuda())
    assert vsa.get_status() == vsa.VSA_ERR_BAD_INDEX
    assert vsa.get_status() == vsa.VSA_OK  # cleared by the read
    # rows of other blocks are unaffected
    rows = np.arange(0, 256 * 3)
    o_ref, lse_ref = oracle.attn_rows(ref["g"], ref["qt"], ref["kt"], ref["vt"], ref["idx"], ref["num"], rows)
    H.compare_o_lse(H.from_dev(o).reshape(-1, 128)[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref)


def _sample_rows(wl, n_per_head, seed):
    rng = np.random.default_rng(seed)
    g = oracle.geometry_of(wl)
    real = np.flatnonzero(H.real_rows(wl))
    rows = []
    for bh in range(wl.B * wl.H):
        pick = rng.choice(real, size=n_per_head, replace=False)
        pick = np.concatenate([pick, real[-2:], real[:2]])  # both ends of the sequence
        rows.append(bh * g.Sp + np.unique(pick))
    return np.concatenate(rows)


@pytest.mark.parametrize("name", ["tiny", "fastwan", "wan81", "long", "tile64", "tile64map"])
def test_full_path_full_size(name):
    """The launch configuration the benchmark times (vsa.Forward) at full size:
    indices bit-exact, o/lse on sampled real rows, untile of o bit-exact.
    tile64 computes the tile-64 selection (prefix tiles dense, video tiles the
    prefix + top-32, forced-empty rows); tile64map takes a caller-supplied bool
    block map through map_to_index."""
    wl = workloads.WORKLOADS[name]
    ref = H.oracle_front(wl)
    inp = H.inputs(wl)
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, prefix_dense=wl.prefix_dense)
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    keep = torch.from_numpy(inp["row_keep"]).cuda() if inp["row_keep"] is not None else None
    o, lse = fwd(H.to_dev(inp["q"]), H.to_dev(inp["k"]), H.to_dev(inp["v"]), bmap, row_keep=keep)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    np.testing.assert_array_equal(fwd.idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(fwd.num.cpu().numpy(), ref["num"])
    np.testing.assert_array_equal(H.from_dev(fwd.qt), ref["qt"])
    rows = _sample_rows(wl, 48 if name != "tiny" else 200, seed=16)
    if wl.map_driven or wl.prefix_dense:  # include rows of zero-count tiles and of dense prefix tiles
        g = ref["g"]
        zero = np.flatnonzero(ref["num"].reshape(-1) == 0)[:8]
        extra = [(z // g.NB) * g.Sp + (z % g.NB) * g.bs + np.arange(0, g.bs, 9) for z in zero]
        extra += [bh * g.Sp + np.arange(0, g.n_pre * g.bs, 37) for bh in range(wl.B * wl.H)]
        rows = np.unique(np.concatenate([rows] + extra))
    o_ref, lse_ref = oracle.attn_rows(ref["g"], ref["qt"], ref["kt"], ref["vt"], ref["idx"], ref["num"], rows)
    ot_bits = H.from_dev(fwd.ot).reshape(-1, 128)
    H.compare_o_lse(ot_bits[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref, name)
    np.testing.assert_array_equal(H.from_dev(o), oracle.untile(ref["g"], H.from_dev(fwd.ot)))


@pytest.mark.parametrize("shape,H_,k", [((15, 14, 15, (4, 8, 8), 0), 24, 8), ((31, 22, 40, (4, 8, 8), 0), 2, 64),
                                        ((5, 6, 7, (4, 4, 4), 100), 24, 6)])
def test_attention_many_items_per_cta(shape, H_, k):
    """More items than CTAs and long selections on grids with partial blocks (both
    block sizes): exercises item-to-item hand-offs inside a CTA."""
    wl = _wl(shape, H_=H_)
    g = oracle.geometry_of(wl)
    inp = H.inputs(wl)
    qt, kt = oracle.tile(g, inp["q"]), oracle.tile(g, inp["k"])
    idx, num = oracle.topk(oracle.score(oracle.pool(g, qt), oracle.pool(g, kt)), k)
    ref = dict(qt=qt, kt=kt, vt=oracle.tile(g, inp["v"]), g=g)
    rows = _sample_rows(wl, 24, seed=32)
    plan = vsa.Plan.of(wl)
    q, kk, v = (H.to_dev(ref[n]) for n in ("qt", "kt", "vt"))
    o, lse = vsa.sparse_attn_fwd(plan, q, kk, v, torch.from_numpy(idx).cuda(), torch.from_numpy(num).cuda())
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    o_ref, lse_ref = oracle.attn_rows(g, ref["qt"], ref["kt"], ref["vt"], idx, num, rows)
    H.compare_o_lse(H.from_dev(o).reshape(-1, 128)[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref,
                    f"many items {shape}")


@pytest.mark.parametrize("shape", [EDGE_SHAPES[1], EDGE_SHAPES[6]])
def test_attention_batch_of_two(shape):
    """B = 2: the fine stage indexes (b, h) rows correctly (per-row counts 0..max_k)."""
    wl = _wl(shape, H_=2, B=2)
    g = oracle.geometry_of(wl)
    rng = np.random.default_rng(33)
    max_k = min(4, g.NB)
    num = rng.integers(0, max_k + 1, size=(2, 2, g.NB)).astype(np.int32)
    idx = np.full((2, 2, g.NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(2, 2, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    _attn_vs_oracle(wl, idx, num, what=f"B2 {shape}")
