"""Pins of the oracle's block score, top-k and bool-map compaction.

Sources: "FastVideo VSA" (vLLM-Omni user guide), introduction (each query
block scores the key/value blocks and keeps its top-k) and sections "Enable
the backend" / "Choose top-k" (0 < topk <= num_blocks, top-k counts blocks);
FastVideo commit log, examples/inference/basic/README.md (bool block map
compacted by map_to_index; rows of different and zero length).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_sparse_video_gather_b200 import workloads


def test_score_small_integers_exact():
    rng = np.random.default_rng(4)
    q = rng.integers(-8, 9, size=(2, 3, 5, 16)).astype(np.float32)
    k = rng.integers(-8, 9, size=(2, 3, 5, 16)).astype(np.float32)
    s = oracle.score(q, k)
    ref = np.einsum("bhid,bhjd->bhij", q.astype(np.int64), k.astype(np.int64))
    np.testing.assert_array_equal(s, ref.astype(np.float32))


def test_score_uses_single_rounding_per_channel():
    """acc = fma(q1, k1, fma(q0, k0, 0)): with q0 k0 = -1 and q1 = k1 = 1 + 2^-12 the exact
    product 1 + 2^-11 + 2^-24 survives into the sum; a separate multiply would round it
    away and give 2^-11."""
    a = np.float32(1.0 + 2.0 ** -12)
    q = np.array([[[[1.0, a]]]], dtype=np.float32)
    k = np.array([[[[-1.0, a]]]], dtype=np.float32)
    s = oracle.score(q, k)[0, 0, 0, 0]
    exact = Fraction(-1) + Fraction(float(a)) ** 2
    assert Fraction(float(s)) == exact == Fraction(2 ** -11) + Fraction(2 ** -24)


def test_score_close_to_fp64_dot():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 2, 7, 128)).astype(np.float32)
    k = rng.standard_normal((1, 2, 7, 128)).astype(np.float32)
    s = oracle.score(q, k).astype(np.float64)
    ref = np.einsum("bhid,bhjd->bhij", q.astype(np.float64), k.astype(np.float64))
    bound = 128 * 2.0 ** -24 * np.einsum("bhid,bhjd->bhij", np.abs(q), np.abs(k)).max()
    assert np.abs(s - ref).max() <= bound


def _brute_topk(s, k):
    NB = s.shape[-1]
    idx = np.empty(s.shape[:-1] + (k,), dtype=np.int32)
    for pos in np.ndindex(*s.shape[:-1]):
        order = sorted(range(NB), key=lambda j: (-float(s[pos][j]), j))
        idx[pos] = sorted(order[:k])
    return idx


@pytest.mark.parametrize("k", [1, 3, 6, 9])
def test_topk_brute_force_with_ties(k):
    rng = np.random.default_rng(6)
    s = rng.integers(-3, 4, size=(2, 2, 9, 9)).astype(np.float32)  # many exact ties
    idx, num = oracle.topk(s, k)
    np.testing.assert_array_equal(idx, _brute_topk(s, k))
    assert (num == k).all()


def test_topk_ties_go_to_lower_index():
    s = np.zeros((1, 1, 4, 6), dtype=np.float32)
    s[0, 0, :, :] = [1, 2, 2, 2, 0, 2]
    idx, _ = oracle.topk(np.ascontiguousarray(np.broadcast_to(s[..., :4], (1, 1, 4, 4))), 2)
    # row [1, 2, 2, 2] -> the two highest tie; the lower indices 1 and 2 win
    np.testing.assert_array_equal(idx[0, 0, 0], [1, 2])
    s6 = np.zeros((1, 1, 6, 6), dtype=np.float32)
    s6[0, 0, :] = [1, 2, 2, 2, 0, 2]
    idx6, _ = oracle.topk(s6, 3)
    np.testing.assert_array_equal(idx6[0, 0, 0], [1, 2, 3])


def test_topk_negative_zero_ties_positive_zero():
    s = np.zeros((1, 1, 3, 3), dtype=np.float32)
    s[0, 0, :] = [np.float32(-0.0), 0.0, -1.0]
    idx, _ = oracle.topk(s, 1)
    np.testing.assert_array_equal(idx[0, 0, :, 0], [0, 0, 0])


def test_topk_all_blocks_is_identity():
    rng = np.random.default_rng(7)
    s = rng.standard_normal((1, 2, 8, 8)).astype(np.float32)
    idx, num = oracle.topk(s, 8)
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(8), idx.shape))


def test_topk_rejects_out_of_range_k():
    s = np.zeros((1, 1, 4, 4), dtype=np.float32)
    for bad in (0, -1, 5):
        with pytest.raises(ValueError):
            oracle.topk(s, bad)


def test_coarse_stage_finds_planted_blocks():
    """Give key block j the pooled direction of query block (j + 3) mod NB and make
    everything else small: each query block must select exactly that key block first,
    then the rest by the planted structure."""
    wl = workloads.custom(T=8, Hg=16, Wg=16, H=1, D=128, offset_std=0.0)
    g = oracle.geometry_of(wl)
    NB, bs = g.NB, g.bs
    rng = np.random.default_rng(8)
    dirs = np.linalg.qr(rng.standard_normal((128, NB)))[0].T.astype(np.float32)  # orthonormal rows
    qt = np.zeros((1, 1, g.Sp, 128), dtype=np.float32)
    kt = np.zeros((1, 1, g.Sp, 128), dtype=np.float32)
    for r in range(NB):
        qt[0, 0, r * bs:(r + 1) * bs] = 4 * dirs[r]
        kt[0, 0, ((r - 3) % NB) * bs:((r - 3) % NB + 1) * bs] = 4 * dirs[r]
    qb = workloads.f32_to_bf16_bits(qt)
    kb = workloads.f32_to_bf16_bits(kt)
    (idx, num), _ = oracle.coarse(g, qb, kb, 1)
    np.testing.assert_array_equal(idx[0, 0, :, 0], (np.arange(NB) - 3) % NB)


def test_map_to_index_brute_force():
    rng = np.random.default_rng(9)
    m = rng.random((2, 3, 11, 13)) < 0.3
    m[0, 0, 0] = False
    m[0, 0, 1] = True
    idx, num = oracle.map_to_index(m)
    for pos in np.ndindex(*m.shape[:-1]):
        sel = np.flatnonzero(m[pos])
        assert num[pos] == len(sel)
        np.testing.assert_array_equal(idx[pos][:len(sel)], sel)
        assert (idx[pos][len(sel):] == -1).all()
    assert num[0, 0, 0] == 0 and (idx[0, 0, 0] == -1).all()
    np.testing.assert_array_equal(idx[0, 0, 1], np.arange(13))


def test_map_workload_structure():
    """tile64map: prefix rows select all 264 tiles, video rows 8 + 32, 317 rows empty."""
    wl = workloads.WORKLOADS["tile64map"]
    m = workloads.make_inputs(wl)["map"]
    idx, num = oracle.map_to_index(m)
    counts = np.bincount(num.ravel(), minlength=265)
    assert counts[0] == round(0.05 * 24 * 264) == 317
    assert set(np.flatnonzero(counts).tolist()) == {0, 40, 264}
    video_rows = num[:, :, 8:]
    assert ((video_rows == 40) | (video_rows == 0)).all()
    nz = idx[:, :, 8:][video_rows == 40]
    assert (nz[:, :8] == np.arange(8)).all()


# ---- top-k with dense prefix tiles (FastVideo commit log, tile-64 layout:
# prefix query tiles dense, video query tiles the prefix + a top-k of video tiles)

def _check_prefix_selection(s, n_pre, k, keep, idx, num):
    """Characterise the answer without sorting: counts and layout fixed by the
    statement, and an exchange test -- every kept video tile beats every dropped
    one (higher score, or an equal score and a lower index)."""
    B, H, NB, _ = s.shape
    for b, h, r in np.ndindex(B, H, NB):
        row = idx[b, h, r]
        if keep is not None and not keep[b, h, r]:
            assert num[b, h, r] == 0 and (row == -1).all()
            continue
        if r < n_pre:
            assert num[b, h, r] == NB
            np.testing.assert_array_equal(row[:NB], np.arange(NB))
            continue
        c = int(num[b, h, r])
        assert c == n_pre + k
        np.testing.assert_array_equal(row[:n_pre], np.arange(n_pre))
        kept = row[n_pre:c]
        assert (np.diff(kept) > 0).all() and kept.min() >= n_pre and kept.max() < NB
        assert (row[c:] == -1).all()
        dropped = sorted(set(range(n_pre, NB)) - set(kept.tolist()))
        sv = s[b, h, r]
        for i in kept:
            for j in dropped:
                assert sv[i] > sv[j] or (sv[i] == sv[j] and i < j), (r, i, j)


@pytest.mark.parametrize("n_pre,k", [(0, 1), (0, 5), (1, 1), (3, 4), (3, 9), (2, 10)])
def test_topk_prefix_exchange_property_with_ties(n_pre, k):
    rng = np.random.default_rng(11)
    NB = 12
    s = rng.integers(-2, 3, size=(2, 2, NB, NB)).astype(np.float32)  # many exact ties
    keep = (rng.random((2, 2, NB)) > 0.2).astype(np.uint8)
    idx, num = oracle.topk_prefix(s, n_pre, k, keep)
    assert idx.shape == (2, 2, NB, NB if n_pre else k)
    _check_prefix_selection(s, n_pre, k, keep, idx, num)


def test_topk_prefix_without_prefix_is_plain_topk():
    """No prefix tiles and every row kept: the rule reduces to the coarse
    stage's top-k over all blocks (brute force above)."""
    rng = np.random.default_rng(12)
    s = rng.integers(-3, 4, size=(1, 2, 9, 9)).astype(np.float32)
    idx, num = oracle.topk_prefix(s, 0, 4)
    np.testing.assert_array_equal(idx, _brute_topk(s, 4))
    assert (num == 4).all()


def test_topk_prefix_all_video_tiles_is_dense():
    rng = np.random.default_rng(13)
    s = rng.standard_normal((1, 1, 7, 7)).astype(np.float32)
    idx, num = oracle.topk_prefix(s, 2, 5)
    assert (num == 7).all()
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(7), idx.shape))


def test_topk_prefix_ignores_prefix_scores():
    """A video row ranks video tiles only: huge prefix scores change nothing."""
    rng = np.random.default_rng(14)
    s = rng.standard_normal((1, 1, 10, 10)).astype(np.float32)
    idx, _ = oracle.topk_prefix(s, 3, 2)
    s2 = s.copy()
    s2[..., :3] = 1e30
    idx2, _ = oracle.topk_prefix(s2, 3, 2)
    np.testing.assert_array_equal(idx, idx2)
    # the best two of columns 3..9 of a row, by hand
    r = 5
    best = sorted(3 + np.argsort(-s[0, 0, r, 3:], kind="stable")[:2])
    np.testing.assert_array_equal(idx[0, 0, r, 3:5], best)


def test_topk_prefix_rejects_bad_arguments():
    s = np.zeros((1, 1, 6, 6), dtype=np.float32)
    for n_pre, k in ((2, 0), (2, 5), (6, 1), (-1, 1)):
        with pytest.raises(ValueError):
            oracle.topk_prefix(s, n_pre, k)
    with pytest.raises(ValueError):
        oracle.topk_prefix(s, 2, 2, max_k=5)  # prefix rows need all 6


def test_tile64_row_keep_structure():
    """tile64: 317 = round(0.05 * 24 * 264) rows forced empty, drawn from every row."""
    wl = workloads.WORKLOADS["tile64"]
    keep = workloads.make_inputs(wl)["row_keep"]
    assert keep.shape == (1, 24, 264) and keep.dtype == np.uint8
    assert int((keep == 0).sum()) == 317
    assert wl.max_k == 264 and not wl.map_driven and wl.prefix_dense


def test_coarse_prefix_stage_finds_planted_blocks():
    """Planted pooled directions: video query block r's best video key block is
    the one carrying its direction, whatever the prefix tiles hold."""
    wl = workloads.custom(T=4, Hg=8, Wg=16, block=(4, 4, 4), n_prefix=130, H=1, D=128, offset_std=0.0)
    g = oracle.geometry_of(wl)
    NB, bs, npre = g.NB, g.bs, g.n_pre
    nv = NB - npre
    rng = np.random.default_rng(15)
    dirs = np.linalg.qr(rng.standard_normal((128, NB)))[0].T.astype(np.float32)
    qt = np.zeros((1, 1, g.Sp, 128), dtype=np.float32)
    kt = np.zeros((1, 1, g.Sp, 128), dtype=np.float32)
    for r in range(npre, NB):
        qt[0, 0, r * bs:(r + 1) * bs] = 4 * dirs[r]
        j = npre + (r - npre + 1) % nv
        kt[0, 0, j * bs:(j + 1) * bs] = 4 * dirs[r]
    kt[0, 0, :npre * bs] = 8 * dirs[npre]  # prefix keys aligned with a query direction: ignored
    qb, kb = workloads.f32_to_bf16_bits(qt), workloads.f32_to_bf16_bits(kt)
    s = oracle.score(oracle.pool(g, qb), oracle.pool(g, kb))
    idx, num = oracle.topk_prefix(s, npre, 1)
    for r in range(npre, NB):
        assert num[0, 0, r] == npre + 1
        assert idx[0, 0, r, npre] == npre + (r - npre + 1) % nv
