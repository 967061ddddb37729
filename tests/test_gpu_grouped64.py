"""GPU parity of the fine stage for 64-token tiles, whose kernel groups four
query blocks per item, two per 128-row Q tile, each Q tile walking the union
of its two selections (shared blocks first, loaded once for both Q tiles)
(FastVideo commit log,
examples/inference/basic/README.md: the tile-64 layout with non-uniform and
zero-count rows).  Every case runs the fine stage on oracle-supplied indices
and compares o / lse with the oracle at the parity tolerances: sorted and
unsorted lists, lists that repeat an id (the group then walks its lists as
given), whole groups with nothing selected, a trailing group of two query
blocks, every block selected, bad ids and counts, B = 2, fp16, a grid beyond
the grouped kernel's bitmap capacity (NB > 1024), and groups built to reach
every shape of the two Q tiles' streams."""
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


def _setup(T, Hg, Wg, npre=0, H_=2, B=1, dtype="bf16"):
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=(4, 4, 4), n_prefix=npre, H=H_, B=B)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype=dtype)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    return wl, g, qt, kt, vt


def _random_lists(rng, B, H_, NB, max_k, lo=0, sort=True):
    num = rng.integers(lo, max_k + 1, size=(B, H_, NB)).astype(np.int32)
    idx = np.full((B, H_, NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(B, H_, NB):
        pick = rng.permutation(NB)[:num[pos]]
        idx[pos][:num[pos]] = np.sort(pick) if sort else pick
    return idx, num


def _run(wl, g, qt, kt, vt, idx, num, dtype="bf16", rows=None, status=vsa.VSA_OK, what=""):
    plan = vsa.Plan.of(wl)
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(tdt)
    o, lse = vsa.sparse_attn_fwd(plan, dev(qt), dev(kt), dev(vt), torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(num).cuda())
    torch.cuda.synchronize()
    assert vsa.get_status() == status
    if rows is None:
        rows = np.flatnonzero(np.tile(H.real_rows(wl), wl.B * wl.H))
    o_ref, lse_ref = oracle.attn_rows(g, qt, kt, vt, idx, num, rows, dtype)
    o_bits = o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1, 128)[rows]
    if dtype == "f16":
        o_bits = workloads.f32_to_bf16_bits(oracle.half_to_f32(o_bits, "f16"))  # compare values
    return H.compare_o_lse(o_bits, lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref, what)


@pytest.mark.parametrize("sort", [True, False])
def test_union_of_sorted_and_unsorted_lists(sort):
    """NB = 2 + 3*4*4 = 50: twelve groups of four and a trailing group of two."""
    wl, g, qt, kt, vt = _setup(12, 16, 16, npre=100, H_=3)
    assert g.NB % 4 == 2
    rng = np.random.default_rng(50)
    idx, num = _random_lists(rng, 1, 3, g.NB, 9, sort=sort)
    _run(wl, g, qt, kt, vt, idx, num, what=f"sorted={sort}")


def test_repeated_ids_count_twice():
    """A list that names a block twice: its group walks the lists as given, and the
    block's keys count twice, as the oracle (and the 256-token kernel) define it."""
    wl, g, qt, kt, vt = _setup(8, 16, 16, npre=128, H_=2)
    rng = np.random.default_rng(51)
    idx, num = _random_lists(rng, 1, 2, g.NB, 6, lo=1)
    idx[0, 0, 1, :3] = [4, 4, 0]
    num[0, 0, 1] = 3
    idx[0, 1, 6, :2] = [2, 2]
    num[0, 1, 6] = 2
    idx[0, 1, 7, :4] = [9, 1, 9, 9]
    num[0, 1, 7] = 4
    _run(wl, g, qt, kt, vt, idx, num, what="repeats")


def test_empty_rows_and_empty_groups():
    """Zero-count rows inside groups, and whole groups with nothing selected: o = 0,
    lse = -inf; the other rows are unaffected."""
    wl, g, qt, kt, vt = _setup(8, 16, 32, H_=2)
    rng = np.random.default_rng(52)
    idx, num = _random_lists(rng, 1, 2, g.NB, 5)
    num[0, 0, 4:8] = 0          # a whole group
    num[0, 1, ::3] = 0
    num[0, 1, g.NB - 2:] = 0    # the trailing blocks of the head
    _run(wl, g, qt, kt, vt, idx, num, what="empty")


def test_every_block_selected_is_dense():
    wl, g, qt, kt, vt = _setup(8, 12, 16, npre=100, H_=1)
    idx = np.broadcast_to(np.arange(g.NB, dtype=np.int32), (1, 1, g.NB, g.NB)).copy()
    num = np.full((1, 1, g.NB), g.NB, dtype=np.int32)
    _run(wl, g, qt, kt, vt, idx, num, what="dense")


def test_bad_id_and_bad_count_are_reported_and_skipped():
    """Ids outside [0, NB) are skipped and counts above max_k clamped; both raise
    VSA_ERR_BAD_INDEX.  Rows of other query blocks stay exact."""
    wl, g, qt, kt, vt = _setup(8, 16, 16, H_=1)
    rng = np.random.default_rng(53)
    idx, num = _random_lists(rng, 1, 1, g.NB, 4, lo=1)
    bad_idx, bad_num = idx.copy(), num.copy()
    bad_idx[0, 0, 5, 0] = g.NB + 3
    bad_num[0, 0, 9] = 99
    plan = vsa.Plan.of(wl)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    o, lse = vsa.sparse_attn_fwd(plan, dev(qt), dev(kt), dev(vt), torch.from_numpy(bad_idx).cuda(),
                                 torch.from_numpy(bad_num).cuda())
    assert vsa.get_status() == vsa.VSA_ERR_BAD_INDEX
    assert vsa.get_status() == vsa.VSA_OK
    rows = np.concatenate([np.arange(b * 64, (b + 1) * 64) for b in range(g.NB) if b not in (5, 9)])
    o_ref, lse_ref = oracle.attn_rows(g, qt, kt, vt, idx, num, rows)
    H.compare_o_lse(H.from_dev(o).reshape(-1, 128)[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref,
                    "bad id / count")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_batch_of_two_and_fp16(dtype):
    wl, g, qt, kt, vt = _setup(6, 20, 12, npre=70, H_=3, B=2, dtype=dtype)
    rng = np.random.default_rng(54)
    idx, num = _random_lists(rng, 2, 3, g.NB, 7)
    _run(wl, g, qt, kt, vt, idx, num, dtype=dtype, what=f"B2 {dtype}")


def test_many_groups_per_cta_with_prefix_rule():
    """24 heads x 17 groups: several groups per CTA, dense prefix rows (the tile-64
    rule) and forced-empty rows, the hand-offs between groups inside a CTA."""
    wl, g, qt, kt, vt = _setup(8, 16, 32, npre=256, H_=24)
    qbar, kbar = oracle.pool(g, qt), oracle.pool(g, kt)
    keep = (np.random.default_rng(55).random((1, 24, g.NB)) > 0.05).astype(np.uint8)
    idx, num = oracle.topk_prefix(oracle.score(qbar, kbar), g.n_pre, 12, keep)
    rng = np.random.default_rng(56)
    real = np.flatnonzero(H.real_rows(wl))
    rows = np.concatenate([h * g.Sp + np.unique(np.concatenate([rng.choice(real, 40, replace=False),
                                                                real[:3], real[-3:]])) for h in range(24)])
    _run(wl, g, qt, kt, vt, idx, num, rows=rows, what="many groups")


def test_beyond_bitmap_capacity_uses_the_per_block_kernel():
    """NB = 2048 > 1024: the fine stage runs one query block per item instead."""
    wl, g, qt, kt, vt = _setup(32, 64, 64, H_=1)
    assert g.NB == 2048
    rng = np.random.default_rng(57)
    idx, num = _random_lists(rng, 1, 1, g.NB, 3)
    real = np.flatnonzero(H.real_rows(wl))
    rows = np.unique(np.concatenate([rng.choice(real, 600, replace=False), real[:4], real[-4:]]))
    _run(wl, g, qt, kt, vt, idx, num, rows=rows, what="NB 2048")


def test_shared_queue_gives_the_static_results_and_leaves_the_workspace_zero():
    """vsa_sparse_attn_fwd_ws: groups handed out from a shared queue (prefix
    groups first) give bit for bit the static assignment's results, on the full
    tile64 workload, twice in a row; the workspace is zero after each call."""
    wl = workloads.WORKLOADS["tile64"]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    q, k, v = (H.to_dev(ref[n]) for n in ("qt", "kt", "vt"))
    ti, tn = torch.from_numpy(ref["idx"]).cuda(), torch.from_numpy(ref["num"]).cuda()
    o0, l0 = vsa.sparse_attn_fwd(plan, q, k, v, ti, tn)
    ws = torch.zeros(4, dtype=torch.int32, device="cuda")
    for _ in range(2):
        o1, l1 = vsa.sparse_attn_fwd(plan, q, k, v, ti, tn, workspace=ws)
        torch.cuda.synchronize()
        assert vsa.get_status() == vsa.VSA_OK
        assert int(ws.abs().sum()) == 0
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
        assert torch.equal(l0.view(torch.int32), l1.view(torch.int32))


def test_shared_queue_on_small_grids():
    """Fewer groups than SMs, a trailing group of two, repeated ids and empty rows
    through the queue: against the oracle."""
    wl, g, qt, kt, vt = _setup(12, 16, 16, npre=100, H_=3)
    rng = np.random.default_rng(58)
    idx, num = _random_lists(rng, 1, 3, g.NB, 9)
    idx[0, 1, 3, :3] = [7, 7, 2]
    num[0, 1, 3] = 3
    num[0, 2, :4] = 0
    plan = vsa.Plan.of(wl)
    ws = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, lse = vsa.sparse_attn_fwd(plan, H.to_dev(qt), H.to_dev(kt), H.to_dev(vt), torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(num).cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK and int(ws.abs().sum()) == 0
    rows = np.flatnonzero(np.tile(H.real_rows(wl), 3))
    o_ref, lse_ref = oracle.attn_rows(g, qt, kt, vt, idx, num, rows)
    H.compare_o_lse(H.from_dev(o).reshape(-1, 128)[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref,
                    "queue")


def _stream_shapes(NB):
    """Index lists whose groups of four take every shape of the two Q tiles'
    streams (Q tile 0 = query blocks 0-1 of a group, Q tile 1 = blocks 2-3)."""
    max_k = 12
    idx = np.full((1, 1, NB, max_k), -1, dtype=np.int32)
    num = np.zeros((1, 1, NB), dtype=np.int32)

    def put(row, ids):
        idx[0, 0, row, :len(ids)] = ids
        num[0, 0, row] = len(ids)

    # group 0: Q tile 0 selects nothing, Q tile 1 alone
    put(2, [3, 9, 17, 30]); put(3, [9, 11])
    # group 1: Q tile 1 selects nothing (two Q tiles, one empty)
    put(4, [0, 5, 6]); put(5, [31])
    # group 2: all four select the same 7 blocks (every tile shared, the last
    # one half empty)
    for r in range(8, 12):
        put(r, [1, 4, 8, 13, 21, 25, 29])
    # group 3: disjoint selections, Q tile 0's stream longer (no shared tile)
    put(12, [0, 2, 4, 6, 8]); put(13, [10, 12, 14, 16]); put(14, [1, 3]); put(15, [5])
    # group 4: disjoint, Q tile 1's stream longer
    put(16, [7]); put(18, [0, 2, 4, 6, 8, 10, 12]); put(19, [14, 16, 18, 20, 22])
    # group 5: five shared blocks (an odd count: the third tile pairs the last
    # shared block with each Q tile's first own block), four of Q tile 0's own,
    # seven of Q tile 1's own
    sh = [3, 6, 9, 12, 15]
    put(20, sh[:3] + [0, 1]); put(21, sh[3:] + [2, 4]); put(22, sh + [5, 7, 8, 10]); put(23, [11, 13, 14])
    # group 6: one query block of each Q tile selects, unsorted, partly shared
    put(24, [30, 2, 17, 5]); put(27, [5, 30, 19])
    # group 7: shared blocks only in Q tile 1's second block, with repeats
    # across query blocks but none inside a list
    put(28, [0, 31]); put(29, [31, 16]); put(30, [16]); put(31, [0, 8, 31])
    return idx, num


@pytest.mark.parametrize("queue", [False, True], ids=["static", "queue"])
def test_every_shape_of_the_two_q_tile_streams(queue):
    """Empty Q tiles, all-shared and no-shared groups, tails on either side, an
    odd number of shared blocks: against the oracle, static and queued."""
    wl, g, qt, kt, vt = _setup(8, 16, 16, H_=1)
    assert g.NB == 32
    idx, num = _stream_shapes(g.NB)
    plan = vsa.Plan.of(wl)
    ws = torch.zeros(4, dtype=torch.int32, device="cuda") if queue else None
    o, lse = vsa.sparse_attn_fwd(plan, H.to_dev(qt), H.to_dev(kt), H.to_dev(vt), torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(num).cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    if queue:
        assert int(ws.abs().sum()) == 0
    rows = np.flatnonzero(H.real_rows(wl))
    o_ref, lse_ref = oracle.attn_rows(g, qt, kt, vt, idx, num, rows)
    H.compare_o_lse(H.from_dev(o).reshape(-1, 128)[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref,
                    f"stream shapes queue={queue}")
