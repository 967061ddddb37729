"""GPU parity of the fine stage's backward (vsa_sparse_attn_bwd) against the
fp64 oracle (gradients of the attention step of "FastVideo VSA" with the
selection fixed).

Tolerances, relative to the size of each gradient, per tensor: max-abs error
<= 1e-2 x max |ref| and mean-abs error <= 5e-3 x mean |ref|.  Where they come
from: the outputs are bf16, whose rounding alone costs up to 2^-9 (1.95e-3)
of an element and on average about 2.3e-3 of the mean magnitude (the mean
ratio every full-size case shows); the tensor-core operands P and dS are
rounded to 16 bits (2^-9 each, random sign, summed over many rows in fp32),
and delta = rowsum(do * o) uses the forward's 16-bit o.  Observed on a B200
over every case here: max ratio <= 4.4e-3, mean ratio <= 3.1e-3; the bounds
leave about 2x and 1.6x of margin.
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

MAX_REL = 1e-2
MEAN_REL = 5e-3
TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    vsa_build.build()
    vsa.lib()


def _dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TDT[dtype])


def _host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _vals(bits, dtype):
    return oracle.half_to_f32(bits, dtype).astype(np.float64)


def _check(name, got, ref):
    err = np.abs(got - ref)
    mx, mn = float(err.max()), float(err.mean())
    rmx, rmn = float(np.abs(ref).max()), float(np.abs(ref).mean())
    print(f"{name}: max {mx:.3e} (ref {rmx:.3e}, ratio {mx / max(rmx, 1e-30):.3e}) "
          f"mean {mn:.3e} (ref {rmn:.3e}, ratio {mn / max(rmn, 1e-30):.3e})")
    assert mx <= MAX_REL * rmx, name
    assert mn <= MEAN_REL * rmn, name


def _problem(wl, dtype, k, seed, zero_rows=True, garbage_pad=False):
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype=dtype)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(seed)
    to16 = workloads.f32_to_f16_bits if dtype == "f16" else workloads.f32_to_bf16_bits
    do = oracle.tile(g, to16(rng.standard_normal(inp["q"].shape).astype(np.float32)))
    if garbage_pad:  # the dO of padded rows must be ignored
        pad = ~H.real_rows(wl)
        do[:, :, pad] = to16(np.full((1,), 7.0, np.float32))[0]
    if k is None:
        (idx, num), _ = oracle.coarse(g, qt, kt, wl.topk, dtype)
    else:
        k = min(k, g.NB)
        num = rng.integers(0 if zero_rows else 1, k + 1, size=(wl.B, wl.H, g.NB)).astype(np.int32)
        idx = np.full((wl.B, wl.H, g.NB, k), -1, dtype=np.int32)
        for pos in np.ndindex(wl.B, wl.H, g.NB):
            idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    return g, qt, kt, vt, do, idx, num


def _gpu_bwd(wl, dtype, qt, kt, vt, do, idx, num):
    plan = vsa.Plan.of(wl)
    q, k, v, d = (_dev(x, dtype) for x in (qt, kt, vt, do))
    ti, tn = torch.from_numpy(idx).cuda(), torch.from_numpy(num).cuda()
    o, lse = vsa.sparse_attn_fwd(plan, q, k, v, ti, tn)
    dq, dk, dv = vsa.sparse_attn_bwd(plan, q, k, v, o, lse, d, ti, tn)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    return _host(dq), _host(dk), _host(dv)


CASES = [
    # name, workload kwargs, k (None: oracle top-k), dtype, garbage in padded dO
    ("tiny", None, None, "bf16", False),
    ("ragged-empty-rows", dict(T=5, Hg=9, Wg=11, H=2), 3, "bf16", True),
    ("batch2-f16", dict(T=6, Hg=12, Wg=20, B=2, H=2), 4, "f16", False),
    ("prefix", dict(T=4, Hg=16, Wg=16, n_prefix=300, H=3), 5, "bf16", True),
    ("all-blocks", dict(T=8, Hg=8, Wg=16, H=2), 0, "bf16", False),
    # 64-token tiles (the commit log's layout): prefix tiles, partial tiles
    ("tile64-prefix", dict(T=6, Hg=8, Wg=12, block=(4, 4, 4), n_prefix=100, H=3), 7, "bf16", True),
    ("tile64-ragged-f16", dict(T=5, Hg=9, Wg=11, block=(4, 4, 4), H=2), 5, "f16", False),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bwd_matches_oracle_everywhere(case):
    name, kw, k, dtype, garbage = case
    wl = workloads.WORKLOADS[name] if kw is None else workloads.custom(topk=1, **kw)
    if k == 0:  # every block selected: dense attention over the real tokens
        g = oracle.geometry_of(wl)
        k = g.NB
        g, qt, kt, vt, do, _, _ = _problem(wl, dtype, k, seed=7)
        idx = np.broadcast_to(np.arange(g.NB, dtype=np.int32), (wl.B, wl.H, g.NB, g.NB)).copy()
        num = np.full((wl.B, wl.H, g.NB), g.NB, dtype=np.int32)
    else:
        g, qt, kt, vt, do, idx, num = _problem(wl, dtype, k, seed=7, garbage_pad=garbage)
    dq, dk, dv = _gpu_bwd(wl, dtype, qt, kt, vt, do, idx, num)
    real = H.real_rows(wl)
    rows = np.arange(wl.B * wl.H * g.Sp, dtype=np.int64)
    ref_dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows, dtype).reshape(dq.shape)
    ref_dk, ref_dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num, dtype)
    _check(f"{name} dq", _vals(dq, dtype)[:, :, real], ref_dq[:, :, real])
    _check(f"{name} dk", _vals(dk, dtype)[:, :, real], ref_dk[:, :, real])
    _check(f"{name} dv", _vals(dv, dtype)[:, :, real], ref_dv[:, :, real])
    pad = ~real
    for t in (dq, dk, dv):
        assert (t[:, :, pad] == 0).all()


def test_bwd_repeated_ids_count_twice():
    """A row that lists a block twice sees its keys twice in the softmax (as the
    forward does); the transposed lists carry the repeat, and dq, dk, dv match
    the oracle, which walks the lists as given."""
    wl = workloads.custom(T=8, Hg=8, Wg=16, H=2, topk=1)
    g, qt, kt, vt, do, idx, num = _problem(wl, "bf16", 3, seed=9, zero_rows=False)
    idx[0, 0, 1, :3] = [2, 2, 0]
    num[0, 0, 1] = 3
    idx[0, 1, 3, :2] = [1, 1]
    num[0, 1, 3] = 2
    dq, dk, dv = _gpu_bwd(wl, "bf16", qt, kt, vt, do, idx, num)
    real = H.real_rows(wl)
    rows = np.arange(wl.H * g.Sp, dtype=np.int64)
    ref_dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows).reshape(dq.shape)
    ref_dk, ref_dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    _check("repeat dq", _vals(dq, "bf16")[:, :, real], ref_dq[:, :, real])
    _check("repeat dk", _vals(dk, "bf16")[:, :, real], ref_dk[:, :, real])
    _check("repeat dv", _vals(dv, "bf16")[:, :, real], ref_dv[:, :, real])


def _gpu_bwd_selected(wl, qt, kt, vt, do, inp):
    """Forward with the workload's own selection on the GPU (the tile-64 rule with
    its forced-empty rows, or the block map), then the backward; returns the
    selection too."""
    plan = vsa.Plan.of(wl)
    q, k, v, d = (_dev(x, "bf16") for x in (qt, kt, vt, do))
    if wl.map_driven:
        ti, tn = vsa.map_to_index(torch.from_numpy(inp["map"]).cuda())
    else:
        qb, kb = vsa.tile(plan, _dev(inp["q"], "bf16"), pooled=True)[1], vsa.tile(plan, _dev(inp["k"], "bf16"),
                                                                                 pooled=True)[1]
        ti, tn = vsa.coarse_topk_prefix(plan, qb, kb, wl.topk, torch.from_numpy(inp["row_keep"]).cuda())
    o, lse = vsa.sparse_attn_fwd(plan, q, k, v, ti, tn)
    dq, dk, dv = vsa.sparse_attn_bwd(plan, q, k, v, o, lse, d, ti, tn)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    return _host(dq), _host(dk), _host(dv), ti.cpu().numpy(), tn.cpu().numpy()


def _check_key_blocks(name, wl, g, qt, kt, vt, do, idx, num, dk, dv, heads, picks):
    """dk and dv element by element on the chosen key blocks of the chosen heads
    (every real query row whose block lists the key block contributes)."""
    blocks = np.array([h * g.NB + kb for h in heads for kb in picks], dtype=np.int64)
    ref_dk, ref_dv = oracle.attn_bwd_kv_blocks(g, qt, kt, vt, do, idx, num, blocks)
    real = H.real_rows(wl)
    got_k = _vals(dk, "bf16").reshape(wl.H, g.NB, g.bs, -1)
    got_v = _vals(dv, "bf16").reshape(wl.H, g.NB, g.bs, -1)
    gk = np.stack([got_k[h, kb] for h in heads for kb in picks])
    gv = np.stack([got_v[h, kb] for h in heads for kb in picks])
    m = np.stack([real[kb * g.bs:(kb + 1) * g.bs] for h in heads for kb in picks])
    _check(f"{name} dk blocks", gk[m], ref_dk[m])
    _check(f"{name} dv blocks", gv[m], ref_dv[m])
    assert (gk[~m] == 0).all() and (gv[~m] == 0).all()


@pytest.mark.parametrize("name", ["tile64", "tile64map"])
def test_bwd_full_size_tile64(name):
    """The tile-64 workloads (dense prefix rows, forced-empty rows; the computed
    tile-64 selection and the block map): dq on sampled rows (incl. prefix and
    empty rows), dk and dv element by element on sampled key blocks of two heads
    (prefix tiles among them), against the oracle; plus the sum identities."""
    wl = workloads.WORKLOADS[name]
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(13)
    do = oracle.tile(g, workloads.f32_to_bf16_bits(rng.standard_normal(inp["q"].shape).astype(np.float32)))
    dq, dk, dv, idx, num = _gpu_bwd_selected(wl, qt, kt, vt, do, inp)
    ref = H.oracle_front(wl)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_array_equal(num, ref["num"])
    real = np.flatnonzero(H.real_rows(wl))
    rows = []
    for bh in range(wl.B * wl.H):
        pick = rng.choice(real, 24, replace=False)
        zero = np.flatnonzero(num.reshape(-1, g.NB)[bh] == 0)[:2]
        extra = [z * g.bs + np.arange(0, g.bs, 21) for z in zero] + [np.arange(0, g.n_pre * g.bs, 97)]
        rows.append(bh * g.Sp + np.unique(np.concatenate([pick] + extra)))
    rows = np.concatenate(rows)
    ref_dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows)
    _check(f"{name} dq rows", _vals(dq, "bf16").reshape(-1, 128)[rows], ref_dq)
    picks = [0, g.n_pre - 1, g.n_pre, 100, 171, g.NB - 1] + sorted(rng.choice(np.arange(g.n_pre, g.NB), 2,
                                                                              replace=False).tolist())
    _check_key_blocks(name, wl, g, qt, kt, vt, do, idx, num, dk, dv, [0, wl.H - 1], picks)
    realm = H.real_rows(wl)
    dkv = _vals(dk, "bf16")[0][:, realm]
    dvv = _vals(dv, "bf16")[0][:, realm]
    dov = _vals(do, "bf16")[0]
    for h in range(wl.H):
        rows_h = realm & (np.repeat(num[0, h], g.bs) > 0)
        assert np.abs(dkv[h].sum(axis=0)).max() <= 2e-2 * np.abs(dkv[h]).sum(axis=0).max(), h
        np.testing.assert_allclose(dvv[h].sum(axis=0), dov[h][rows_h].sum(axis=0), rtol=0,
                                   atol=2e-2 * np.abs(dov[h][rows_h]).sum(axis=0).max())


@pytest.mark.parametrize("name", ["fastwan", "wan81", "long"])
def test_bwd_full_size(name):
    """The top-k workloads at full size: dq on sampled rows, dk and dv element by
    element on sampled key blocks of two heads (the partial corner block among
    them), against the oracle; plus identities that hold at any size: the sum
    over keys of dk is 0 and the sum of dv is the sum of do over rows with a
    non-empty selection."""
    wl = workloads.WORKLOADS[name]
    g, qt, kt, vt, do, idx, num = _problem(wl, "bf16", None, seed=11)
    dq, dk, dv = _gpu_bwd(wl, "bf16", qt, kt, vt, do, idx, num)
    real = np.flatnonzero(H.real_rows(wl))
    rng = np.random.default_rng(12)
    rows = np.concatenate([bh * g.Sp + np.unique(np.concatenate([rng.choice(real, 24, replace=False),
                                                                 real[:2], real[-2:]]))
                           for bh in range(wl.H)])
    ref = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows)
    _check(f"{name} dq rows", _vals(dq, "bf16").reshape(-1, 128)[rows], ref)
    nblk = 8 if name != "long" else 4
    picks = [0, g.NB - 1] + sorted(rng.choice(np.arange(1, g.NB - 1), nblk - 2, replace=False).tolist())
    _check_key_blocks(name, wl, g, qt, kt, vt, do, idx, num, dk, dv, [0, wl.H - 1], picks)
    realm = H.real_rows(wl)
    dkv = _vals(dk, "bf16")[0][:, realm]
    dvv = _vals(dv, "bf16")[0][:, realm]
    dov = _vals(do, "bf16")[0][:, realm]
    for h in range(wl.H):
        s = dkv[h].sum(axis=0)
        assert np.abs(s).max() <= 2e-2 * np.abs(dkv[h]).sum(axis=0).max(), h
        # top-k workloads give every row topk > 0 selections
        np.testing.assert_allclose(dvv[h].sum(axis=0), dov[h].sum(axis=0), rtol=0,
                                   atol=2e-2 * np.abs(dov[h]).sum(axis=0).max())


def test_bwd_bad_ids_are_reported_and_skipped():
    """A block id outside [0, NB) and a count above max_k: VSA_ERR_BAD_INDEX is
    reported, the bad id is skipped and the count clamped (its list's -1 padding
    then skipped as well), so the gradients equal the oracle's on the cleaned
    lists."""
    wl = workloads.custom(T=8, Hg=8, Wg=16, H=2, topk=1)
    g, qt, kt, vt, do, idx, num = _problem(wl, "bf16", 4, seed=19, zero_rows=False)
    bad_idx, bad_num = idx.copy(), num.copy()
    r = int(np.flatnonzero(num[0, 0] >= 2)[0])
    bad_idx[0, 0, r, num[0, 0, r] - 1] = g.NB + 3      # the last id of row r: out of range
    idx[0, 0, r, num[0, 0, r] - 1] = -1                 # cleaned: dropped
    num[0, 0, r] -= 1
    bad_num[0, 1, 2] = 99                               # clamped to max_k; the -1 entries past the
    plan = vsa.Plan.of(wl)                              # real count are skipped
    q, k, v, d = (_dev(x, "bf16") for x in (qt, kt, vt, do))
    ti, tn = torch.from_numpy(bad_idx).cuda(), torch.from_numpy(bad_num).cuda()
    o, lse = vsa.sparse_attn_fwd(plan, q, k, v, ti, tn)
    assert vsa.get_status() == vsa.VSA_ERR_BAD_INDEX
    dq, dk, dv = vsa.sparse_attn_bwd(plan, q, k, v, o, lse, d, ti, tn)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_ERR_BAD_INDEX
    assert vsa.get_status() == vsa.VSA_OK
    real = H.real_rows(wl)
    rows = np.arange(wl.H * g.Sp, dtype=np.int64)
    ref_dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows).reshape(dq.shape)
    ref_dk, ref_dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    _check("bad dq", _vals(_host(dq), "bf16")[:, :, real], ref_dq[:, :, real])
    _check("bad dk", _vals(_host(dk), "bf16")[:, :, real], ref_dk[:, :, real])
    _check("bad dv", _vals(_host(dv), "bf16")[:, :, real], ref_dv[:, :, real])


def test_bwd_grid_beyond_the_transpose_bitmap():
    """1100 64-token blocks (above the 1024 the transposed selection builds from
    a bitmap): the lists are placed one query block at a time; dq on sampled
    rows and dk, dv on sampled key blocks against the oracle."""
    wl = workloads.custom(T=8, Hg=100, Wg=88, block=(4, 4, 4), H=1, topk=1)
    g, qt, kt, vt, do, idx, num = _problem(wl, "bf16", 3, seed=21)
    assert g.NB == 1100
    dq, dk, dv = _gpu_bwd(wl, "bf16", qt, kt, vt, do, idx, num)
    rng = np.random.default_rng(22)
    real = np.flatnonzero(H.real_rows(wl))
    rows = np.unique(np.concatenate([rng.choice(real, 400, replace=False), real[:3], real[-3:]]))
    ref_dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows)
    _check("NB 1100 dq rows", _vals(dq, "bf16").reshape(-1, 128)[rows], ref_dq)
    picks = [0, 1, 517, g.NB - 2, g.NB - 1] + sorted(rng.choice(g.NB, 3, replace=False).tolist())
    _check_key_blocks("NB 1100", wl, g, qt, kt, vt, do, idx, num, dk, dv, [0], picks)
