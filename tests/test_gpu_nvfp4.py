"""GPU parity of the NVFP4 Q/K path (FastVideo "Optimizations" page, section
"FP4 Flash Attention 4 (Blackwell only)").

Quantisation: codes and scales bit-exact against the oracle (the oracle's
row-major scales are rearranged here into the tensor core's layout, a pure
index permutation).  Fine stage: o and lse against the oracle's attention on
the values the codes stand for, with the 16-bit fine stage's tolerances (the
FP4 products are exact; P is rounded to 16 bits as in the 16-bit path).  The
fine stage is run on oracle-supplied codes and indices; the full path
(Forward(nvfp4=True)) on its own.
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

SHAPES = [
    (8, 16, 16, (4, 8, 8), 0),
    (5, 9, 9, (4, 8, 8), 0),
    (7, 8, 16, (4, 8, 8), 0),
    (12, 20, 20, (4, 8, 8), 0),
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


def sf_layout(sf_rows: np.ndarray) -> np.ndarray:
    """Row-major scales [..., rows, 8] -> [..., rows/128, 1024]: byte kh*512 + (r%32)*16 + (r/32)*4 + j
    holds the scale of row r, block 4kh + j."""
    lead = sf_rows.shape[:-2]
    t = sf_rows.shape[-2] // 128
    s = sf_rows.reshape(lead + (t, 4, 32, 2, 4))  # [t, r/32, r%32, kh, j]
    n = len(lead)
    perm = tuple(range(n)) + (n, n + 3, n + 2, n + 1, n + 4)
    return np.ascontiguousarray(s.transpose(perm)).reshape(lead + (t, 1024))


def _dev16(bits, f16=False):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.float16 if f16 else torch.bfloat16)


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _special_rows(x: np.ndarray) -> np.ndarray:
    """Plant blocks that reach every branch: all zero, signed zeros, a scale
    that rounds to E4M3 zero, a saturating scale (amax/6 > 448), exact ties."""
    x = x.copy()
    flat = x.reshape(-1, x.shape[-1])
    bf = workloads.f32_to_bf16_bits
    flat[0, :16] = 0
    flat[0, 16:32] = 0x8000
    flat[1, :16] = bf(np.full(16, 1e-5, np.float32))
    flat[2, :16] = bf(np.linspace(-3000, 3000, 16).astype(np.float32))
    flat[3, :16] = bf((np.arange(16) * 0.25 - 2).astype(np.float32))
    flat[3, 15] = bf(np.array([6.0], np.float32))[0]
    return x


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("f16", [False, True])
def test_quantize_bit_exact(shape, f16):
    wl = _wl(shape, H_=3, B=2)
    g = oracle.geometry_of(wl)
    plan = vsa.Plan.of(wl)
    inp = workloads.make_inputs(wl, dtype="f16" if f16 else "bf16")
    xt = oracle.tile(g, inp["q"])
    if not f16:
        xt = _special_rows(xt)
    codes, scales = vsa.quantize_nvfp4(plan, _dev16(xt, f16))
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    rc, rs = oracle.quant_nvfp4(xt, "f16" if f16 else "bf16")
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(scales.cpu().numpy(), sf_layout(rs))


def test_quantize_full_size_fastwan():
    wl = workloads.WORKLOADS["fastwan"]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    for n in ("qt", "kt"):
        codes, scales = vsa.quantize_nvfp4(plan, H.to_dev(ref[n]))
        torch.cuda.synchronize()
        rc, rs = oracle.quant_nvfp4(ref[n])
        np.testing.assert_array_equal(codes.cpu().numpy(), rc)
        np.testing.assert_array_equal(scales.cpu().numpy(), sf_layout(rs))
    assert vsa.get_status() == vsa.VSA_OK


def _fp4_vs_oracle(wl, qt, kt, vt, idx, num, rows=None, f16=False, what=""):
    """Fine stage on oracle codes and indices vs the oracle's NVFP4 attention."""
    g = oracle.geometry_of(wl)
    plan = vsa.Plan.of(wl)
    dt = "f16" if f16 else "bf16"
    (qc, qs), (kc, ks) = oracle.quant_nvfp4(qt, dt), oracle.quant_nvfp4(kt, dt)
    o, lse = vsa.sparse_attn_fwd_nvfp4(plan, _u8(qc), _u8(sf_layout(qs)), _u8(kc), _u8(sf_layout(ks)),
                                       _dev16(vt, f16), torch.from_numpy(idx).cuda(), torch.from_numpy(num).cuda())
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    if rows is None:
        rows = np.flatnonzero(np.tile(H.real_rows(wl), wl.B * wl.H))
    o_ref, lse_ref = oracle.attn_rows_nvfp4(g, qc, qs, kc, ks, vt, idx, num, rows, dt)
    raw = o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1, 128)[rows]
    lse_g = lse.cpu().numpy().reshape(-1)[rows]
    if not f16:
        H.compare_o_lse(raw, lse_g, o_ref, lse_ref, what)
        return
    err = np.abs(raw.view(np.float16).astype(np.float64) - o_ref)
    assert err.max(initial=0) <= H.O_MAX_ABS and err.mean() <= H.O_MEAN_ABS, what
    lg = lse_g.astype(np.float64)
    np.testing.assert_array_equal(np.isneginf(lg), np.isneginf(lse_ref))
    fin = ~np.isneginf(lse_ref)
    assert np.abs(lg[fin] - lse_ref[fin]).max(initial=0) <= H.LSE_ABS, what


def _random_selection(g, Hh, seed, max_k=5):
    rng = np.random.default_rng(seed)
    max_k = min(max_k, g.NB)
    num = rng.integers(0, max_k + 1, size=(1, Hh, g.NB)).astype(np.int32)
    num.reshape(-1)[0] = max_k
    idx = np.full((1, Hh, g.NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(1, Hh, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    return idx, num


def test_fp4_attention_tiny_every_row():
    wl = workloads.WORKLOADS["tiny"]
    ref = H.oracle_front(wl)
    _fp4_vs_oracle(wl, ref["qt"], ref["kt"], ref["vt"], ref["idx"], ref["num"], what="tiny")


@pytest.mark.parametrize("shape", SHAPES)
def test_fp4_attention_nonuniform_rows(shape):
    """Counts 0..max_k per row (zero rows included) on grids with partial blocks
    along every axis, and 64-token tiles after a prefix."""
    wl = _wl(shape, H_=2)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx, num = _random_selection(g, 2, seed=21)
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what=str(shape))


@pytest.mark.parametrize("shape", [SHAPES[0], SHAPES[5]])
def test_fp4_attention_fp16(shape):
    wl = _wl(shape, H_=2)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, dtype="f16")
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx, num = _random_selection(g, 2, seed=22)
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, f16=True, what=f"f16 {shape}")


def test_fp4_attention_all_blocks_and_repeated_ids():
    wl = _wl((12, 20, 20, (4, 8, 8), 0), H_=2)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx = np.broadcast_to(np.arange(g.NB, dtype=np.int32), (1, 2, g.NB, g.NB)).copy()
    num = np.full((1, 2, g.NB), g.NB, dtype=np.int32)
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what="all blocks")
    idx[0, 1, :, 1] = idx[0, 1, :, 0]  # a block listed twice counts twice
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what="repeated")


def test_fp4_bad_index_is_reported():
    wl = workloads.WORKLOADS["tiny"]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    idx = ref["idx"].copy()
    idx[0, 1, 3, 0] = 99
    (qc, qs), (kc, ks) = oracle.quant_nvfp4(ref["qt"]), oracle.quant_nvfp4(ref["kt"])
    vsa.sparse_attn_fwd_nvfp4(plan, _u8(qc), _u8(sf_layout(qs)), _u8(kc), _u8(sf_layout(ks)), H.to_dev(ref["vt"]),
                              torch.from_numpy(idx).cuda(), torch.from_numpy(ref["num"]).cuda())
    assert vsa.get_status() == vsa.VSA_ERR_BAD_INDEX
    assert vsa.get_status() == vsa.VSA_OK


def _sample_rows(wl, n_per_head, seed):
    rng = np.random.default_rng(seed)
    g = oracle.geometry_of(wl)
    real = np.flatnonzero(H.real_rows(wl))
    rows = []
    for bh in range(wl.B * wl.H):
        pick = rng.choice(real, size=n_per_head, replace=False)
        rows.append(bh * g.Sp + np.unique(np.concatenate([pick, real[-2:], real[:2]])))
    return np.concatenate(rows)


@pytest.mark.parametrize("name", ["fastwan", "wan81", "tile64", "long"])
def test_full_path_nvfp4_full_size(name):
    """Forward(nvfp4=True) at full size: the quantised q, k bit-exact, o/lse on
    sampled real rows against the oracle's NVFP4 attention."""
    wl = workloads.WORKLOADS[name]
    ref = H.oracle_front(wl)
    inp = H.inputs(wl)
    plan = vsa.Plan.of(wl)
    fwd = vsa.Forward(plan, wl.B, wl.H, wl.topk, nvfp4=True, prefix_dense=wl.prefix_dense)
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    keep = torch.from_numpy(inp["row_keep"]).cuda() if inp["row_keep"] is not None else None
    o, lse = fwd(H.to_dev(inp["q"]), H.to_dev(inp["k"]), H.to_dev(inp["v"]), bmap, row_keep=keep)
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    (qc, qs), (kc, ks) = oracle.quant_nvfp4(ref["qt"]), oracle.quant_nvfp4(ref["kt"])
    np.testing.assert_array_equal(fwd.qc.cpu().numpy(), qc)
    np.testing.assert_array_equal(fwd.ks.cpu().numpy(), sf_layout(ks))
    rows = _sample_rows(wl, 32, seed=23)
    o_ref, lse_ref = oracle.attn_rows_nvfp4(ref["g"], qc, qs, kc, ks, ref["vt"], ref["idx"], ref["num"], rows)
    ot_bits = H.from_dev(fwd.ot).reshape(-1, 128)
    H.compare_o_lse(ot_bits[rows], lse.cpu().numpy().reshape(-1)[rows], o_ref, lse_ref, name)


@pytest.mark.parametrize("shape,H_,k", [((15, 14, 15, (4, 8, 8), 0), 24, 8), ((31, 22, 40, (4, 8, 8), 0), 2, 64)])
def test_fp4_attention_many_items_per_cta(shape, H_, k):
    """More items than CTAs and long selections on a grid with partial blocks:
    exercises item-to-item hand-offs inside a CTA (every small case above has
    at most one item per CTA)."""
    wl = _wl(shape, H_=H_)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx, num = oracle.topk(oracle.score(oracle.pool(g, qt), oracle.pool(g, kt)), k)
    rows = _sample_rows(wl, 24, seed=31)
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, rows=rows, what=f"many items {shape} H{H_} k{k}")


@pytest.mark.parametrize("shape", [SHAPES[1], SHAPES[5]])
def test_fp4_attention_batch_of_two(shape):
    wl = _wl(shape, H_=2, B=2)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(34)
    max_k = min(4, g.NB)
    num = rng.integers(0, max_k + 1, size=(2, 2, g.NB)).astype(np.int32)
    idx = np.full((2, 2, g.NB, max_k), -1, dtype=np.int32)
    for pos in np.ndindex(2, 2, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what=f"B2 {shape}")


@pytest.mark.parametrize("name", ["tiny", "fastwan", "wan81", "tile64", "long"])
def test_fp4_cosine_to_bf16_per_call(name):
    """The FastVideo "Optimizations" page (section "FP4 Flash Attention 4",
    "Known Limitations") quotes a per-call cosine similarity of about 0.99 between
    the FP4 and the BF16 attention output.  Here: the cosine of the NVFP4 fine
    stage's o against the bf16 fine stage's o on the same inputs and selection,
    over the real rows of one call, on every workload."""
    wl = workloads.WORKLOADS[name]
    inp = H.inputs(wl)
    plan = vsa.Plan.of(wl)
    bmap = torch.from_numpy(inp["map"]).cuda() if wl.map_driven else None
    keep = torch.from_numpy(inp["row_keep"]).cuda() if inp["row_keep"] is not None else None
    args = (H.to_dev(inp["q"]), H.to_dev(inp["k"]), H.to_dev(inp["v"]), bmap)
    f16 = vsa.Forward(plan, wl.B, wl.H, wl.topk, prefix_dense=wl.prefix_dense)
    f4 = vsa.Forward(plan, wl.B, wl.H, wl.topk, nvfp4=True, prefix_dense=wl.prefix_dense)
    o16 = f16(*args, row_keep=keep)[0].float()
    o4 = f4(*args, row_keep=keep)[0].float()
    torch.cuda.synchronize()
    assert vsa.get_status() == vsa.VSA_OK
    assert torch.equal(f16.idx, f4.idx)
    cos = float(torch.nn.functional.cosine_similarity(o4.reshape(1, -1), o16.reshape(1, -1)).item())
    print(f"{name}: cosine(o_fp4, o_bf16) = {cos:.5f}")
    assert cos >= 0.99, cos


def test_fp4_grouped_every_stream_shape_and_repeats():
    """64-token tiles run four query blocks per item in the NVFP4 kernel too:
    crafted groups reaching every shape of the two Q tiles' key streams (empty
    Q tile on either side, all or no shared blocks, tails on either side, an
    odd shared count), then lists that repeat an id (those groups walk the
    lists as given), against the oracle's NVFP4 attention."""
    from tests.test_gpu_grouped64 import _stream_shapes
    wl = _wl((8, 16, 16, (4, 4, 4), 0), H_=1)
    g = oracle.geometry_of(wl)
    assert g.NB == 32
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx, num = _stream_shapes(g.NB)
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what="fp4 stream shapes")
    idx[0, 0, 9, :3] = [13, 13, 1]   # group 2: a repeat
    num[0, 0, 9] = 3
    idx[0, 0, 30, :2] = [16, 16]     # group 7
    num[0, 0, 30] = 2
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, what="fp4 repeats")


def test_fp4_shared_queue_gives_the_static_results():
    """vsa_sparse_attn_fwd_nvfp4_ws: the 64-token groups handed out from a
    shared queue give bit for bit the static assignment's results on the full
    tile64 workload, twice in a row; the workspace is zero after each call."""
    wl = workloads.WORKLOADS["tile64"]
    ref = H.oracle_front(wl)
    plan = vsa.Plan.of(wl)
    (qc, qs), (kc, ks) = oracle.quant_nvfp4(ref["qt"]), oracle.quant_nvfp4(ref["kt"])
    args = (plan, _u8(qc), _u8(sf_layout(qs)), _u8(kc), _u8(sf_layout(ks)), H.to_dev(ref["vt"]),
            torch.from_numpy(ref["idx"]).cuda(), torch.from_numpy(ref["num"]).cuda())
    o0, l0 = vsa.sparse_attn_fwd_nvfp4(*args)
    ws = torch.zeros(4, dtype=torch.int32, device="cuda")
    for _ in range(2):
        o1, l1 = vsa.sparse_attn_fwd_nvfp4(*args, workspace=ws)
        torch.cuda.synchronize()
        assert vsa.get_status() == vsa.VSA_OK
        assert int(ws.abs().sum()) == 0
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
        assert torch.equal(l0.view(torch.int32), l1.view(torch.int32))


def test_fp4_beyond_bitmap_capacity_uses_the_per_item_kernel():
    """NB = 2048 > 1024 64-token blocks: the NVFP4 fine stage runs one query
    block per item (the per-item kernel's 64-token path) instead of groups."""
    wl = _wl((32, 64, 64, (4, 4, 4), 0), H_=1)
    g = oracle.geometry_of(wl)
    assert g.NB == 2048
    inp = workloads.make_inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    idx, num = _random_selection(g, 1, seed=41, max_k=3)
    rng = np.random.default_rng(42)
    real = np.flatnonzero(H.real_rows(wl))
    rows = np.unique(np.concatenate([rng.choice(real, 600, replace=False), real[:4], real[-4:]]))
    _fp4_vs_oracle(wl, qt, kt, vt, idx, num, rows=rows, what="fp4 NB 2048")
