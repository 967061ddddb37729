"""Host-side checks of the C ABI (no kernel is launched by any test here).

Every call below either fails argument validation -- which returns before
any CUDA call -- or only touches host state (plans, strings).
"""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_video_gather_b200 as vsa
from block_sparse_video_gather_b200 import build as vsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")
FAKE = 0x100000  # an aligned, non-null address; never dereferenced (validation fails first)


@pytest.fixture(scope="module")
def L():
    vsa_build.build()
    return vsa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(vsa.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_library_exports_nothing_else(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", vsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln and ln.split()[-1].startswith("vsa_")})
    assert exported == declared_functions()


def test_strerror(L):
    for code in range(8):
        assert L.vsa_strerror(code)
    assert b"unknown" in L.vsa_strerror(99)


def _plan(*args):
    p = vsa.Plan(*args)
    return p


def test_plan_sizes_match_oracle_geometry():
    import oracle
    from block_sparse_video_gather_b200 import workloads
    for wl in workloads.WORKLOADS.values():
        p = vsa.Plan.of(wl)
        g = oracle.geometry_of(wl)
        assert (p.NB, p.S, p.Sp, p.bs) == (g.NB, g.S, g.Sp, g.bs)


def test_describe_reproduces_route_log_fields():
    """Fields of the routing log printed on "FastVideo VSA", section "Choose top-k"."""
    gold = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "fastwan_route.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            gold[k] = v
    p = vsa.Plan(31, 22, 40)
    s = p.describe(64)
    assert f"seq_len={gold['seq_len'][0]}" in s
    assert "dit_seq_shape=({}, {}, {})".format(*gold["dit_seq_shape"]) in s
    assert "block_size=({}, {}, {})".format(*gold["block_size"]) in s
    assert f"num_blocks={gold['num_blocks'][0]}" in s
    assert f"topk={gold['topk'][0]}" in s
    assert f"keep_ratio={gold['keep_ratio_percent'][0]}%" in s


@pytest.mark.parametrize("args,code", [
    ((0, 8, 8, 4, 8, 8), vsa.VSA_ERR_INVALID_ARG),
    ((4, 8, 8, 0, 8, 8), vsa.VSA_ERR_INVALID_ARG),
    ((4, 8, 8, 3, 8, 8), vsa.VSA_ERR_UNSUPPORTED),   # not a power of two
    ((4, 8, 8, 4, 8, 4), vsa.VSA_ERR_UNSUPPORTED),   # 128 tokens per block
    ((4, 8, 8, 1, 1, 64), vsa.VSA_ERR_UNSUPPORTED),  # bw > 32
])
def test_plan_rejects_bad_geometry(L, args, code):
    h = ctypes.c_void_p()
    assert L.vsa_plan_create(*args, ctypes.byref(h)) == code
    assert not h.value


def test_plan_rejects_null_out(L):
    assert L.vsa_plan_create(4, 8, 8, 4, 8, 8, None) == vsa.VSA_ERR_INVALID_ARG


def test_describe_rejects_bad_topk(L):
    p = vsa.Plan(31, 22, 40)
    buf = ctypes.create_string_buffer(256)
    assert L.vsa_plan_describe(p.handle, 0, buf, 256) == vsa.VSA_ERR_TOPK
    assert L.vsa_plan_describe(p.handle, 121, buf, 256) == vsa.VSA_ERR_TOPK


def test_calls_reject_invalid_arguments(L):
    p = vsa.Plan(8, 16, 16)
    h = p.handle
    F, M = ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 8)  # aligned / misaligned
    # tile / untile
    assert L.vsa_tile(None, F, F, None, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile(h, None, F, None, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile(h, M, F, None, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile(h, F, F, M, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile(h, F, F, None, 0, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile(h, F, F, None, 1, 2, 64, None) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_untile(h, F, M, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_untile(h, F, F, 1, 2, 96, None) == vsa.VSA_ERR_UNSUPPORTED
    # coarse stage: topk must satisfy 0 < topk <= NB (NB = 8 here)
    assert L.vsa_coarse_topk(h, F, F, 1, 2, 128, 0, F, F, None) == vsa.VSA_ERR_TOPK
    assert L.vsa_coarse_topk(h, F, F, 1, 2, 128, 9, F, F, None) == vsa.VSA_ERR_TOPK
    assert L.vsa_coarse_topk(h, F, M, 1, 2, 128, 4, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    # map compaction
    assert L.vsa_map_to_index(None, 1, 1, 4, 4, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_map_to_index(F, 1, 1, 0, 4, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    # fine stage
    assert L.vsa_sparse_attn_fwd(h, F, F, F, F, F, 0, 1, 2, 128, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd(h, F, F, M, F, F, 4, 1, 2, 128, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd(h, F, F, F, F, F, 4, 1, 2, 256, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    odd = vsa.Plan(4, 4, 12, (4, 4, 4))  # 3 tiles of 64: the tile count must be even
    assert L.vsa_sparse_attn_fwd(odd.handle, F, F, F, F, F, 4, 1, 2, 128, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_get_status(None, None) == vsa.VSA_ERR_INVALID_ARG
    # dtype must be one of the two 16-bit formats
    assert L.vsa_tile_ex(h, 7, F, F, None, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_ex(h, 2, F, F, F, F, F, 4, 1, 2, 128, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_ex(h, vsa.VSA_F16, F, F, F, F, F, 4, 1, 2, 96, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    # compression branch: 0 <= topk <= NB; index outputs exactly when topk > 0
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, -1, None, None, F, None) == vsa.VSA_ERR_TOPK
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, 9, F, F, F, None) == vsa.VSA_ERR_TOPK
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, 0, F, None, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, 4, None, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_coarse_compress(h, F, F, M, 1, 2, 128, 4, F, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, 4, F, F, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 64, 4, F, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    # one-launch front end: workspace required; vbar and o_compress together
    args = lambda topk, vb, idx, num, oc, ws: (h, vsa.VSA_BF16, F, F, F, 1, 2, 128, topk, F, F, F, F, F, vb, idx,
                                                num, oc, ws, None)
    assert L.vsa_tile_coarse(*args(4, None, F, F, None, None)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile_coarse(*args(4, None, F, F, None, M)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile_coarse(*args(4, F, F, F, None, F)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile_coarse(*args(4, None, F, F, F, F)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile_coarse(*args(9, None, F, F, None, F)) == vsa.VSA_ERR_TOPK
    assert L.vsa_tile_coarse(*args(-1, None, None, None, None, F)) == vsa.VSA_ERR_TOPK
    assert L.vsa_tile_coarse(*args(0, None, F, None, None, F)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_tile_coarse(*args(4, None, None, F, None, F)) == vsa.VSA_ERR_INVALID_ARG
    # backward: dtype, pointers, sizes, block size
    bw = lambda dt, ws, mk, D, plan=h: (plan, dt, F, F, F, F, F, F, F, F, mk, 1, 2, D, F, F, F, ws, None)
    assert L.vsa_sparse_attn_bwd(*bw(3, F, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_bwd(*bw(vsa.VSA_BF16, None, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_bwd(*bw(vsa.VSA_BF16, M, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_bwd(*bw(vsa.VSA_BF16, F, 0, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_bwd(*bw(vsa.VSA_F16, F, 4, 64)) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_sparse_attn_bwd_workspace(h, 1, 2, 0, ctypes.byref(ctypes.c_size_t())) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_bwd_workspace(h, 1, 2, 4, None) == vsa.VSA_ERR_INVALID_ARG
    # gated untile
    assert L.vsa_untile_gate(h, 5, F, F, F, F, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_untile_gate(h, vsa.VSA_BF16, F, F, M, F, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_untile_gate(h, vsa.VSA_BF16, F, None, F, F, 1, 2, 128, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_untile_gate(h, vsa.VSA_F16, F, F, F, F, 1, 2, 96, None) == vsa.VSA_ERR_UNSUPPORTED
    # NVFP4: dtype, pointers, head size, whole 128-row scale tiles
    assert L.vsa_quantize_nvfp4(h, 2, F, 1, 2, 128, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_quantize_nvfp4(h, vsa.VSA_BF16, F, 1, 2, 128, F, M, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_quantize_nvfp4(None, vsa.VSA_BF16, F, 1, 2, 128, F, F, None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_quantize_nvfp4(h, vsa.VSA_BF16, F, 1, 2, 64, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_quantize_nvfp4(odd.handle, vsa.VSA_BF16, F, 1, 2, 128, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    f4 = lambda dt, qs, mk, D, plan=h: (plan, dt, F, qs, F, F, F, F, F, mk, 1, 2, D, F, F, None)
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(3, F, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(vsa.VSA_BF16, M, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(vsa.VSA_BF16, None, 4, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(vsa.VSA_BF16, F, 0, 128)) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(vsa.VSA_F16, F, 4, 256)) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_sparse_attn_fwd_nvfp4(*f4(vsa.VSA_BF16, F, 4, 128, odd.handle)) == vsa.VSA_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_reports_no_device(L):
    p = vsa.Plan(8, 16, 16)
    F = ctypes.c_void_p(FAKE)
    assert L.vsa_tile(p.handle, F, F, None, 1, 2, 128, None) == vsa.VSA_ERR_NO_DEVICE


def test_backward_workspace_size_is_host_only():
    p = vsa.Plan(31, 22, 40)
    a = vsa.bwd_workspace_bytes(p, 1, 24, 64)
    b = vsa.bwd_workspace_bytes(p, 1, 24, 65)
    assert a > 2 * 24 * p.Sp * 4 and b > a and a % 4 == 0


def test_coarse_calls_reject_more_than_2048_blocks(L):
    """The coarse stage stages eight rows of NB scores in shared memory: NB <= 2048."""
    big = vsa.Plan(64, 128, 72)  # 16 x 16 x 9 = 2304 blocks
    assert big.NB == 2304
    h = big.handle
    F = ctypes.c_void_p(FAKE)
    assert L.vsa_coarse_topk(h, F, F, 1, 2, 128, 4, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_coarse_compress(h, F, F, F, 1, 2, 128, 4, F, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    front = (h, vsa.VSA_BF16, F, F, F, 1, 2, 128, 4, F, F, F, F, F, None, F, F, None)
    assert L.vsa_tile_coarse(*front, F, None) == vsa.VSA_ERR_UNSUPPORTED
    assert L.vsa_tile_coarse_static(*front, None) == vsa.VSA_ERR_UNSUPPORTED


def test_prefix_selection_calls_reject_invalid_arguments(L):
    """Tile-64 selection: 0 < topk <= video tiles, a row stride that holds the
    longest row (NB with prefix tiles), aligned pointers, NB <= 2048."""
    p = vsa.Plan(4, 8, 12, (4, 4, 4), n_prefix=130)  # 3 prefix tiles + 6 video tiles
    assert p.NB == 9
    h = p.handle
    F, M = ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 8)
    call = lambda topk, max_k, keep=None, qbar=F, plan=h: L.vsa_coarse_topk_prefix(
        plan, qbar, F, keep, 1, 2, 128, topk, max_k, F, F, None)
    assert call(0, 9) == vsa.VSA_ERR_TOPK
    assert call(7, 9) == vsa.VSA_ERR_TOPK           # only 6 video tiles
    assert call(2, 8) == vsa.VSA_ERR_INVALID_ARG    # prefix rows need all 9 entries
    assert call(2, 9, keep=M) == vsa.VSA_ERR_INVALID_ARG
    assert call(2, 9, qbar=M) == vsa.VSA_ERR_INVALID_ARG
    assert call(2, 9, plan=None) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_coarse_topk_prefix(h, F, F, None, 1, 2, 64, 2, 9, F, F, None) == vsa.VSA_ERR_UNSUPPORTED
    plain = vsa.Plan(8, 16, 16)  # no prefix: the stride only needs topk entries
    assert call(3, 2, plan=plain.handle) == vsa.VSA_ERR_INVALID_ARG
    assert call(9, 9, plan=plain.handle) == vsa.VSA_ERR_TOPK
    big = vsa.Plan(64, 128, 72)
    assert call(4, big.NB, plan=big.handle) == vsa.VSA_ERR_UNSUPPORTED
    front = lambda topk, max_k, ws=F, dt=vsa.VSA_BF16: L.vsa_tile_coarse_prefix(
        h, dt, F, F, F, None, 1, 2, 128, topk, max_k, F, F, F, F, F, F, F, ws, None)
    assert front(7, 9) == vsa.VSA_ERR_TOPK
    assert front(2, 8) == vsa.VSA_ERR_INVALID_ARG
    assert front(2, 9, ws=None) == vsa.VSA_ERR_INVALID_ARG
    assert front(2, 9, ws=M) == vsa.VSA_ERR_INVALID_ARG
    assert front(2, 9, dt=5) == vsa.VSA_ERR_INVALID_ARG


def test_backward_rejects_more_than_28672_blocks(L):
    """The backward builds each head's transposed selection in shared memory
    (8 bytes per block): NB <= 28672, checked before any launch."""
    big = vsa.Plan(128, 128, 128, (4, 4, 4))  # 32 x 32 x 32 = 32768 tiles of 64
    assert big.NB == 32768
    F = ctypes.c_void_p(FAKE)
    args = (big.handle, vsa.VSA_BF16, F, F, F, F, F, F, F, F, 4, 1, 2, 128, F, F, F, F, None)
    assert L.vsa_sparse_attn_bwd(*args) == vsa.VSA_ERR_UNSUPPORTED


def test_fine_stage_with_workspace_checks_it(L):
    p = vsa.Plan(8, 16, 16)
    F, M = ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 8)
    call = lambda ws: L.vsa_sparse_attn_fwd_ws(p.handle, vsa.VSA_BF16, F, F, F, F, F, 4, 1, 2, 128, F, F, ws, None)
    assert call(None) == vsa.VSA_ERR_INVALID_ARG
    assert call(M) == vsa.VSA_ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd_ws(p.handle, vsa.VSA_BF16, F, F, F, F, F, 4, 1, 2, 96, F, F, F, None) \
        == vsa.VSA_ERR_UNSUPPORTED
    call4 = lambda ws: L.vsa_sparse_attn_fwd_nvfp4_ws(p.handle, vsa.VSA_BF16, F, F, F, F, F, F, F, 4, 1, 2, 128,
                                                     F, F, ws, None)
    assert call4(None) == vsa.VSA_ERR_INVALID_ARG
    assert call4(M) == vsa.VSA_ERR_INVALID_ARG
