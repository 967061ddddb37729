"""Video Sparse Attention forward path on B200 -- Python binding of libvsa.so.

The binding only marshals arguments: torch CUDA tensors become device
pointers, the current torch stream becomes the launch stream, and outputs are
allocated with torch when the caller does not pass them.  Every step of the
path runs in the CUDA library (include/vsa.h).  There is no fallback: if
libvsa.so is missing or a call fails, a ``VSAError`` is raised.

Path ("FastVideo VSA", vLLM-Omni user guide, introduction):
    tile(q, k, v) -> coarse_topk(qbar, kbar) -> sparse_attn_fwd -> untile(o)
or, with a caller-supplied bool block map (FastVideo commit log),
    tile -> map_to_index(map) -> sparse_attn_fwd -> untile.
With the gate-compress branch ("FastVideo VSA", section "Checkpoint
behavior"), v is pooled too, coarse_compress adds the block-level branch to
the selection, and untile_gate sums the two branches under the caller's gate.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvsa.so")

# Every symbol include/vsa.h declares.
SYMBOLS = (
    "vsa_plan_create", "vsa_plan_create_prefix", "vsa_plan_destroy", "vsa_plan_sizes",
    "vsa_plan_describe", "vsa_tile", "vsa_tile_ex", "vsa_untile", "vsa_coarse_topk", "vsa_map_to_index",
    "vsa_sparse_attn_fwd", "vsa_sparse_attn_fwd_ex", "vsa_get_status", "vsa_strerror",
    "vsa_coarse_compress", "vsa_untile_gate", "vsa_tile_coarse", "vsa_tile_coarse_static",
    "vsa_sparse_attn_bwd_workspace", "vsa_sparse_attn_bwd", "vsa_quantize_nvfp4", "vsa_sparse_attn_fwd_nvfp4",
    "vsa_coarse_topk_prefix", "vsa_tile_coarse_prefix", "vsa_sparse_attn_fwd_ws", "vsa_sparse_attn_fwd_nvfp4_ws",
)

VSA_BF16 = 0
VSA_F16 = 1

VSA_OK = 0
VSA_ERR_INVALID_ARG = 1
VSA_ERR_UNSUPPORTED = 2
VSA_ERR_TOPK = 3
VSA_ERR_CUDA = 4
VSA_ERR_BAD_INDEX = 5
VSA_ERR_TIMEOUT = 6
VSA_ERR_NO_DEVICE = 7

_lib = None


class VSAError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = _lib.vsa_strerror(code).decode() if _lib is not None else f"status {code}"
        super().__init__(f"{what}: {msg} (code {code})" if what else f"{msg} (code {code})")


def lib():
    """Load libvsa.so (built in-tree); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m block_sparse_video_gather_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.vsa_plan_create.argtypes = [i, i, i, i, i, i, P]
        L.vsa_plan_create_prefix.argtypes = [i, i, i, i, i, i, i, P]
        L.vsa_plan_destroy.argtypes = [P]
        L.vsa_plan_destroy.restype = None
        L.vsa_plan_sizes.argtypes = [P, P, P, P, P]
        L.vsa_plan_describe.argtypes = [P, i, ctypes.c_char_p, sz]
        L.vsa_tile.argtypes = [P, P, P, P, i, i, i, P]
        L.vsa_tile_ex.argtypes = [P, i, P, P, P, i, i, i, P]
        L.vsa_sparse_attn_fwd_ex.argtypes = [P, i, P, P, P, P, P, i, i, i, i, P, P, P]
        L.vsa_sparse_attn_fwd_ws.argtypes = [P, i, P, P, P, P, P, i, i, i, i, P, P, P, P]
        L.vsa_untile.argtypes = [P, P, P, i, i, i, P]
        L.vsa_coarse_topk.argtypes = [P, P, P, i, i, i, i, P, P, P]
        L.vsa_map_to_index.argtypes = [P, i, i, i, i, P, P, P]
        L.vsa_coarse_topk_prefix.argtypes = [P, P, P, P, i, i, i, i, i, P, P, P]
        L.vsa_tile_coarse_prefix.argtypes = [P, i, P, P, P, P, i, i, i, i, i] + [P] * 9
        L.vsa_coarse_compress.argtypes = [P, P, P, P, i, i, i, i, P, P, P, P]
        L.vsa_untile_gate.argtypes = [P, i, P, P, P, P, i, i, i, P]
        L.vsa_tile_coarse.argtypes = [P, i, P, P, P, i, i, i, i] + [P] * 11
        L.vsa_tile_coarse_static.argtypes = [P, i, P, P, P, i, i, i, i] + [P] * 10
        L.vsa_sparse_attn_bwd_workspace.argtypes = [P, i, i, i, P]
        L.vsa_sparse_attn_bwd.argtypes = [P, i, P, P, P, P, P, P, P, P, i, i, i, i, P, P, P, P, P]
        L.vsa_sparse_attn_fwd.argtypes = [P, P, P, P, P, P, i, i, i, i, P, P, P]
        L.vsa_quantize_nvfp4.argtypes = [P, i, P, i, i, i, P, P, P]
        L.vsa_sparse_attn_fwd_nvfp4.argtypes = [P, i, P, P, P, P, P, P, P, i, i, i, i, P, P, P]
        L.vsa_sparse_attn_fwd_nvfp4_ws.argtypes = [P, i, P, P, P, P, P, P, P, i, i, i, i, P, P, P, P]
        L.vsa_get_status.argtypes = [P, P]
        L.vsa_strerror.argtypes = [i]
        L.vsa_strerror.restype = ctypes.c_char_p
        for name in SYMBOLS:
            if name not in ("vsa_plan_destroy", "vsa_strerror"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != VSA_OK:
        raise VSAError(rc, what)


class Plan:
    """Geometry of one latent grid: block partition, padding, block count."""

    def __init__(self, T: int, Hg: int, Wg: int, block=(4, 8, 8), n_prefix: int = 0):
        L = lib()
        h = ctypes.c_void_p()
        _check(L.vsa_plan_create_prefix(n_prefix, T, Hg, Wg, *block, ctypes.byref(h)), "vsa_plan_create")
        self._h = h
        nb, bs = ctypes.c_int(), ctypes.c_int()
        s, sp = ctypes.c_int64(), ctypes.c_int64()
        _check(L.vsa_plan_sizes(h, ctypes.byref(nb), ctypes.byref(s), ctypes.byref(sp), ctypes.byref(bs)),
               "vsa_plan_sizes")
        self.T, self.Hg, self.Wg, self.block, self.n_prefix = T, Hg, Wg, tuple(block), n_prefix
        self.NB, self.S, self.Sp, self.bs = nb.value, s.value, sp.value, bs.value

    @classmethod
    def of(cls, wl) -> "Plan":
        return cls(wl.T, wl.Hg, wl.Wg, wl.block, wl.n_prefix)

    @property
    def handle(self):
        return self._h

    def describe(self, topk: int) -> str:
        buf = ctypes.create_string_buffer(512)
        _check(lib().vsa_plan_describe(self._h, topk, buf, len(buf)), "vsa_plan_describe")
        return buf.value.decode()

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.vsa_plan_destroy(h)
            self._h = None


def _torch():
    import torch
    return torch


def _ptr(t, dtype, what):
    torch = _torch()
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(t, what):
    """bf16 -> VSA_BF16, fp16 -> VSA_F16 (the two formats the kernels take)."""
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return VSA_BF16
    if t.dtype == torch.float16:
        return VSA_F16
    raise ValueError(f"{what} must be bfloat16 or float16, got {t.dtype}")


def _stream():
    return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)


def tile(plan: Plan, x, pooled: bool = False, out=None, pooled_out=None):
    """x [B,S,H,D] bf16/fp16 -> x_tiled [B,H,Sp,D] (and fp32 block means [B,H,NB,D])."""
    torch = _torch()
    B, S, H, D = x.shape
    code = _dtype_code(x, "x")
    if out is None:
        out = torch.empty((B, H, plan.Sp, D), dtype=x.dtype, device=x.device)
    if pooled and pooled_out is None:
        pooled_out = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=x.device)
    if S != plan.S:
        raise ValueError(f"x has {S} tokens, plan expects {plan.S}")
    _check(lib().vsa_tile_ex(plan.handle, code, _ptr(x, x.dtype, "x"), _ptr(out, x.dtype, "x_tiled"),
                             _ptr(pooled_out, torch.float32, "pooled") if pooled else None, B, H, D, _stream()),
           "vsa_tile")
    return (out, pooled_out) if pooled else out


def untile(plan: Plan, xt, out=None):
    """x_tiled [B,H,Sp,D] bf16/fp16 -> x [B,S,H,D] (padded rows dropped)."""
    torch = _torch()
    B, H, Sp, D = xt.shape
    _dtype_code(xt, "x_tiled")
    if Sp != plan.Sp:
        raise ValueError(f"x_tiled has {Sp} rows, plan expects {plan.Sp}")
    if out is None:
        out = torch.empty((B, plan.S, H, D), dtype=xt.dtype, device=xt.device)
    _check(lib().vsa_untile(plan.handle, _ptr(xt, xt.dtype, "x_tiled"), _ptr(out, xt.dtype, "x"),
                            B, H, D, _stream()), "vsa_untile")
    return out


def coarse_topk(plan: Plan, qbar, kbar, topk: int, idx_out=None, num_out=None):
    """Block scores + per-row top-k -> (q2k_idx [B,H,NB,topk], q2k_num [B,H,NB])."""
    torch = _torch()
    B, H, NB, D = qbar.shape
    if idx_out is None:
        idx_out = torch.empty((B, H, NB, max(topk, 1)), dtype=torch.int32, device=qbar.device)
    if num_out is None:
        num_out = torch.empty((B, H, NB), dtype=torch.int32, device=qbar.device)
    _check(lib().vsa_coarse_topk(plan.handle, _ptr(qbar, torch.float32, "qbar"), _ptr(kbar, torch.float32, "kbar"),
                                 B, H, D, topk, _ptr(idx_out, torch.int32, "q2k_idx"),
                                 _ptr(num_out, torch.int32, "q2k_num"), _stream()), "vsa_coarse_topk")
    return idx_out, num_out


def coarse_topk_prefix(plan: Plan, qbar, kbar, topk: int, row_keep=None, max_k: int | None = None, idx_out=None,
                       num_out=None):
    """Tile-64 selection: prefix query tiles take every block, video query tiles the
    prefix plus their top-k video blocks; rows whose row_keep byte [B,H,NB] is 0 take
    nothing -> (q2k_idx [B,H,NB,max_k] -1 padded, q2k_num [B,H,NB])."""
    torch = _torch()
    B, H, NB, D = qbar.shape
    if max_k is None:
        max_k = NB if plan.n_prefix > 0 else topk
    if idx_out is None:
        idx_out = torch.empty((B, H, NB, max_k), dtype=torch.int32, device=qbar.device)
    if num_out is None:
        num_out = torch.empty((B, H, NB), dtype=torch.int32, device=qbar.device)
    _check(lib().vsa_coarse_topk_prefix(plan.handle, _ptr(qbar, torch.float32, "qbar"),
                                        _ptr(kbar, torch.float32, "kbar"), _ptr(row_keep, torch.uint8, "row_keep"),
                                        B, H, D, topk, max_k, _ptr(idx_out, torch.int32, "q2k_idx"),
                                        _ptr(num_out, torch.int32, "q2k_num"), _stream()), "vsa_coarse_topk_prefix")
    return idx_out, num_out


def coarse_compress(plan: Plan, qbar, kbar, vbar, topk: int = 0, o_out=None, idx_out=None, num_out=None):
    """Compression branch o_compress [B,H,NB,D] fp32: attention among the block
    means.  With topk > 0 the same launch also writes the selection of
    coarse_topk; returns (o_compress, q2k_idx, q2k_num) then, else o_compress."""
    torch = _torch()
    B, H, NB, D = qbar.shape
    if o_out is None:
        o_out = torch.empty((B, H, NB, D), dtype=torch.float32, device=qbar.device)
    if topk > 0:
        if idx_out is None:
            idx_out = torch.empty((B, H, NB, topk), dtype=torch.int32, device=qbar.device)
        if num_out is None:
            num_out = torch.empty((B, H, NB), dtype=torch.int32, device=qbar.device)
        ip, nump = _ptr(idx_out, torch.int32, "q2k_idx"), _ptr(num_out, torch.int32, "q2k_num")
    else:
        ip = nump = None
    _check(lib().vsa_coarse_compress(plan.handle, _ptr(qbar, torch.float32, "qbar"), _ptr(kbar, torch.float32, "kbar"),
                                     _ptr(vbar, torch.float32, "vbar"), B, H, D, topk, ip, nump,
                                     _ptr(o_out, torch.float32, "o_compress"), _stream()), "vsa_coarse_compress")
    return (o_out, idx_out, num_out) if topk > 0 else o_out


def workspace(B: int, H: int, device="cuda"):
    """The zeroed 2*B*H int32 workspace tile_coarse synchronises its CTAs with."""
    return _torch().zeros(2 * B * H, dtype=_torch().int32, device=device)


def tile_coarse(plan: Plan, q, k, v, topk: int, ws, gated: bool = False, out: dict | None = None):
    """Front end in one launch: tile q, k, v with block means, then the coarse
    stage (topk > 0) and, when gated, the compression branch.  Returns a dict
    with qt, kt, vt, qbar, kbar (+ vbar, oc when gated; + idx, num when topk > 0);
    tensors given in `out` are written in place.  ws=None runs
    vsa_tile_coarse_static (the library's own counters, B*H <= 4096)."""
    torch = _torch()
    B, S, H, D = q.shape
    code = _dtype_code(q, "q")
    if S != plan.S:
        raise ValueError(f"q has {S} tokens, plan expects {plan.S}")
    o = dict(out or {})
    for n in ("qt", "kt", "vt"):
        if n not in o:
            o[n] = torch.empty((B, H, plan.Sp, D), dtype=q.dtype, device=q.device)
    names = ["qbar", "kbar"] + (["vbar", "oc"] if gated else [])
    for n in names:
        if n not in o:
            o[n] = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=q.device)
    if topk > 0:
        if "idx" not in o:
            o["idx"] = torch.empty((B, H, plan.NB, topk), dtype=torch.int32, device=q.device)
        if "num" not in o:
            o["num"] = torch.empty((B, H, plan.NB), dtype=torch.int32, device=q.device)
    f32, i32 = torch.float32, torch.int32
    args = [
        plan.handle, code, _ptr(q, q.dtype, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"), B, H, D, topk,
        _ptr(o["qt"], q.dtype, "q_tiled"), _ptr(o["kt"], q.dtype, "k_tiled"), _ptr(o["vt"], q.dtype, "v_tiled"),
        _ptr(o["qbar"], f32, "qbar"), _ptr(o["kbar"], f32, "kbar"), _ptr(o["vbar"], f32, "vbar") if gated else None,
        _ptr(o["idx"], i32, "q2k_idx") if topk > 0 else None, _ptr(o["num"], i32, "q2k_num") if topk > 0 else None,
        _ptr(o["oc"], f32, "o_compress") if gated else None]
    if ws is None:
        _check(lib().vsa_tile_coarse_static(*args, _stream()), "vsa_tile_coarse_static")
    else:
        _check(lib().vsa_tile_coarse(*args, _ptr(ws, i32, "workspace"), _stream()), "vsa_tile_coarse")
    return o


def tile_coarse_prefix(plan: Plan, q, k, v, topk: int, ws, row_keep=None, max_k: int | None = None,
                       out: dict | None = None):
    """Front end in one launch with the tile-64 selection (coarse_topk_prefix): tile q, k, v
    with block means of q and k, then the selection.  Returns a dict with qt, kt, vt, qbar,
    kbar, idx, num; tensors given in `out` are written in place."""
    torch = _torch()
    B, S, H, D = q.shape
    code = _dtype_code(q, "q")
    if S != plan.S:
        raise ValueError(f"q has {S} tokens, plan expects {plan.S}")
    if max_k is None:
        max_k = plan.NB if plan.n_prefix > 0 else topk
    o = dict(out or {})
    for n in ("qt", "kt", "vt"):
        if n not in o:
            o[n] = torch.empty((B, H, plan.Sp, D), dtype=q.dtype, device=q.device)
    for n in ("qbar", "kbar"):
        if n not in o:
            o[n] = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=q.device)
    if "idx" not in o:
        o["idx"] = torch.empty((B, H, plan.NB, max_k), dtype=torch.int32, device=q.device)
    if "num" not in o:
        o["num"] = torch.empty((B, H, plan.NB), dtype=torch.int32, device=q.device)
    f32, i32 = torch.float32, torch.int32
    _check(lib().vsa_tile_coarse_prefix(
        plan.handle, code, _ptr(q, q.dtype, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
        _ptr(row_keep, torch.uint8, "row_keep"), B, H, D, topk, max_k,
        _ptr(o["qt"], q.dtype, "q_tiled"), _ptr(o["kt"], q.dtype, "k_tiled"), _ptr(o["vt"], q.dtype, "v_tiled"),
        _ptr(o["qbar"], f32, "qbar"), _ptr(o["kbar"], f32, "kbar"), _ptr(o["idx"], i32, "q2k_idx"),
        _ptr(o["num"], i32, "q2k_num"), _ptr(ws, i32, "workspace"), _stream()), "vsa_tile_coarse_prefix")
    return o


def untile_gate(plan: Plan, ot, o_compress, gate, out=None):
    """o [B,S,H,D] = untile(ot) + gate * o_compress of each token's block (gate untiled, same dtype)."""
    torch = _torch()
    B, H, Sp, D = ot.shape
    code = _dtype_code(ot, "o_tiled")
    if Sp != plan.Sp:
        raise ValueError(f"o_tiled has {Sp} rows, plan expects {plan.Sp}")
    if tuple(gate.shape) != (B, plan.S, H, D):
        raise ValueError(f"gate must be [B,S,H,D] = {(B, plan.S, H, D)}, got {tuple(gate.shape)}")
    if out is None:
        out = torch.empty((B, plan.S, H, D), dtype=ot.dtype, device=ot.device)
    _check(lib().vsa_untile_gate(plan.handle, code, _ptr(ot, ot.dtype, "o_tiled"),
                                 _ptr(o_compress, torch.float32, "o_compress"), _ptr(gate, ot.dtype, "gate"),
                                 _ptr(out, ot.dtype, "o"), B, H, D, _stream()), "vsa_untile_gate")
    return out


def map_to_index(block_map, idx_out=None, num_out=None):
    """Bool map [B,H,NQ,NK] -> (q2k_idx [B,H,NQ,NK] ascending then -1, q2k_num [B,H,NQ])."""
    torch = _torch()
    m = block_map.view(torch.uint8) if block_map.dtype == torch.bool else block_map
    B, H, NQ, NK = m.shape
    if idx_out is None:
        idx_out = torch.empty((B, H, NQ, NK), dtype=torch.int32, device=m.device)
    if num_out is None:
        num_out = torch.empty((B, H, NQ), dtype=torch.int32, device=m.device)
    _check(lib().vsa_map_to_index(_ptr(m, torch.uint8, "map"), B, H, NQ, NK, _ptr(idx_out, torch.int32, "q2k_idx"),
                                  _ptr(num_out, torch.int32, "q2k_num"), _stream()), "vsa_map_to_index")
    return idx_out, num_out


def sparse_attn_fwd(plan: Plan, q, k, v, q2k_idx, q2k_num, o_out=None, lse_out=None, workspace=None):
    """Attention of every query block over its selected blocks (tiled layout) -> (o, lse).
    workspace: optional zeroed int32 tensor of 4 entries (2 used) for the 64-token
    kernel's shared work queue (vsa_sparse_attn_fwd_ws); left zero by every call."""
    torch = _torch()
    B, H, Sp, D = q.shape
    max_k = q2k_idx.shape[-1]
    code = _dtype_code(q, "q")
    if o_out is None:
        o_out = torch.empty_like(q)
    if lse_out is None:
        lse_out = torch.empty((B, H, Sp), dtype=torch.float32, device=q.device)
    args = (plan.handle, code, _ptr(q, q.dtype, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
            _ptr(q2k_idx, torch.int32, "q2k_idx"), _ptr(q2k_num, torch.int32, "q2k_num"), max_k, B, H, D,
            _ptr(o_out, q.dtype, "o"), _ptr(lse_out, torch.float32, "lse"))
    if workspace is None:
        _check(lib().vsa_sparse_attn_fwd_ex(*args, _stream()), "vsa_sparse_attn_fwd")
    else:
        _check(lib().vsa_sparse_attn_fwd_ws(*args, _ptr(workspace, torch.int32, "workspace"), _stream()),
               "vsa_sparse_attn_fwd_ws")
    return o_out, lse_out


def quantize_nvfp4(plan: Plan, xt, codes=None, scales=None):
    """Tiled q or k [B,H,Sp,D] -> NVFP4 (codes [B,H,Sp,D/2] uint8, scales [B,H,Sp/128,1024] uint8 in the
    tensor core's layout; see vsa_quantize_nvfp4)."""
    torch = _torch()
    B, H, Sp, D = xt.shape
    code = _dtype_code(xt, "x_tiled")
    if codes is None:
        codes = torch.empty((B, H, Sp, D // 2), dtype=torch.uint8, device=xt.device)
    if scales is None:
        scales = torch.empty((B, H, Sp // 128, 64 * D // 8), dtype=torch.uint8, device=xt.device)
    if codes.numel() != B * H * Sp * D // 2 or scales.numel() != B * H * Sp * D // 16:
        raise ValueError("codes / scales have the wrong size")
    _check(lib().vsa_quantize_nvfp4(plan.handle, code, _ptr(xt, xt.dtype, "x_tiled"), B, H, D,
                                    _ptr(codes, torch.uint8, "codes"), _ptr(scales, torch.uint8, "scales"),
                                    _stream()), "vsa_quantize_nvfp4")
    return codes, scales


def sparse_attn_fwd_nvfp4(plan: Plan, q_codes, q_scales, k_codes, k_scales, v, q2k_idx, q2k_num, o_out=None,
                          lse_out=None, workspace=None):
    """Fine stage with NVFP4 q, k (from quantize_nvfp4) and 16-bit v (tiled layout) -> (o, lse).
    workspace: optional zeroed int32 device tensor of >= 2 elements for the 64-token
    kernel's shared work queue (vsa_sparse_attn_fwd_nvfp4_ws); left zero by every call."""
    torch = _torch()
    B, H, Sp, D = v.shape
    max_k = q2k_idx.shape[-1]
    code = _dtype_code(v, "v")
    for t, n in ((q_codes, "q_codes"), (k_codes, "k_codes")):
        if t.numel() != B * H * Sp * D // 2:
            raise ValueError(f"{n} has the wrong size")
    for t, n in ((q_scales, "q_scales"), (k_scales, "k_scales")):
        if t.numel() != B * H * Sp * D // 16:
            raise ValueError(f"{n} has the wrong size")
    if o_out is None:
        o_out = torch.empty_like(v)
    if lse_out is None:
        lse_out = torch.empty((B, H, Sp), dtype=torch.float32, device=v.device)
    u8 = torch.uint8
    args = [plan.handle, code, _ptr(q_codes, u8, "q_codes"), _ptr(q_scales, u8, "q_scales"),
            _ptr(k_codes, u8, "k_codes"), _ptr(k_scales, u8, "k_scales"), _ptr(v, v.dtype, "v"),
            _ptr(q2k_idx, torch.int32, "q2k_idx"), _ptr(q2k_num, torch.int32, "q2k_num"), max_k, B, H, D,
            _ptr(o_out, v.dtype, "o"), _ptr(lse_out, torch.float32, "lse")]
    if workspace is None:
        _check(lib().vsa_sparse_attn_fwd_nvfp4(*args, _stream()), "vsa_sparse_attn_fwd_nvfp4")
    else:
        if workspace.numel() < 2:
            raise ValueError("workspace needs 2 int32")
        _check(lib().vsa_sparse_attn_fwd_nvfp4_ws(*args, _ptr(workspace, torch.int32, "workspace"), _stream()),
               "vsa_sparse_attn_fwd_nvfp4_ws")
    return o_out, lse_out


def bwd_workspace_bytes(plan: Plan, B: int, H: int, max_k: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().vsa_sparse_attn_bwd_workspace(plan.handle, B, H, max_k, ctypes.byref(n)),
           "vsa_sparse_attn_bwd_workspace")
    return n.value


def sparse_attn_bwd(plan: Plan, q, k, v, o, lse, do, q2k_idx, q2k_num, dq=None, dk=None, dv=None, workspace=None):
    """Gradients of the fine stage (tiled layout) -> (dq, dk, dv), selection fixed."""
    torch = _torch()
    B, H, Sp, D = q.shape
    max_k = q2k_idx.shape[-1]
    code = _dtype_code(q, "q")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(plan, B, H, max_k), dtype=torch.uint8, device=q.device)
    t = q.dtype
    _check(lib().vsa_sparse_attn_bwd(
        plan.handle, code, _ptr(q, t, "q"), _ptr(k, t, "k"), _ptr(v, t, "v"), _ptr(o, t, "o"),
        _ptr(lse, torch.float32, "lse"), _ptr(do, t, "do"), _ptr(q2k_idx, torch.int32, "q2k_idx"),
        _ptr(q2k_num, torch.int32, "q2k_num"), max_k, B, H, D, _ptr(dq, t, "dq"), _ptr(dk, t, "dk"),
        _ptr(dv, t, "dv"), _ptr(workspace, torch.uint8, "workspace"), _stream()), "vsa_sparse_attn_bwd")
    return dq, dk, dv


def get_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the device status word."""
    torch = _torch()
    st = ctypes.c_int(0)
    s = ctypes.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
    _check(lib().vsa_get_status(s, ctypes.byref(st)), "vsa_get_status")
    return st.value


class Forward:
    """The whole forward path with its intermediates allocated once.

    __call__(q, k, v[, block_map]) runs the front end (tile q, k, v with
    block means and the coarse stage, or map_to_index when a block map is
    given), the fine stage and untile(o); it returns o [B,S,H,D] and the tiled
    lse [B,H,Sp].  The three stages are also callable one by one (front,
    fine, back).

    prefix_dense=True selects with the tile-64 rule (coarse_topk_prefix:
    prefix query tiles take every block, video query tiles the prefix plus
    their top-k video blocks); __call__ then takes the optional row-keep mask
    [B,H,NB] uint8 (0 = row forced empty) as row_keep=.

    fused=True (default) runs the front end as one launch (tile_coarse);
    fused=False as separate tile / coarse launches.

    gated=True adds the gate-compress branch: v is pooled as well, the coarse
    stage also computes o_compress, and untile_gate replaces untile, so
    __call__(q, k, v, gate=g) returns o_fine + g * o_compress per token
    (g [B,S,H,D], same dtype as q).

    nvfp4=True runs the fine stage with NVFP4 q and k: the tiled q and k are
    quantised (two launches) and the FP4 attention kernel replaces the 16-bit
    one; v stays 16-bit.
    """

    def __init__(self, plan: Plan, B: int, H: int, topk: int | None, device="cuda", D: int = 128, dtype=None,
                 gated: bool = False, fused: bool = True, nvfp4: bool = False, prefix_dense: bool = False):
        torch = _torch()
        if prefix_dense and (gated or topk is None):
            raise ValueError("prefix_dense needs a top-k and no gate-compress branch")
        self.plan, self.B, self.H, self.D, self.topk = plan, B, H, D, topk
        self.gated, self.fused, self.nvfp4, self.prefix_dense = gated, fused, nvfp4, prefix_dense
        t = dict(dtype=dtype or torch.bfloat16, device=device)
        self.qt = torch.empty((B, H, plan.Sp, D), **t)
        self.kt = torch.empty((B, H, plan.Sp, D), **t)
        self.vt = torch.empty((B, H, plan.Sp, D), **t)
        self.ot = torch.empty((B, H, plan.Sp, D), **t)
        self.o = torch.empty((B, plan.S, H, D), **t)
        self.lse = torch.empty((B, H, plan.Sp), dtype=torch.float32, device=device)
        self.qbar = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=device)
        self.kbar = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=device)
        width = topk if (topk is not None and not (prefix_dense and plan.n_prefix > 0)) else plan.NB
        self.idx = torch.empty((B, H, plan.NB, width), dtype=torch.int32, device=device)
        self.num = torch.empty((B, H, plan.NB), dtype=torch.int32, device=device)
        if gated:
            self.vbar = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=device)
            self.oc = torch.empty((B, H, plan.NB, D), dtype=torch.float32, device=device)
        if fused:
            self.ws = workspace(B, H, device)
        self.fws = torch.zeros(4, dtype=torch.int32, device=device)  # the fine stage's work queue
        if nvfp4:
            u8 = dict(dtype=torch.uint8, device=device)
            self.qc = torch.empty((B, H, plan.Sp, D // 2), **u8)
            self.kc = torch.empty((B, H, plan.Sp, D // 2), **u8)
            self.qs = torch.empty((B, H, plan.Sp // 128, 64 * D // 8), **u8)
            self.ks = torch.empty((B, H, plan.Sp // 128, 64 * D // 8), **u8)

    def front(self, q, k, v, block_map=None, row_keep=None):
        p = self.plan
        if row_keep is not None and not self.prefix_dense:
            raise ValueError("row_keep applies to the tile-64 selection (prefix_dense=True)")
        if self.prefix_dense:
            if block_map is not None:
                raise ValueError("prefix_dense computes the selection; no block map")
            if self.fused:
                out = dict(qt=self.qt, kt=self.kt, vt=self.vt, qbar=self.qbar, kbar=self.kbar, idx=self.idx,
                           num=self.num)
                tile_coarse_prefix(p, q, k, v, self.topk, self.ws, row_keep, self.idx.shape[-1], out)
            else:
                tile(p, q, pooled=True, out=self.qt, pooled_out=self.qbar)
                tile(p, k, pooled=True, out=self.kt, pooled_out=self.kbar)
                tile(p, v, out=self.vt)
                coarse_topk_prefix(p, self.qbar, self.kbar, self.topk, row_keep, self.idx.shape[-1],
                                   idx_out=self.idx, num_out=self.num)
            return
        if self.fused:
            out = dict(qt=self.qt, kt=self.kt, vt=self.vt, qbar=self.qbar, kbar=self.kbar)
            if self.gated:
                out.update(vbar=self.vbar, oc=self.oc)
            if block_map is None:
                out.update(idx=self.idx, num=self.num)
            tile_coarse(p, q, k, v, self.topk if block_map is None else 0, self.ws, self.gated, out)
            if block_map is not None:
                map_to_index(block_map, idx_out=self.idx, num_out=self.num)
            return
        tile(p, q, pooled=True, out=self.qt, pooled_out=self.qbar)
        tile(p, k, pooled=True, out=self.kt, pooled_out=self.kbar)
        if self.gated:
            tile(p, v, pooled=True, out=self.vt, pooled_out=self.vbar)
        else:
            tile(p, v, out=self.vt)
        if block_map is None:
            if self.gated:
                coarse_compress(p, self.qbar, self.kbar, self.vbar, self.topk, o_out=self.oc, idx_out=self.idx,
                                num_out=self.num)
            else:
                coarse_topk(p, self.qbar, self.kbar, self.topk, idx_out=self.idx, num_out=self.num)
        else:
            map_to_index(block_map, idx_out=self.idx, num_out=self.num)
            if self.gated:
                coarse_compress(p, self.qbar, self.kbar, self.vbar, 0, o_out=self.oc)

    def quantize(self):
        """nvfp4: quantise the tiled q and k (nothing to do otherwise)."""
        if self.nvfp4:
            quantize_nvfp4(self.plan, self.qt, self.qc, self.qs)
            quantize_nvfp4(self.plan, self.kt, self.kc, self.ks)

    def attend(self):
        """The fine-stage attention kernel alone."""
        if self.nvfp4:
            sparse_attn_fwd_nvfp4(self.plan, self.qc, self.qs, self.kc, self.ks, self.vt, self.idx, self.num,
                                  o_out=self.ot, lse_out=self.lse, workspace=self.fws)
        else:
            sparse_attn_fwd(self.plan, self.qt, self.kt, self.vt, self.idx, self.num, o_out=self.ot,
                            lse_out=self.lse, workspace=self.fws)

    def fine(self):
        self.quantize()
        self.attend()

    def back(self, gate=None, out=None):
        out = self.o if out is None else out
        if self.gated:
            untile_gate(self.plan, self.ot, self.oc, gate, out=out)
        else:
            untile(self.plan, self.ot, out=out)
        return out

    def __call__(self, q, k, v, block_map=None, gate=None, out=None, row_keep=None):
        """One forward step; o goes to `out` when given (else to self.o)."""
        if self.gated != (gate is not None):
            raise ValueError("a gate is required exactly when the Forward was built with gated=True")
        self.front(q, k, v, block_map, row_keep)
        self.fine()
        return self.back(gate, out), self.lse

    def graph(self, q, k, v, block_map=None, gate=None, row_keep=None):
        """Capture one forward step on these device tensors in a CUDA graph and
        return it (torch.cuda.CUDAGraph); replay() reruns the step's launches
        with the inputs read from the same buffers and o / lse written to
        self.o / self.lse.  One eager step runs first so that every host-side
        set-up (device state, tensor-map encoder, kernel attributes) happens
        outside the capture."""
        torch = _torch()
        self(q, k, v, block_map, gate, row_keep=row_keep)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(q, k, v, block_map, gate, row_keep=row_keep)
        return g

    def launches(self, block_map: bool = False) -> int:
        """Kernels one call launches."""
        quant = 2 if self.nvfp4 else 0  # q and k quantisation
        if self.fused:
            return 3 + quant + (1 if block_map else 0)  # front (+ map_to_index), attention, untile
        return 6 + quant + (1 if (self.gated and block_map) else 0)  # 3 tiles, index stage (+compress), attention, untile


class HostPipeline:
    """Forward steps on pinned host tensors with the copies overlapped.

    submit(q, k, v, o[, block_map, gate, row_keep, lse]) enqueues one step:
    the inputs go to the device on a copy stream (into one of two input
    slots), the forward runs on a compute stream once they have landed, and o
    (and lse, when a host tensor is given) come back on a second copy stream
    (from one of two output slots).  While step i computes, step
    i+1's inputs and step i-1's output are in flight.  Calls return at once;
    synchronize() waits for every submitted step.  The host tensors must stay
    untouched until then.
    """

    def __init__(self, fwd: Forward, device="cuda"):
        torch = _torch()
        self.fwd = fwd
        self.h2d, self.comp, self.d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        self.slots_out = [torch.empty_like(fwd.o) for _ in range(2)]
        self.slots_lse = [torch.empty_like(fwd.lse) for _ in range(2)]
        self.slots_in = [None, None]
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_in, self.ev_used, self.ev_out, self.ev_back = ev(), ev(), ev(), ev()
        self.n = 0

    def _inputs(self, s, named):
        torch = _torch()
        if self.slots_in[s] is None:
            self.slots_in[s] = {k: torch.empty(t.shape, dtype=t.dtype, device="cuda") for k, t in named.items()}
        return self.slots_in[s]

    def submit(self, q, k, v, o, block_map=None, gate=None, row_keep=None, lse=None):
        """lse: an optional pinned host tensor [B,H,Sp] fp32 that receives the step's lse."""
        torch = _torch()
        s = self.n & 1
        named = {"q": q, "k": k, "v": v}
        if block_map is not None:
            named["map"] = block_map
        if gate is not None:
            named["gate"] = gate
        if row_keep is not None:
            named["row_keep"] = row_keep
        dev = self._inputs(s, named)
        with torch.cuda.stream(self.h2d):
            if self.n >= 2:
                self.h2d.wait_event(self.ev_used[s])  # step n-2 no longer reads this slot
            for name, src in named.items():
                dev[name].copy_(src, non_blocking=True)
            self.ev_in[s].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(self.ev_in[s])
            if self.n >= 2:
                self.comp.wait_event(self.ev_back[s])  # step n-2's output has left this slot
            self.fwd(dev["q"], dev["k"], dev["v"], dev.get("map"), dev.get("gate"), out=self.slots_out[s],
                     row_keep=dev.get("row_keep"))
            if lse is not None:
                self.slots_lse[s].copy_(self.fwd.lse)
            self.ev_used[s].record(self.comp)
            self.ev_out[s].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.ev_out[s])
            o.copy_(self.slots_out[s], non_blocking=True)
            if lse is not None:
                lse.copy_(self.slots_lse[s], non_blocking=True)
            self.ev_back[s].record(self.d2h)
        self.n += 1

    def synchronize(self):
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()
