"""CPU oracle of the Video Sparse Attention forward path (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it.

The arithmetic lives in ``vsa_oracle.c`` (plain C, built with gcc,
``-ffp-contract=off``); this module builds it on demand and wraps each
function for numpy arrays.  bf16 tensors travel as uint16 bit patterns.
Each step follows the statement cited in the C file's header:

* ``geometry``/``tile``/``untile``/``pool``/``score``/``topk``: "FastVideo VSA"
  (vLLM-Omni user guide), introduction and section "Choose top-k";
* ``map_to_index``: FastVideo commit log, examples/inference/basic/README.md;
* ``topk_prefix``: the same commit log's tile-64 layout (prefix query tiles
  dense, video query tiles the prefix plus a top-k of the video tiles, some
  rows forced empty), with the block score and tie rule of ``topk``;
* ``attn_rows``: "FastVideo VSA", introduction and section "Verify routing
  and fallback" (non-causal, scale head_size^-1/2), computed in fp64;
* ``attn_bwd_q_rows``/``attn_bwd_kv``/``attn_bwd_kv_blocks``: gradients of the attention step with
  the selection fixed (definition of softmax attention's derivative; the
  commit log keeps the grad path separate), in fp64, real query rows only;
* ``quant_nvfp4``/``dequant_nvfp4``/``attn_rows_nvfp4``: FastVideo
  "Optimizations" page, section "FP4 Flash Attention 4 (Blackwell only)" (Q
  and K as NVFP4: 4-bit E2M1 codes, one E4M3 scale per block of channels; V 16-bit); block length
  16 and the amax/6 scale are NVFP4's own definition, stated in the C file;
* ``compress``/``gate_rows``: "FastVideo VSA", section "Checkpoint behavior"
  (learned gate_compress projection) and the FastVideo commit log (the
  gate-compress branch pools per tile); the formula is a reading, stated in
  the C file: dense attention among block means, broadcast to the block's
  tokens, times the caller's gate, added to the sparse branch.

Pins (tests/test_oracle_*.py) check every function against results fixed by
the pages or by mathematics, never against itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vsa_oracle.c")
_LIB = os.path.join(_HERE, "libvsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile vsa_oracle.c into libvsa_oracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L = ctypes.c_long
        geo = [i] * 7
        lib.oracle_geometry.argtypes = geo + [P]
        lib.oracle_block_valid_counts.argtypes = geo + [P]
        lib.oracle_tile.argtypes = geo + [P, P, i, i, i]
        lib.oracle_untile.argtypes = geo + [P, P, i, i, i]
        lib.oracle_pool.argtypes = geo + [P, P, i, i, i, i]
        lib.oracle_half_to_f32.argtypes = [P, P, L, i]
        lib.oracle_score.argtypes = [P, P, P, i, i, i, i]
        lib.oracle_topk.argtypes = [P, i, i, i, i, P, P]
        lib.oracle_map_to_index.argtypes = [P, i, i, i, i, P, P]
        lib.oracle_topk_prefix.argtypes = [P, i, i, i, i, i, P, i, P, P]
        lib.oracle_attn_rows.argtypes = geo + [P, P, P, P, P, i, i, i, i, P, L, P, P, i]
        lib.oracle_compress.argtypes = [P, P, P, i, i, i, i, P]
        lib.oracle_gate_rows.argtypes = geo + [P, L, P, P, P, i, i, i, P, i]
        lib.oracle_attn_bwd_q_rows.argtypes = geo + [P, P, P, P, P, P, i, i, i, i, P, L, P, i]
        lib.oracle_attn_bwd_kv.argtypes = geo + [P, P, P, P, P, P, i, i, i, i, P, P, i]
        lib.oracle_quant_nvfp4.argtypes = [P, L, i, P, P, i]
        lib.oracle_dequant_nvfp4.argtypes = [P, P, L, i, P]
        lib.oracle_e4m3_round.argtypes = [P, L, P]
        lib.oracle_attn_rows_nvfp4.argtypes = geo + [P, P, P, P, P, P, P, i, i, P, L, P, P, i]
        lib.oracle_max_threads.argtypes = []
        for f in ("oracle_geometry", "oracle_block_valid_counts", "oracle_tile", "oracle_untile",
                  "oracle_pool", "oracle_score", "oracle_topk", "oracle_map_to_index",
                  "oracle_attn_rows", "oracle_max_threads", "oracle_half_to_f32", "oracle_compress",
                  "oracle_gate_rows", "oracle_attn_bwd_q_rows", "oracle_attn_bwd_kv", "oracle_quant_nvfp4",
                  "oracle_dequant_nvfp4", "oracle_e4m3_round", "oracle_attn_rows_nvfp4", "oracle_topk_prefix"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


@dataclass(frozen=True)
class Geometry:
    n_prefix: int
    T: int
    Hg: int
    Wg: int
    bt: int
    bh: int
    bw: int
    bs: int
    nT: int
    nH: int
    nW: int
    n_pre: int
    NB: int
    S: int
    Sp: int

    @property
    def args(self):
        return (self.n_prefix, self.T, self.Hg, self.Wg, self.bt, self.bh, self.bw)


def geometry(T, Hg, Wg, block=(4, 8, 8), n_prefix=0) -> Geometry:
    out = np.zeros(8, dtype=np.int64)
    _check(_load().oracle_geometry(n_prefix, T, Hg, Wg, *block, _ptr(out)), "geometry")
    bs, nT, nH, nW, n_pre, NB, S, Sp = (int(x) for x in out)
    return Geometry(n_prefix, T, Hg, Wg, *block, bs, nT, nH, nW, n_pre, NB, S, Sp)


def geometry_of(wl) -> Geometry:
    return geometry(wl.T, wl.Hg, wl.Wg, wl.block, wl.n_prefix)


def block_valid_counts(g: Geometry) -> np.ndarray:
    out = np.zeros(g.NB, dtype=np.int32)
    _check(_load().oracle_block_valid_counts(*g.args, _ptr(out)), "block_valid_counts")
    return out


def tile(g: Geometry, x: np.ndarray) -> np.ndarray:
    """x [B,S,H,D] bf16 bits -> [B,H,Sp,D] bf16 bits."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, S, H, D = x.shape
    assert S == g.S
    out = np.empty((B, H, g.Sp, D), dtype=np.uint16)
    _check(_load().oracle_tile(*g.args, _ptr(x), _ptr(out), B, H, D), "tile")
    return out


def untile(g: Geometry, xt: np.ndarray) -> np.ndarray:
    """xt [B,H,Sp,D] -> [B,S,H,D] (padded rows dropped). Works for any 2-byte dtype."""
    xt = np.ascontiguousarray(xt)
    assert xt.dtype.itemsize == 2
    B, H, Sp, D = xt.shape
    assert Sp == g.Sp
    src = xt.view(np.uint16)
    out = np.empty((B, g.S, H, D), dtype=np.uint16)
    _check(_load().oracle_untile(*g.args, _ptr(src), _ptr(out), B, H, D), "untile")
    return out.view(xt.dtype)


DTYPES = {"bf16": 0, "f16": 1}


def half_to_f32(x: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """16-bit patterns -> fp32 values (bf16 or IEEE fp16)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    out = np.empty(x.shape, dtype=np.float32)
    _check(_load().oracle_half_to_f32(_ptr(x), _ptr(out), x.size, DTYPES[dtype]), "half_to_f32")
    return out


def pool(g: Geometry, xt: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """Tiled xt [B,H,Sp,D] 16-bit patterns -> fp32 block means [B,H,NB,D]."""
    xt = np.ascontiguousarray(xt, dtype=np.uint16)
    B, H, Sp, D = xt.shape
    out = np.empty((B, H, g.NB, D), dtype=np.float32)
    _check(_load().oracle_pool(*g.args, _ptr(xt), _ptr(out), B, H, D, DTYPES[dtype]), "pool")
    return out


def score(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    qbar = np.ascontiguousarray(qbar, dtype=np.float32)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, H, NB, D = qbar.shape
    assert kbar.shape == qbar.shape
    out = np.empty((B, H, NB, NB), dtype=np.float32)
    _check(_load().oracle_score(_ptr(qbar), _ptr(kbar), _ptr(out), B, H, NB, D), "score")
    return out


def topk(s: np.ndarray, k: int):
    """Block scores [B,H,NB,NB] -> (q2k_idx [B,H,NB,k] ascending, q2k_num [B,H,NB])."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    B, H, NB, NB2 = s.shape
    assert NB == NB2
    idx = np.empty((B, H, NB, max(k, 1)), dtype=np.int32)
    num = np.empty((B, H, NB), dtype=np.int32)
    _check(_load().oracle_topk(_ptr(s), B, H, NB, k, _ptr(idx), _ptr(num)), "topk")
    return idx, num


def topk_prefix(s: np.ndarray, n_pre: int, k: int, row_keep=None, max_k: int | None = None):
    """Top-k with dense prefix tiles (tile-64 layout): prefix query tiles list
    every tile; a video query tile lists the n_pre prefix tiles and its k
    best-scoring video tiles (ties to the lower index), ascending; rows whose
    row_keep byte is 0 list nothing.  Returns (q2k_idx [B,H,NB,max_k] -1
    padded, q2k_num [B,H,NB]); max_k defaults to NB (k when n_pre == 0)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    B, H, NB, NB2 = s.shape
    assert NB == NB2
    if max_k is None:
        max_k = NB if n_pre > 0 else k
    keep = None if row_keep is None else np.ascontiguousarray(row_keep, dtype=np.uint8)
    if keep is not None:
        assert keep.shape == (B, H, NB)
    idx = np.empty((B, H, NB, max_k), dtype=np.int32)
    num = np.empty((B, H, NB), dtype=np.int32)
    _check(_load().oracle_topk_prefix(_ptr(s), B, H, NB, n_pre, k, None if keep is None else _ptr(keep), max_k,
                                      _ptr(idx), _ptr(num)), "topk_prefix")
    return idx, num


def map_to_index(m: np.ndarray):
    """Bool map [B,H,NQ,NK] -> (q2k_idx [B,H,NQ,NK] ascending, -1 padded; q2k_num)."""
    m = np.ascontiguousarray(m, dtype=np.uint8)
    B, H, NQ, NK = m.shape
    idx = np.empty((B, H, NQ, NK), dtype=np.int32)
    num = np.empty((B, H, NQ), dtype=np.int32)
    _check(_load().oracle_map_to_index(_ptr(m), B, H, NQ, NK, _ptr(idx), _ptr(num)), "map_to_index")
    return idx, num


def attn_rows(g: Geometry, qt, kt, vt, idx, num, rows, dtype: str = "bf16"):
    """fp64 attention for flat rows of [B,H,Sp]; returns (o [n,D] f64, lse [n] f64)."""
    qt = np.ascontiguousarray(qt, dtype=np.uint16)
    kt = np.ascontiguousarray(kt, dtype=np.uint16)
    vt = np.ascontiguousarray(vt, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    num = np.ascontiguousarray(num, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    B, H, Sp, D = qt.shape
    max_k = idx.shape[-1]
    o = np.empty((len(rows), D), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    _check(_load().oracle_attn_rows(*g.args, _ptr(qt), _ptr(kt), _ptr(vt), _ptr(idx), _ptr(num),
                                    max_k, B, H, D, _ptr(rows), len(rows), _ptr(o), _ptr(lse), DTYPES[dtype]),
           "attn_rows")
    return o, lse


def attn(g: Geometry, qt, kt, vt, idx, num, dtype: str = "bf16"):
    """fp64 attention over every row: (o [B,H,Sp,D], lse [B,H,Sp])."""
    B, H, Sp, D = qt.shape
    rows = np.arange(B * H * Sp, dtype=np.int64)
    o, lse = attn_rows(g, qt, kt, vt, idx, num, rows, dtype)
    return o.reshape(B, H, Sp, D), lse.reshape(B, H, Sp)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def coarse(g: Geometry, qt, kt, k: int, dtype: str = "bf16"):
    """pool -> score -> top-k, the whole coarse stage on tiled Q and K."""
    qbar = pool(g, qt, dtype)
    kbar = pool(g, kt, dtype)
    return topk(score(qbar, kbar), k), (qbar, kbar)


def compress(qbar: np.ndarray, kbar: np.ndarray, vbar: np.ndarray) -> np.ndarray:
    """Compression branch: fp64 attention among block means, [B,H,NB,D] each -> [B,H,NB,D] f64."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float32)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    vbar = np.ascontiguousarray(vbar, dtype=np.float32)
    B, H, NB, D = qbar.shape
    assert kbar.shape == qbar.shape and vbar.shape == qbar.shape
    out = np.empty((B, H, NB, D), dtype=np.float64)
    _check(_load().oracle_compress(_ptr(qbar), _ptr(kbar), _ptr(vbar), B, H, NB, D, _ptr(out)), "compress")
    return out


def gate_rows(g: Geometry, rows, o_fine, gate, o_compress, dtype: str = "bf16") -> np.ndarray:
    """o_fine [n,D] + gate (untiled [B,S,H,D] 16-bit) * o_compress of each row's block; f64 [n,D]."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    o_fine = np.ascontiguousarray(o_fine, dtype=np.float64)
    gate = np.ascontiguousarray(gate, dtype=np.uint16)
    o_compress = np.ascontiguousarray(o_compress, dtype=np.float64)
    B, S, H, D = gate.shape
    assert S == g.S and o_fine.shape == (len(rows), D)
    out = np.empty((len(rows), D), dtype=np.float64)
    _check(_load().oracle_gate_rows(*g.args, _ptr(rows), len(rows), _ptr(o_fine), _ptr(gate), _ptr(o_compress),
                                    B, H, D, _ptr(out), DTYPES[dtype]), "gate_rows")
    return out


def attn_bwd_q_rows(g: Geometry, qt, kt, vt, dot, idx, num, rows, dtype: str = "bf16") -> np.ndarray:
    """dq (fp64 [n, D]) of flat query rows of [B,H,Sp]; padded rows give 0."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (qt, kt, vt, dot)]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    num = np.ascontiguousarray(num, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    B, H, Sp, D = arrs[0].shape
    out = np.empty((len(rows), D), dtype=np.float64)
    _check(_load().oracle_attn_bwd_q_rows(*g.args, *[_ptr(a) for a in arrs], _ptr(idx), _ptr(num), idx.shape[-1],
                                          B, H, D, _ptr(rows), len(rows), _ptr(out), DTYPES[dtype]), "attn_bwd_q_rows")
    return out


def attn_bwd_kv(g: Geometry, qt, kt, vt, dot, idx, num, dtype: str = "bf16"):
    """(dk, dv) fp64 [B,H,Sp,D] over all key rows (small problems only)."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (qt, kt, vt, dot)]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    num = np.ascontiguousarray(num, dtype=np.int32)
    B, H, Sp, D = arrs[0].shape
    dk = np.empty((B, H, Sp, D), dtype=np.float64)
    dv = np.empty((B, H, Sp, D), dtype=np.float64)
    _check(_load().oracle_attn_bwd_kv(*g.args, *[_ptr(a) for a in arrs], _ptr(idx), _ptr(num), idx.shape[-1],
                                      B, H, D, _ptr(dk), _ptr(dv), DTYPES[dtype]), "attn_bwd_kv")
    return dk, dv


def slot_valid(g: Geometry) -> np.ndarray:
    """[Sp] bool: which tiled slots hold a real token (the tile of an all-ones grid)."""
    ones = np.full((1, g.S, 1, 8), 0x3F80, dtype=np.uint16)  # bf16 1.0
    return tile(g, ones)[0, 0, :, 0] != 0


def attn_bwd_kv_blocks(g: Geometry, qt, kt, vt, dot, idx, num, blocks, dtype: str = "bf16"):
    """(dk, dv) fp64 [n, bs, D] of chosen key blocks (flat ids b*H*NB + h*NB + kb).

    The definition of the key-side gradients (C file header, "backward"),
    written with fp64 matrix products so that full-size problems finish: for
    every query block r of the head whose list names a chosen block, over the
    real query rows i of r and the real key slots j of r's listed blocks in
    list order (a repeated id appears, and counts, twice):
      P = softmax_j(scale q_i . k_j),  dP_ij = do_i . v_j,
      dS = P (dP - rowsum(P dP)),
    then dv_j += sum_i P_ij do_i and dk_j += scale sum_i dS_ij q_i for the
    slots j of each chosen block.  Padded slots get 0."""
    qt, kt, vt, dot = (np.ascontiguousarray(a, dtype=np.uint16) for a in (qt, kt, vt, dot))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    num = np.ascontiguousarray(num, dtype=np.int32)
    blocks = np.ascontiguousarray(blocks, dtype=np.int64)
    B, H, Sp, D = qt.shape
    NB, bs = g.NB, g.bs
    if ((blocks < 0) | (blocks >= B * H * NB)).any():
        raise ValueError("oracle attn_bwd_kv_blocks: block id out of range")
    max_k = idx.shape[-1]
    scale = 1.0 / np.sqrt(D)
    valid = slot_valid(g)
    dk = np.zeros((len(blocks), bs, D))
    dv = np.zeros((len(blocks), bs, D))
    wanted = {}
    for n, fb in enumerate(blocks.tolist()):
        wanted.setdefault(fb // NB, []).append((n, fb % NB))
    for bhh, reqs in wanted.items():
        b, h = divmod(bhh, H)
        Q, K, V, dO = (half_to_f32(a[b, h], dtype).astype(np.float64) for a in (qt, kt, vt, dot))
        for r in range(NB):
            cnt = int(num[b, h, r])
            if cnt < 0 or cnt > max_k:
                raise ValueError("oracle attn_bwd_kv_blocks: count out of range")
            ids = idx[b, h, r, :cnt]
            if ((ids < 0) | (ids >= NB)).any():
                raise ValueError("oracle attn_bwd_kv_blocks: block id out of range")
            hits = [(n, kb) for n, kb in reqs if (ids == kb).any()]
            if not hits:
                continue
            rows = np.arange(r * bs, (r + 1) * bs)[valid[r * bs:(r + 1) * bs]]
            keys = np.concatenate([np.arange(kb * bs, (kb + 1) * bs) for kb in ids.tolist()])
            keys = keys[valid[keys]]
            s = (Q[rows] @ K[keys].T) * scale
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dp = dO[rows] @ V[keys].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            for n, kb in hits:
                cols = np.flatnonzero(keys // bs == kb)
                slots = keys[cols] - kb * bs
                np.add.at(dv[n], slots, p[:, cols].T @ dO[rows])
                np.add.at(dk[n], slots, scale * (ds[:, cols].T @ Q[rows]))
    return dk, dv


def quant_nvfp4(x: np.ndarray, dtype: str = "bf16"):
    """16-bit rows [..., D] -> (codes [..., D/2] uint8, scales [..., D/16] uint8 E4M3)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.empty(x.shape[:-1] + (D // 2,), dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (D // 16,), dtype=np.uint8)
    _check(_load().oracle_quant_nvfp4(_ptr(x), rows, D, _ptr(codes), _ptr(sf), DTYPES[dtype]), "quant_nvfp4")
    return codes, sf


def dequant_nvfp4(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """The values NVFP4 codes and scales stand for, fp64 [..., D]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    D = codes.shape[-1] * 2
    rows = codes.size // (D // 2)
    y = np.empty(codes.shape[:-1] + (D,), dtype=np.float64)
    _check(_load().oracle_dequant_nvfp4(_ptr(codes), _ptr(sf), rows, D, _ptr(y)), "dequant_nvfp4")
    return y


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """E4M3 bits of non-negative fp32 values (nearest, ties to even, capped at 448)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = np.empty(x.shape, dtype=np.uint8)
    _check(_load().oracle_e4m3_round(_ptr(x), x.size, _ptr(bits)), "e4m3_round")
    return bits


def attn_rows_nvfp4(g: Geometry, qc, qs, kc, ks, vt, idx, num, rows, dtype: str = "bf16"):
    """fp64 attention of flat rows of [B,H,Sp] with NVFP4 q, k (row-major codes/scales) and 16-bit v."""
    qc, kc = (np.ascontiguousarray(a, dtype=np.uint8) for a in (qc, kc))
    qs, ks = (np.ascontiguousarray(a, dtype=np.uint8) for a in (qs, ks))
    vt = np.ascontiguousarray(vt, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    num = np.ascontiguousarray(num, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    D = vt.shape[-1]
    o = np.empty((len(rows), D), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    _check(_load().oracle_attn_rows_nvfp4(*g.args, _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), _ptr(vt), _ptr(idx),
                                          _ptr(num), idx.shape[-1], D, _ptr(rows), len(rows), _ptr(o), _ptr(lse),
                                          DTYPES[dtype]), "attn_rows_nvfp4")
    return o, lse
