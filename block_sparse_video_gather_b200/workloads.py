"""Seeded synthetic workloads for the Video Sparse Attention forward path.

This module only draws random numbers and lays them out in the untiled
``[B, S, H, D]`` token layout of a video DiT.  It computes nothing of the
attention method: no tiling, pooling, scoring, selection or softmax.  The
CPU oracle and the CUDA library are both fed from here, and from nowhere else.

Workload shapes follow the latent grids named on the pages:

* "FastVideo VSA" (vLLM-Omni user guide), section "Choose top-k": the
  FastWan2.2-TI2V-5B grid (31, 22, 40), block (4, 8, 8), top-k 64.
* The Wan2.1-1.3B grids at 81 and 321 frames (latent T = 21 and 81 at
  30 x 52) from the LVSA long-video pages' horizon sweeps.
* The FastVideo commit log (examples/inference/basic/README.md): a tile-64
  layout with dense prefix query tiles, video query tiles that see the
  prefix plus a top-k of video tiles, and rows whose count is zero.

Recipe (stated once, used by every test and by the benchmark):

* noise: Q, K, V are i.i.d. N(0, 1) in fp32, drawn from child streams of
  ``numpy.random.SeedSequence(seed)``, one stream per fixed 2**20-element
  chunk, so the values do not depend on how many threads draw them;
* per-block offsets: one D-vector per (tensor, b, h, video block) drawn
  N(0, offset_std**2) and added to every token of that block; with
  ``offset_ar > 0`` the offsets follow an AR(1) chain along the temporal
  block index, ``o[t] = a o[t-1] + sqrt(1 - a^2) e[t]``, which keeps the
  marginal N(0, offset_std**2);
* the fp32 values are rounded to bf16 (or, on request, IEEE fp16) with
  round-to-nearest-even and kept as their raw 16-bit patterns (numpy has no
  bf16 dtype);
* gate (only when asked for): i.i.d. N(0, 1) in the untiled [B, S, H, D]
  layout, rounded the same way -- a stand-in for the output of a learned
  gate_compress projection ("FastVideo VSA", section "Checkpoint behavior");
* forced-empty rows (``zero_row_frac > 0``): ``round(zero_row_frac * B * H *
  NB)`` query rows, chosen uniformly at random, select nothing.  With a
  computed selection (``prefix_dense``) they arrive as a row-keep byte mask
  [B, H, NB] (0 = forced empty); with a block map, as cleared map rows;
* block maps (map-driven workloads only): prefix query tiles select every
  tile; a video query tile selects every prefix tile plus ``map_video_k``
  distinct video tiles chosen uniformly at random; then the forced-empty
  rows are cleared.

Selections: ``topk`` set and ``prefix_dense`` False -- the coarse stage's
plain top-k over all blocks; ``prefix_dense`` -- prefix query tiles select
every tile and a video query tile selects the prefix tiles plus its top-k
video tiles, both computed by the coarse stage from the pooled scores;
``topk`` None -- a caller-supplied bool block map.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_CHUNK = 1 << 20


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    T: int
    Hg: int
    Wg: int
    block: tuple  # (bt, bh, bw) tokens per block along (T, H, W)
    topk: int | None = None  # coarse-stage top-k; None for map-driven workloads
    n_prefix: int = 0  # tokens placed before the video grid, tiled contiguously
    prefix_dense: bool = False  # prefix query tiles select all; video query tiles the prefix + top-k video tiles
    offset_std: float = 0.5
    offset_ar: float = 0.0
    map_video_k: int = 0
    zero_row_frac: float = 0.0
    seed: int = 0

    # ---- shape bookkeeping (ceil divisions of the grid; no method arithmetic)
    @property
    def block_tokens(self) -> int:
        bt, bh, bw = self.block
        return bt * bh * bw

    @property
    def grid_blocks(self) -> tuple:
        bt, bh, bw = self.block
        return (-(-self.T // bt), -(-self.Hg // bh), -(-self.Wg // bw))

    @property
    def n_prefix_blocks(self) -> int:
        return -(-self.n_prefix // self.block_tokens)

    @property
    def num_blocks(self) -> int:
        nT, nH, nW = self.grid_blocks
        return self.n_prefix_blocks + nT * nH * nW

    @property
    def seq_len(self) -> int:
        return self.n_prefix + self.T * self.Hg * self.Wg

    @property
    def padded_len(self) -> int:
        return self.num_blocks * self.block_tokens

    @property
    def map_driven(self) -> bool:
        return self.topk is None

    @property
    def max_k(self) -> int:
        """Row stride of q2k_idx: the longest possible row."""
        if self.map_driven or self.prefix_dense:
            return self.num_blocks
        return self.topk


WORKLOADS = {
    # B=1, H=2, grid (8,16,16) = 2048 tokens, 8 blocks, top-k 4.
    "tiny": Workload("tiny", B=1, H=2, D=128, T=8, Hg=16, Wg=16, block=(4, 8, 8), topk=4),
    # FastWan2.2-TI2V-5B: (31,22,40) = 27280 tokens -> 120 blocks, top-k 64.
    "fastwan": Workload("fastwan", B=1, H=24, D=128, T=31, Hg=22, Wg=40, block=(4, 8, 8), topk=64),
    # Wan2.1-1.3B, 81 frames: (21,30,52) = 32760 tokens -> 168 blocks, top-k 32.
    "wan81": Workload("wan81", B=1, H=12, D=128, T=21, Hg=30, Wg=52, block=(4, 8, 8), topk=32),
    # Tile-64, non-uniform rows: 512 prefix tokens + (16,32,32) video, 264 tiles;
    # prefix query tiles dense, video query tiles the prefix + their top-32 video
    # tiles (computed), 5% of rows forced empty.
    "tile64": Workload("tile64", B=1, H=24, D=128, T=16, Hg=32, Wg=32, block=(4, 4, 4),
                       topk=32, n_prefix=512, prefix_dense=True, offset_std=0.0,
                       zero_row_frac=0.05),
    # The same layout with the selection as a caller-supplied bool block map
    # (32 random video tiles per video row) compacted by map_to_index.
    "tile64map": Workload("tile64map", B=1, H=24, D=128, T=16, Hg=32, Wg=32, block=(4, 4, 4),
                          topk=None, n_prefix=512, offset_std=0.0, map_video_k=32,
                          zero_row_frac=0.05),
    # Wan2.1-1.3B, 321 frames (4x horizon): (81,30,52) = 126360 tokens -> 588 blocks.
    "long": Workload("long", B=1, H=12, D=128, T=81, Hg=30, Wg=52, block=(4, 8, 8), topk=59,
                     offset_ar=0.9),
}


def custom(name="custom", **kw) -> Workload:
    """A workload of any shape with the same recipe (used for edge cases)."""
    base = dict(B=1, H=1, D=128, T=4, Hg=8, Wg=8, block=(4, 8, 8), topk=1)
    base.update(kw)
    return Workload(name, **base)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); return the bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_fill(seq: np.random.SeedSequence, n: int, threads: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nchunk = -(-n // _CHUNK)
    kids = seq.spawn(nchunk)

    def fill(i):
        lo = i * _CHUNK
        hi = min(n, lo + _CHUNK)
        np.random.default_rng(kids[i]).standard_normal(out=out[lo:hi], dtype=np.float32)

    if threads > 1 and nchunk > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nchunk)))
    else:
        for i in range(nchunk):
            fill(i)
    return out


def _block_offsets(wl: Workload, seq: np.random.SeedSequence) -> np.ndarray:
    """[B, H, nT, nH, nW, D] fp32 offsets (AR(1) along nT when offset_ar > 0)."""
    nT, nH, nW = wl.grid_blocks
    rng = np.random.default_rng(seq)
    e = rng.standard_normal((wl.B, wl.H, nT, nH, nW, wl.D), dtype=np.float32) * np.float32(wl.offset_std)
    if wl.offset_ar > 0.0:
        a = np.float32(wl.offset_ar)
        c = np.float32(math.sqrt(1.0 - wl.offset_ar * wl.offset_ar))
        for t in range(1, nT):
            e[:, :, t] = a * e[:, :, t - 1] + c * e[:, :, t]
    return e


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to IEEE fp16 (nearest even); return the bit patterns."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def _tensor(wl: Workload, noise_seq, off_seq, threads: int, dtype: str = "bf16") -> np.ndarray:
    B, S, H, D = wl.B, wl.seq_len, wl.H, wl.D
    x = _normal_fill(noise_seq, B * S * H * D, threads).reshape(B, S, H, D)
    if wl.offset_std > 0.0:
        off = _block_offsets(wl, off_seq)
        bt, bh, bw = wl.block
        ti = np.arange(wl.T) // bt
        yi = np.arange(wl.Hg) // bh
        xi = np.arange(wl.Wg) // bw
        for b in range(B):
            # x[b, n_prefix:] is contiguous, so this reshape is a view of x
            video = x[b, wl.n_prefix:].reshape(wl.T, wl.Hg, wl.Wg, H, D)
            assert np.shares_memory(video, x)
            # [H, T, Hg, Wg, D] -> [T, Hg, Wg, H, D], one b at a time to bound memory
            ob = off[b][:, ti][:, :, yi][:, :, :, xi]
            video += np.transpose(ob, (1, 2, 3, 0, 4))
    return f32_to_f16_bits(x) if dtype == "f16" else f32_to_bf16_bits(x)


def _block_map(wl: Workload, seq: np.random.SeedSequence) -> np.ndarray:
    NB = wl.num_blocks
    npre = wl.n_prefix_blocks
    nvid = NB - npre
    rng = np.random.default_rng(seq)
    m = np.zeros((wl.B, wl.H, NB, NB), dtype=np.bool_)
    m[:, :, :npre, :] = True
    m[:, :, npre:, :npre] = True
    k = min(wl.map_video_k, nvid)
    if k > 0:
        keys = rng.random((wl.B, wl.H, nvid, nvid))
        pick = np.argsort(keys, axis=-1, kind="stable")[..., :k] + npre
        bb, hh, rr = np.meshgrid(np.arange(wl.B), np.arange(wl.H), np.arange(npre, NB), indexing="ij")
        m[bb[..., None], hh[..., None], rr[..., None], pick] = True
    nzero = int(round(wl.zero_row_frac * wl.B * wl.H * NB))
    if nzero > 0:
        rows = rng.permutation(wl.B * wl.H * NB)[:nzero]
        m.reshape(wl.B * wl.H * NB, NB)[rows] = False
    return m


def _row_keep(wl: Workload, seq: np.random.SeedSequence) -> np.ndarray:
    """[B, H, NB] uint8: 0 for the forced-empty rows, 1 elsewhere."""
    n = wl.B * wl.H * wl.num_blocks
    keep = np.ones(n, dtype=np.uint8)
    nzero = int(round(wl.zero_row_frac * n))
    if nzero > 0:
        keep[np.random.default_rng(seq).permutation(n)[:nzero]] = 0
    return keep.reshape(wl.B, wl.H, wl.num_blocks)


def make_inputs(wl: Workload | str, threads: int = 8, dtype: str = "bf16", gate: bool = False) -> dict:
    """Q, K, V as bf16 (or fp16) bit patterns [B, S, H, D] (uint16), for
    map-driven workloads the bool block map [B, H, NB, NB], for workloads
    with forced-empty rows and a computed selection the row-keep mask
    [B, H, NB] uint8 ("row_keep", else None), and on request the gate
    [B, S, H, D] (same format)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    root = np.random.SeedSequence(wl.seed)
    # children are numbered: the eighth (gate) leaves the first seven unchanged
    nq, nk, nv, oq, ok, ov, mp, ng = root.spawn(8)
    out = {
        "q": _tensor(wl, nq, oq, threads, dtype),
        "k": _tensor(wl, nk, ok, threads, dtype),
        "v": _tensor(wl, nv, ov, threads, dtype),
        "map": _block_map(wl, mp) if wl.map_driven else None,
        "row_keep": _row_keep(wl, mp) if (not wl.map_driven and wl.zero_row_frac > 0) else None,
    }
    if gate:
        g = _normal_fill(ng, wl.B * wl.seq_len * wl.H * wl.D, threads).reshape(wl.B, wl.seq_len, wl.H, wl.D)
        out["gate"] = f32_to_f16_bits(g) if dtype == "f16" else f32_to_bf16_bits(g)
    return out
