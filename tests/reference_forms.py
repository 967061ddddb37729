"""Independent restatements used to pin the oracle (tests only).

Each function states a step of the method in a different form from the
oracle's index arithmetic: whole-array reshapes and transposes for the block
partition ("FastVideo VSA", vLLM-Omni user guide, introduction and section
"Choose top-k"), and an explicit token-by-token mask with a dense softmax for
the attention of a query block against its selected blocks (same page,
introduction and section "Verify routing and fallback").  They are small and
slow by design.
"""
from __future__ import annotations

import numpy as np


def tile_by_reshape(x: np.ndarray, T, Hg, Wg, block, n_prefix=0) -> np.ndarray:
    """[B,S,H,D] -> [B,H,Sp,D]: zero-pad the grid, cut it into blocks, flatten."""
    bt, bh, bw = block
    bs = bt * bh * bw
    B, S, H, D = x.shape
    npre = -(-n_prefix // bs)
    pre = np.zeros((B, npre * bs, H, D), dtype=x.dtype)
    pre[:, :n_prefix] = x[:, :n_prefix]
    nT, nH, nW = -(-T // bt), -(-Hg // bh), -(-Wg // bw)
    vid = np.zeros((B, nT * bt, nH * bh, nW * bw, H, D), dtype=x.dtype)
    vid[:, :T, :Hg, :Wg] = x[:, n_prefix:].reshape(B, T, Hg, Wg, H, D)
    vid = vid.reshape(B, nT, bt, nH, bh, nW, bw, H, D)
    vid = vid.transpose(0, 7, 1, 3, 5, 2, 4, 6, 8).reshape(B, H, nT * nH * nW * bs, D)
    return np.concatenate([pre.transpose(0, 2, 1, 3), vid], axis=2)


def valid_slots_by_reshape(T, Hg, Wg, block, n_prefix=0) -> np.ndarray:
    """[Sp] bool: which tiled slots hold a real token."""
    ones = np.ones((1, n_prefix + T * Hg * Wg, 1, 1), dtype=np.uint8)
    return tile_by_reshape(ones, T, Hg, Wg, block, n_prefix)[0, 0, :, 0].astype(bool)


def dense_masked_attention(q, k, v, allowed):
    """fp64 softmax attention with an explicit [Sq, Sk] boolean mask.

    q [Sq,D], k [Sk,D], v [Sk,D] float64.  Rows with no allowed key give
    o = 0 and lse = -inf.
    """
    D = q.shape[1]
    logits = (q @ k.T) / np.sqrt(D)
    logits = np.where(allowed, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    empty = ~allowed.any(axis=1)
    m[empty] = 0.0
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (p @ v) / l
        lse = (m + np.log(l))[:, 0]
    o[empty] = 0.0
    lse[empty] = -np.inf
    return o, lse


def block_mask(idx, num, NB, bs, valid):
    """[Sp, Sp] mask of one head: query slot i may see key slot j iff the block
    of j is listed for the block of i and j holds a real token."""
    Sp = NB * bs
    allowed = np.zeros((Sp, Sp), dtype=bool)
    for r in range(NB):
        for t in range(int(num[r])):
            kb = int(idx[r, t])
            allowed[r * bs:(r + 1) * bs, kb * bs:(kb + 1) * bs] = True
    return allowed & valid[None, :]
