"""Shared helpers of the GPU parity tests: host<->device moves of bf16 bit patterns,
cached seeded workloads and their oracle results, and the error metrics the
tolerances are written against."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import valid_slots_by_reshape

# Tolerances for the bf16 attention output against the fp64 oracle, and for lse.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev(t: torch.Tensor) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(bits: np.ndarray) -> np.ndarray:
    return workloads.bf16_bits_to_f32(bits)


@functools.lru_cache(maxsize=4)
def inputs(wl: workloads.Workload):
    return workloads.make_inputs(wl)


@functools.lru_cache(maxsize=4)
def oracle_front(wl: workloads.Workload):
    """Oracle tile of q, k, v and the coarse stage (plain or tile-64 rule) or the map compaction."""
    g = oracle.geometry_of(wl)
    inp = inputs(wl)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    qbar, kbar = oracle.pool(g, qt), oracle.pool(g, kt)
    if wl.map_driven:
        idx, num = oracle.map_to_index(inp["map"])
    elif wl.prefix_dense:
        idx, num = oracle.topk_prefix(oracle.score(qbar, kbar), g.n_pre, wl.topk, inp["row_keep"], wl.max_k)
    else:
        idx, num = oracle.topk(oracle.score(qbar, kbar), wl.topk)
    return dict(g=g, qt=qt, kt=kt, vt=vt, qbar=qbar, kbar=kbar, idx=idx, num=num)


def real_rows(wl) -> np.ndarray:
    """[Sp] bool: tiled rows that hold a real token (reshape form, independent of both sides)."""
    return valid_slots_by_reshape(wl.T, wl.Hg, wl.Wg, wl.block, wl.n_prefix)


def compare_o_lse(o_gpu_bits, lse_gpu, o_ref, lse_ref, what=""):
    """o_gpu_bits [...,D] bf16 bits vs o_ref [...,D] fp64; lse vs lse_ref."""
    o = f32(o_gpu_bits).astype(np.float64)
    err = np.abs(o - o_ref)
    max_abs, mean_abs = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert max_abs <= O_MAX_ABS, f"{what}: o max-abs {max_abs:.3e}"
    assert mean_abs <= O_MEAN_ABS, f"{what}: o mean-abs {mean_abs:.3e}"
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    inf_ref = np.isneginf(lse_ref)
    np.testing.assert_array_equal(np.isneginf(lse_gpu), inf_ref, err_msg=f"{what}: lse -inf pattern")
    fin = ~inf_ref
    lerr = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max(initial=0.0))
    assert lerr <= LSE_ABS, f"{what}: lse max-abs {lerr:.3e}"
    return max_abs, mean_abs, lerr
