"""Pins of the oracle's backward pass (gradients of the attention step with the
selection held fixed).

The attention step is "FastVideo VSA" (vLLM-Omni user guide), introduction
and section "Verify routing and fallback"; the FastVideo commit log keeps the
grad path on its own kernels and prints no formula, so the reference here is
the derivative itself: torch autograd in fp64 through a dense softmax with an
explicit block mask, finite differences, and the identities every softmax
attention gradient satisfies.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_video_gather_b200 import workloads
from tests.reference_forms import block_mask, valid_slots_by_reshape

f32 = workloads.bf16_bits_to_f32


def _problem(T, Hg, Wg, block=(4, 8, 8), npre=0, H=2, D=64, k=3, seed=0, zero_rows=True):
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, H=H, D=D, seed=seed)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, threads=1)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(seed + 100)
    do = oracle.tile(g, workloads.f32_to_bf16_bits(rng.standard_normal(inp["q"].shape).astype(np.float32)))
    k = min(k, g.NB)
    num = rng.integers(0 if zero_rows else 1, k + 1, size=(1, H, g.NB)).astype(np.int32)
    idx = np.full((1, H, g.NB, k), -1, dtype=np.int32)
    for pos in np.ndindex(1, H, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    valid = valid_slots_by_reshape(T, Hg, Wg, block, npre)
    return g, qt, kt, vt, do, idx, num, valid


def _autograd(qt, kt, vt, do, idx, num, g, valid, h):
    """Dense fp64 softmax attention with the block mask; loss = sum(o * do) over real query rows."""
    q = torch.tensor(f32(qt[0, h]), dtype=torch.float64, requires_grad=True)
    k = torch.tensor(f32(kt[0, h]), dtype=torch.float64, requires_grad=True)
    v = torch.tensor(f32(vt[0, h]), dtype=torch.float64, requires_grad=True)
    allowed = torch.from_numpy(block_mask(idx[0, h], num[0, h], g.NB, g.bs, valid))
    logits = (q @ k.T) / np.sqrt(q.shape[1])
    logits = logits.masked_fill(~allowed, float("-inf"))
    has = allowed.any(dim=1)
    p = torch.softmax(logits.masked_fill(~has[:, None], 0.0), dim=1) * has[:, None]
    o = p @ v
    rows = torch.from_numpy(valid) & has
    loss = (o[rows] * torch.tensor(f32(do[0, h]), dtype=torch.float64)[rows]).sum()
    loss.backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("shape", [((5, 9, 11), (4, 8, 8), 0), ((6, 8, 12), (4, 4, 4), 100)])
def test_matches_autograd_through_dense_masked_softmax(shape):
    (T, Hg, Wg), block, npre = shape
    g, qt, kt, vt, do, idx, num, valid = _problem(T, Hg, Wg, block, npre)
    dk, dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    rows = np.arange(2 * g.Sp, dtype=np.int64)
    dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows).reshape(1, 2, g.Sp, -1)
    for h in range(2):
        rq, rk, rv = _autograd(qt, kt, vt, do, idx, num, g, valid, h)
        np.testing.assert_allclose(dq[0, h], rq, rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk[0, h], rk, rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[0, h], rv, rtol=0, atol=1e-11)


def test_finite_differences_of_the_oracle_forward():
    """d/dt of sum(o(q + t e) * do) at t = 0 equals <dq, e>, with o from the
    forward oracle (central differences in fp64 on bf16-exact inputs)."""
    g, qt, kt, vt, do, idx, num, valid = _problem(4, 8, 8, H=1, D=16, k=1, zero_rows=False)
    rows = np.flatnonzero(valid).astype(np.int64)
    dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows)
    # the forward oracle reads 16-bit inputs; move q along an exactly representable
    # direction: one channel of one row, by +-2^-7 around a value with room for it
    r, c = int(rows[5]), 3
    base = qt.copy()
    base[0, 0, r, c] = workloads.f32_to_bf16_bits(np.array([0.5], np.float32))[0]
    f = []
    for step in (+1, -1):
        x = base.copy()
        x[0, 0, r, c] = workloads.f32_to_bf16_bits(np.array([0.5 + step * 2.0 ** -7], np.float32))[0]
        o, _ = oracle.attn_rows(g, x, kt, vt, idx, num, rows)
        f.append((o * f32(do[0, 0, rows])).sum())
    fd = (f[0] - f[1]) / (2 * 2.0 ** -7)
    dq_b = oracle.attn_bwd_q_rows(g, base, kt, vt, do, idx, num, rows)
    assert abs(fd - dq_b[5, c]) <= 1e-4 * max(1.0, abs(fd))
    assert np.isfinite(dq).all()


def test_gradient_identities():
    """sum_j dk_j = 0 (each row's dS sums to zero) and sum_j dv_j = sum of do over
    the real rows with a non-empty selection."""
    g, qt, kt, vt, do, idx, num, valid = _problem(5, 9, 11, H=2, D=32, k=4)
    dk, dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    for h in range(2):
        np.testing.assert_allclose(dk[0, h].sum(axis=0), 0.0, atol=1e-10)
        rows = valid & (np.repeat(num[0, h], g.bs) > 0)
        np.testing.assert_allclose(dv[0, h].sum(axis=0), f32(do[0, h][rows]).astype(np.float64).sum(axis=0),
                                   atol=1e-10)


def test_padded_rows_and_empty_rows_get_nothing():
    g, qt, kt, vt, do, idx, num, valid = _problem(5, 9, 11, H=1, D=32, k=3)
    dk, dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    assert (dk[0, 0][~valid] == 0).all() and (dv[0, 0][~valid] == 0).all()
    rows = np.arange(g.Sp, dtype=np.int64)
    dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, rows)
    assert (dq[~valid] == 0).all()
    empty = np.repeat(num[0, 0] == 0, g.bs)
    assert empty.any() and (dq[empty] == 0).all()


def test_single_key_row():
    """One real token in the whole grid: its row sees one key, P = 1, so dq = 0,
    dk = 0 and dv of that key is the row's do."""
    wl = workloads.custom(T=1, Hg=1, Wg=1, H=1, D=32)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, threads=1)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    do = oracle.tile(g, inp["k"])  # any 16-bit values
    idx = np.zeros((1, 1, 1, 1), np.int32)
    num = np.ones((1, 1, 1), np.int32)
    dq = oracle.attn_bwd_q_rows(g, qt, kt, vt, do, idx, num, np.array([0], np.int64))
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    dk, dv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    assert np.array_equal(dv[0, 0, 0], f32(do[0, 0, 0]).astype(np.float64))
    assert (dv[0, 0, 1:] == 0).all()


def _autograd_gather(qt, kt, vt, do, idx, num, g, valid, h):
    """The same gradients by a second form: per query block, gather the key and
    value rows of its listed blocks in list order (a repeated id appears
    twice), mask padded keys, softmax, o = P V; torch autograd accumulates the
    gradient of every gathered copy back onto its row."""
    q = torch.tensor(f32(qt[0, h]), dtype=torch.float64, requires_grad=True)
    k = torch.tensor(f32(kt[0, h]), dtype=torch.float64, requires_grad=True)
    v = torch.tensor(f32(vt[0, h]), dtype=torch.float64, requires_grad=True)
    dot = torch.tensor(f32(do[0, h]), dtype=torch.float64)
    bs, D = g.bs, q.shape[1]
    loss = torch.zeros((), dtype=torch.float64)
    for r in range(g.NB):
        ids = [int(x) for x in idx[0, h, r, :num[0, h, r]]]
        if not ids:
            continue
        keys = torch.tensor(np.concatenate([np.arange(b * bs, (b + 1) * bs) for b in ids]))
        real_k = torch.from_numpy(valid[keys.numpy()])
        rows = torch.arange(r * bs, (r + 1) * bs)
        real_q = torch.from_numpy(valid[rows.numpy()])
        logits = (q[rows] @ k[keys].T) / np.sqrt(D)
        p = torch.softmax(logits.masked_fill(~real_k[None, :], float("-inf")), dim=1)
        o = p @ v[keys]
        loss = loss + (o[real_q] * dot[rows][real_q]).sum()
    loss.backward()
    return k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("shape", [((5, 9, 11), (4, 8, 8), 0), ((6, 8, 12), (4, 4, 4), 100)])
def test_kv_blocks_match_autograd(shape):
    """dk, dv of chosen key blocks (full-size checks use this form) equal the
    fp64 autograd gradients, partial blocks and prefix tiles included."""
    (T, Hg, Wg), block, npre = shape
    g, qt, kt, vt, do, idx, num, valid = _problem(T, Hg, Wg, block, npre)
    H = 2
    blocks = np.array([h * g.NB + kb for h in range(H) for kb in range(g.NB)], dtype=np.int64)
    dk, dv = oracle.attn_bwd_kv_blocks(g, qt, kt, vt, do, idx, num, blocks)
    for h in range(H):
        _, rk, rv = _autograd(qt, kt, vt, do, idx, num, g, valid, h)
        got_k = dk[h * g.NB:(h + 1) * g.NB].reshape(g.Sp, -1)
        got_v = dv[h * g.NB:(h + 1) * g.NB].reshape(g.Sp, -1)
        np.testing.assert_allclose(got_k, rk, rtol=0, atol=1e-11)
        np.testing.assert_allclose(got_v, rv, rtol=0, atol=1e-11)


def test_kv_blocks_repeated_ids_count_twice():
    """A block listed twice in a row counts twice (the gather form accumulates
    both copies); a sample of blocks in any order gives the same rows."""
    g, qt, kt, vt, do, idx, num, valid = _problem(5, 9, 11, (4, 8, 8), 0, H=1, D=32, k=3, zero_rows=False)
    idx = idx.copy()
    r = 1
    idx[0, 0, r, :3] = [idx[0, 0, r, 0], idx[0, 0, r, 0], (idx[0, 0, r, 0] + 1) % g.NB]
    num = num.copy()
    num[0, 0, r] = 3
    rk, rv = _autograd_gather(qt, kt, vt, do, idx, num, g, valid, 0)
    order = np.array([5, 0, 3, 1], dtype=np.int64) % g.NB
    dk, dv = oracle.attn_bwd_kv_blocks(g, qt, kt, vt, do, idx, num, order)
    for n, kb in enumerate(order):
        np.testing.assert_allclose(dk[n], rk[kb * g.bs:(kb + 1) * g.bs], rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[n], rv[kb * g.bs:(kb + 1) * g.bs], rtol=0, atol=1e-11)
    # and the whole-problem form agrees with the gather form on the repeated ids
    fk, fv = oracle.attn_bwd_kv(g, qt, kt, vt, do, idx, num)
    np.testing.assert_allclose(fk[0, 0], rk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(fv[0, 0], rv, rtol=0, atol=1e-11)


def test_kv_blocks_rejects_out_of_range_block():
    g, qt, kt, vt, do, idx, num, valid = _problem(4, 8, 8, H=1, D=16, k=1)
    with pytest.raises(ValueError):
        oracle.attn_bwd_kv_blocks(g, qt, kt, vt, do, idx, num, np.array([g.NB], np.int64))
