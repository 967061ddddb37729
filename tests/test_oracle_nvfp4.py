"""Pins of the oracle's NVFP4 quantisation of Q and K and of its attention on
the quantised operands.

Source: FastVideo "Optimizations" page, section "FP4 Flash Attention 4
(Blackwell only)": Q and K go to NVFP4 (4-bit E2M1 codes, one E4M3 scale per
block of channels), V keeps its 16-bit format.  Readings (NVFP4's own definition): blocks
of 16 consecutive channels, scale = E4M3(fl32(amax / 6)), value codes =
E2M1(fl32(x * fl32(1 / scale))), both roundings to nearest with ties to an even
last mantissa bit, capped at the largest finite value, E2M1 keeping the sign.

The pins below fix each step from outside the oracle: torch's float8_e4m3fn
cast (a library rounding to E4M3), brute force over the eight E2M1 magnitudes,
the format tables written out by hand, error bounds, and the already pinned
16-bit attention on values that are exactly representable in bf16.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_video_gather_b200 import workloads

bf16 = workloads.f32_to_bf16_bits
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _e4m3_value(bits):
    """E4M3 bits -> value, from the format table (sign, 4 exponent bits bias 7, 3 mantissa bits)."""
    bits = np.asarray(bits, np.int64)
    e, m = (bits >> 3) & 15, bits & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7.0))
    return np.where(bits & 0x80, -mag, mag)


def _nearest_e2m1(y):
    """Brute force: nearest of the eight magnitudes, ties to the even code, sign kept."""
    a = np.minimum(np.abs(y), 6.0)
    d = np.abs(a[:, None] - E2M1[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(d == best, np.arange(8)[None, :], 99)
    # among tied codes take the even one (there are at most two, adjacent)
    code = np.where((cand % 2 == 0) & (cand < 99), cand, 99).min(axis=1)
    code = np.where(code == 99, cand.min(axis=1), code)
    return code | np.where(np.signbit(y), 8, 0)


def _unpack(codes):
    lo, hi = codes & 15, codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))


def test_scale_rounding_matches_library_e4m3_cast():
    """Every E4M3 grid point, every midpoint between neighbours (ties), and a
    dense random sweep, up to the last value that rounds to 448."""
    grid = _e4m3_value(np.arange(0x7F)).astype(np.float64)
    mids = (grid[:-1] + grid[1:]) / 2
    rng = np.random.default_rng(0)
    sweep = np.exp(rng.uniform(np.log(1e-4), np.log(460.0), 20000))
    x = np.concatenate([grid, mids, sweep, [455.0, 463.9]]).astype(np.float32)
    assert np.array_equal(oracle.e4m3_round(x), _torch_e4m3(x))


def test_scale_saturates_at_448():
    assert (oracle.e4m3_round(np.array([464.0, 500.0, 1e6, 3e38], np.float32)) == 0x7E).all()


def test_scale_of_a_block_is_e4m3_of_amax_over_6():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 128)) * np.exp(rng.uniform(-6, 4, (64, 1)))).astype(np.float32)
    xb = bf16(x)
    _, sf = oracle.quant_nvfp4(xb)
    xf = workloads.bf16_bits_to_f32(xb).reshape(64, 8, 16)
    amax = np.abs(xf).max(axis=2).astype(np.float32)
    assert np.array_equal(sf, _torch_e4m3(amax / np.float32(6.0)))


def test_codes_with_unit_scale_are_nearest_e2m1():
    """A block whose amax is 6 has scale exactly 1, so its codes are E2M1(x):
    brute force over every multiple of 1/64 in [-6, 6] (all ties between E2M1
    neighbours included) and both zeros."""
    vals = np.concatenate([np.arange(-6 * 64, 6 * 64 + 1) / 64.0, [-0.0]]).astype(np.float32)
    pad = (-len(vals)) % 15
    vals = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(-1, 15)
    x = np.concatenate([np.full((len(vals), 1), 6.0, np.float32), vals], axis=1)
    x = np.tile(x, (1, 8))  # D = 128: eight identical blocks
    codes, sf = oracle.quant_nvfp4(bf16(x))
    assert (sf == 0x38).all()  # E4M3 1.0
    got = _unpack(codes)
    want = _nearest_e2m1(workloads.bf16_bits_to_f32(bf16(x)).astype(np.float64).ravel()).reshape(got.shape)
    assert np.array_equal(got, want)


def test_nibble_order_and_dequantised_values():
    """Channel 2j is the low nibble of byte j; the decoded value is the E2M1
    magnitude times the E4M3 scale (tables written out here)."""
    rng = np.random.default_rng(2)
    x = bf16((rng.standard_normal((32, 128)) * 3).astype(np.float32))
    codes, sf = oracle.quant_nvfp4(x)
    c = _unpack(codes)
    mag = E2M1[c & 7] * np.where(c & 8, -1.0, 1.0)
    want = mag * np.repeat(_e4m3_value(sf), 16, axis=1)
    assert np.array_equal(oracle.dequant_nvfp4(codes, sf), want)
    # and the first channel of a block is the low nibble: put a lone 6 there
    y = np.zeros((1, 128), np.float32)
    y[0, 0] = 6.0
    cy, _ = oracle.quant_nvfp4(bf16(y))
    assert cy[0, 0] == 0x07 and (cy[0, 1:] == 0).all()


def test_quantisation_error_bound():
    """|x - deq(x)| is at most half the E2M1 spacing at |x|/s, times s, except
    where |x|/s exceeds 6 (the scale was rounded down): there the code is 6."""
    rng = np.random.default_rng(3)
    x = bf16((rng.standard_normal((256, 128)) * np.exp(rng.uniform(-3, 3, (256, 1)))).astype(np.float32))
    codes, sf = oracle.quant_nvfp4(x)
    xf = workloads.bf16_bits_to_f32(x).astype(np.float64)
    s = np.repeat(_e4m3_value(sf), 16, axis=1)
    y = np.abs(xf) / s
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    err = np.abs(xf - oracle.dequant_nvfp4(codes, sf))
    over = y > 6
    assert (err[~over] <= half[~over] * s[~over] * (1 + 1e-6)).all()
    assert np.array_equal(np.abs(_unpack(codes)[over]) & 7, np.full(over.sum(), 7))
    # the scale is never far from amax / 6: |y| <= 6 * (1 + 2^-4) at most
    assert y.max() <= 6.0 * (1 + 2.0 ** -4)


def test_zero_and_tiny_blocks():
    x = np.zeros((2, 128), np.float32)
    x[1, :16] = 1e-5  # amax / 6 rounds to E4M3 zero
    xb = bf16(x)
    xb[0, 16] = 0x8000  # -0.0
    codes, sf = oracle.quant_nvfp4(xb)
    assert (sf == 0).all()
    c = _unpack(codes)
    assert c[0, 16] == 8 and (np.delete(c[0], 16) == 0).all() and (c[1] == 0).all()


def test_exactly_representable_block_round_trips():
    s = 0.375  # E4M3 exact, and 6 * s = 2.25 exact in fp32
    pattern = np.array([6, -4, 3, -2, 1.5, -1, 0.5, 0, -6, 4, -3, 2, -1.5, 1, -0.5, 6]) * s
    x = np.tile(pattern, 8)[None, :].astype(np.float32)
    codes, sf = oracle.quant_nvfp4(bf16(x))
    assert (sf == _torch_e4m3(np.float32(s))).all()
    assert np.array_equal(oracle.dequant_nvfp4(codes, sf), x.astype(np.float64))


@pytest.mark.parametrize("shape", [((5, 9, 11), (4, 8, 8), 0), ((6, 8, 12), (4, 4, 4), 100)])
def test_attention_on_codes_is_attention_on_their_values(shape):
    """The dequantised values fit bf16 exactly (at most 2 + 4 significant bits),
    so attention on NVFP4 q, k equals the pinned 16-bit attention run on
    bf16(deq(q)), bf16(deq(k)), row for row and bit for bit."""
    (T, Hg, Wg), block, npre = shape
    wl = workloads.custom(T=T, Hg=Hg, Wg=Wg, block=block, n_prefix=npre, H=2, D=128, seed=4)
    g = oracle.geometry_of(wl)
    inp = workloads.make_inputs(wl, threads=1)
    qt, kt, vt = (oracle.tile(g, inp[n]) for n in ("q", "k", "v"))
    (qc, qs), (kc, ks) = oracle.quant_nvfp4(qt), oracle.quant_nvfp4(kt)
    qd, kd = oracle.dequant_nvfp4(qc, qs), oracle.dequant_nvfp4(kc, ks)
    assert np.array_equal(workloads.bf16_bits_to_f32(bf16(qd.astype(np.float32))).astype(np.float64), qd)
    rng = np.random.default_rng(5)
    k = min(3, g.NB)
    num = rng.integers(0, k + 1, size=(1, 2, g.NB)).astype(np.int32)
    idx = np.full((1, 2, g.NB, k), -1, np.int32)
    for pos in np.ndindex(1, 2, g.NB):
        idx[pos][:num[pos]] = np.sort(rng.permutation(g.NB)[:num[pos]])
    rows = np.arange(2 * g.Sp, dtype=np.int64)
    o4, l4 = oracle.attn_rows_nvfp4(g, qc, qs, kc, ks, vt, idx, num, rows)
    o2, l2 = oracle.attn_rows(g, bf16(qd.astype(np.float32)), bf16(kd.astype(np.float32)), vt, idx, num, rows)
    assert np.array_equal(o4, o2) and np.array_equal(l4, l2)
