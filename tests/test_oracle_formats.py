"""Pins of the oracle's number formats: binary16, round-half-away, Q4_0, Q8_0.

The formats are the Q4_0-family weights and 8-bit activations of the Dutch
technical summary of "A 35B Hybrid-Attention Mixture-of-Experts Model on a 6GB
2011 GPU" (Methodologie 1 and 2).  Pins: hand-worked blocks (tests/golden/),
numpy's own binary16 conversion, and properties every Q8_0 block must have.
"""
import numpy as np
import pytest

import oracle
from golden_io import hexbytes, rows


def test_half_to_double_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_float_to_half_golden():
    for val, bits in rows("fp16_rne.txt"):
        got = int(oracle.float_to_half_rne(np.float32(float(val))))
        assert got == int(bits, 16), (val, hex(got), bits)


def test_float_to_half_matches_numpy_random_and_edges():
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(0.02),
        rng.standard_normal(5000).astype(np.float32) * np.float32(3e4),
        (rng.random(5000) * 2e-4).astype(np.float32),          # subnormal and near-normal halves
        np.float32([65504, 65519, 65520, 65536, 1e30, -1e30, 2.0 ** -24, 2.0 ** -25, 0.0, -0.0]),
        # every binary16 value and the midpoints next to each, as binary32
        np.arange(0, 31744, dtype=np.uint16).view(np.float16).astype(np.float32),
    ])
    mids = np.arange(1, 31744, dtype=np.uint16).view(np.float16).astype(np.float64)
    lows = np.arange(0, 31743, dtype=np.uint16).view(np.float16).astype(np.float64)
    vals = np.concatenate([vals, ((mids + lows) / 2).astype(np.float32)])
    ours = oracle.float_to_half_rne(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("v,expect", [
    (2.5, 3), (-2.5, -3), (0.5, 1), (-0.5, -1), (1.5, 2), (3.5, 4), (4.5, 5),
    (np.nextafter(np.float32(0.5), np.float32(0)), 0), (-np.nextafter(np.float32(0.5), np.float32(0)), 0),
    (126.5, 127), (127.49998, 127), (0.0, 0), (-0.0, 0), (1e-30, 0),
])
def test_round_half_away(v, expect):
    assert int(oracle.round_half_away(np.float32(v))) == expect


def test_q4_0_golden_blocks():
    for name, hx, vals in rows("q4_0_blocks.txt"):
        blk = np.frombuffer(hexbytes(hx), dtype=np.uint8).reshape(1, 18)
        expect = np.array([float(v) for v in vals.split()])
        assert expect.size == 32, name
        got = oracle.q4_0_dequant(blk)
        assert np.array_equal(got, expect), name


def test_q8_0_golden_blocks():
    for name, d16, xs, qs in rows("q8_0_blocks.txt"):
        x = np.array([float(v) for v in xs.split()], dtype=np.float32)
        eq = np.array([int(v) for v in qs.split()], dtype=np.int8)
        assert x.size == 32 and eq.size == 32, name
        q, d, ov = oracle.quantize_q8_0(x)
        assert not ov
        assert int(d[0]) == int(d16, 16), name
        assert np.array_equal(q, eq), (name, q, eq)


def _q8_props(x, q, d):
    """Properties of Q8_0 that do not restate its formula: |q| <= 127; the
    largest |x| of a block maps to +-127; reconstruction error at most half
    a binary32 step (plus binary32 rounding of d and of the quotient)."""
    xb = x.reshape(-1, 32).astype(np.float64)
    qb = q.reshape(-1, 32).astype(np.int64)
    amax = np.abs(xb).max(axis=1)
    d32 = (amax / 127.0)
    assert np.all(np.abs(qb) <= 127)
    nz = amax > 0
    arg = np.abs(xb).argmax(axis=1)
    assert np.all(np.abs(qb[np.arange(len(qb)), arg])[nz] == 127)
    err = np.abs(xb - qb * d32[:, None])
    assert np.all(err <= d32[:, None] * (0.5 + 1e-5) + 1e-30)
    assert np.all(qb[~nz] == 0)
    # signs agree where q != 0
    assert np.all(np.sign(qb) * np.sign(xb) >= 0)
    # stored scale is binary16 of d within half a binary16 step
    dd = d.astype(np.uint16).view(np.float16).astype(np.float64)
    fin = np.isfinite(dd)
    assert np.all(np.abs(dd[fin] - d32[fin]) <= np.abs(d32[fin]) * 2.0 ** -11 + 2.0 ** -25)


def test_q8_0_properties_random():
    rng = np.random.default_rng(11)
    x = rng.standard_normal(32 * 4000).astype(np.float32) * np.float32(3.0)
    x[:32] = 0.0
    x[32:64] *= np.float32(1e-20)
    q, d, ov = oracle.quantize_q8_0(x)
    assert not ov
    _q8_props(x, q, d)


def test_q8_0_scale_overflow_flag():
    x = np.zeros(64, np.float32)
    x[0] = 1e8        # d = 1e8/127 > 65504 -> binary16 infinity
    q, d, ov = oracle.quantize_q8_0(x)
    assert ov
    assert int(d[0]) == 0x7C00 and int(d[1]) == 0
