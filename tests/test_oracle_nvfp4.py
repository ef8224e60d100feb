"""Pins of the oracle's FP4 (E2M1 + E4M3 block scale) codec, on CPU.

What the format fixes, checked against things other than the oracle itself:

* the E2M1 value table: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit,
  magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
* encoding = brute-force nearest table value, ties to the even code,
  saturation at 6, sign kept for zero, NaN -> +0;
* block quantisation: rows built from known codes and a power-of-two scale
  come back exactly; random rows stay within the error the two roundings
  allow; all-zero blocks, NaN elements and the nibble order.
"""
import math
import os

import numpy as np
import pytest

import oracle

# E2M1 magnitudes in code order (exponent field 0: 0, 0.5; then (1 + m/2) 2^(e-1))
_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _brute_e2m1(y: float) -> int:
    if math.isnan(y):
        return 0
    sign = 8 if math.copysign(1.0, y) < 0 else 0
    a = abs(y)
    if a >= 6.0:
        return sign | 7
    best = min(range(8), key=lambda c: (abs(_MAGS[c] - a), c & 1))  # tie: even code
    return sign | best


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bits (the inputs here are exact)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def test_e2m1_value_table():
    v = oracle.e2m1_decode(np.arange(16))
    assert list(v[:8]) == _MAGS
    assert list(-v[8:]) == _MAGS
    assert math.copysign(1.0, v[8]) < 0  # code 8 is -0


def test_e2m1_encode_matches_brute_force():
    grid = np.arange(-8.0, 8.0 + 1e-9, 1.0 / 64).astype(np.float32)
    # the exact midpoints and their fp32 neighbours
    mids = np.array([(a + b) / 2 for a, b in zip(_MAGS, _MAGS[1:])], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                           np.nextafter(mids, np.float32(10))])
    ys = np.concatenate([grid, near, -near, np.float32([np.inf, -np.inf, np.nan, -0.0, 1e-30])])
    got = oracle.e2m1_encode(ys)
    want = np.array([_brute_e2m1(float(y)) for y in ys], np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_round_trip_of_every_code():
    v = oracle.e2m1_decode(np.arange(16)).astype(np.float32)
    assert list(oracle.e2m1_encode(v)) == list(range(16))


@pytest.mark.parametrize("s_exp", [-10, -4, 0, 3])
def test_block_quantisation_is_exact_on_representable_rows(s_exp):
    rng = np.random.default_rng(11 + s_exp)
    s = np.float32(2.0 ** s_exp)
    rows, n = 6, 64
    codes = rng.integers(0, 16, size=(rows, n)).astype(np.uint8)
    codes[:, ::16] = 7  # every block's largest magnitude is 6, so amax / (6 s) = block scale
    blocks = rng.integers(0x20, 0x60, size=(rows, n // 16)).astype(np.uint8)  # normal E4M3 scales
    vals = oracle.e2m1_decode(codes) * oracle.e4m3_decode(np.repeat(blocks, 16, axis=1)) * float(s)
    assert np.array_equal(vals.astype(np.float32).astype(np.float64), vals)  # exact in fp32
    x_bits = _bf16_bits(vals.astype(np.float32))
    back = x_bits.astype(np.uint32) << 16
    assert np.array_equal(back.view(np.float32).astype(np.float64), vals)  # exact in bf16
    packed, got_blocks = oracle.nvfp4_quantize(x_bits, s)
    assert np.array_equal(got_blocks, blocks)
    lo, hi = packed & 0xF, packed >> 4
    got = np.empty_like(codes)
    got[:, 0::2], got[:, 1::2] = lo, hi
    # -0 and +0 are the same value: compare values, then the codes of nonzero ones
    assert np.array_equal(oracle.nvfp4_dequantize(packed, got_blocks, s), vals)
    nz = vals != 0
    assert np.array_equal(got[nz], codes[nz])


def test_block_quantisation_error_bound_on_random_rows():
    rng = np.random.default_rng(5)
    rows, n = 32, 128
    x = rng.standard_normal((rows, n)).astype(np.float32)
    x_bits = _bf16_bits(x)
    xf = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = (np.abs(xf).max(axis=1) / (448.0 * 6.0)).astype(np.float32)  # the harness's choice
    packed, blocks = oracle.nvfp4_quantize(x_bits, s)
    xq = oracle.nvfp4_dequantize(packed, blocks, s)
    for r in range(rows):
        for b in range(n // 16):
            blk = slice(16 * b, 16 * b + 16)
            amax = np.abs(xf[r, blk]).max()
            # E4M3 rounding of the block scale: relative error <= 2^-4
            unit = oracle.e4m3_decode(blocks[r, b]) * float(s[r])
            assert abs(unit * 6.0 - amax) <= amax * 2.0**-4 + 1e-30
            err = np.abs(xq[r, blk] - xf[r, blk])
            # unsaturated: half the E2M1 spacing (at most 1 unit); saturated: amax - 6 unit.
            # Codes are chosen against fp32(sb * s) while values use the exact sb * s:
            # a relative slack of 2^-20 covers that rounding.
            bound = max(unit, amax - 6.0 * unit) * (1.0 + 2.0**-20)
            assert np.all(err <= bound)
            # order and sign are kept
            o = np.argsort(xf[r, blk], kind="stable")
            assert np.all(np.diff(xq[r, blk][o]) >= 0)
            assert np.all(np.sign(xq[r, blk]) * np.sign(xf[r, blk]) >= 0)


def test_zero_block_nan_and_nibble_order():
    x = np.zeros((1, 32), np.float32)
    x[0, 16] = 3.0   # block 1: amax 3 -> its largest code is 6 (value 3 / unit 0.5 = 6)
    x[0, 17] = np.nan
    x[0, 18] = -1.5
    x_bits = _bf16_bits(x)
    packed, blocks = oracle.nvfp4_quantize(x_bits, np.float32(1.0))
    assert blocks[0, 0] == 0 and np.all(packed[0, :8] == 0)  # all-zero block
    unit = oracle.e4m3_decode(blocks[0, 1])
    assert unit == 0.5  # 3 / 6 is exact in E4M3
    assert packed[0, 8] & 0xF == 7          # element 16 (low nibble): 3 / 0.5 = 6
    assert packed[0, 8] >> 4 == 0           # element 17 (high nibble): NaN -> 0
    assert packed[0, 9] & 0xF == 8 | 5      # element 18: -1.5 / 0.5 = -3
    vals = oracle.nvfp4_dequantize(packed, blocks, np.float32(1.0))
    assert vals[0, 16] == 3.0 and vals[0, 17] == 0.0 and vals[0, 18] == -1.5


GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_points.txt")


def test_golden_points():
    elems, blocks = [], []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        f = line.split()
        if f[0] == "block":
            blocks.append(f[1:])
        else:
            elems.append((np.float32(float(f[0])), int(f[1], 16)))
    assert len(elems) >= 15 and blocks
    got = oracle.e2m1_encode(np.array([v for v, _ in elems], np.float32))
    assert got.tolist() == [c for _, c in elems]
    for b in blocks:
        s = np.float32(float(b[0]))
        x = np.array([float(v) for v in b[1:17]], np.float32)
        packed, scales = oracle.nvfp4_quantize(_bf16_bits(x)[None], s)
        assert scales[0, 0] == int(b[17], 16)
        assert packed[0].tolist() == [int(v, 16) for v in b[18:26]]
