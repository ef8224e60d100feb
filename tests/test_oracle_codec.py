"""Pins of the oracle's E4M3 codec (CPU only).

The codec follows the E4M3 format definition (bias 7, 3 mantissa bits,
subnormals m*2^-9, no infinities, 0x7F NaN, max 448); FP8 KV storage is named
by the yololab.net TensorRT-LLM guide, "FP8 與極致量化".  Pinned against:
  * torch's float8_e4m3fn conversion (a library routine) for every code and
    for every bf16 input under three scales,
  * hand-derived points in tests/golden/e4m3_points.txt.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros are distinct codes
    assert math.copysign(1.0, ours[0x80]) == -1.0 and ours[0] == 0.0


@pytest.mark.parametrize("scale", [1.0, 0.37, 2.0**-4])
def test_quantize_exhaustive_bf16_vs_torch(scale):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    finite = np.isfinite(x)
    bits, x = bits[finite], x[finite]
    codes = oracle.fp8_quantize(bits, np.float32(scale))
    # Library route: IEEE fp32 quotient, clamp to the finite range (satfinite),
    # then torch's round-to-nearest-even cast.
    y = (x / np.float32(scale)).astype(np.float32)
    yc = np.clip(y, -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(yc).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch drops the sign of values that round to zero only if they were +0;
    # compare magnitudes for zero codes and exact codes elsewhere.
    mism = codes != ref
    zero_sign_only = mism & ((codes & 0x7F) == 0) & ((ref & 0x7F) == 0)
    assert not np.any(mism & ~zero_sign_only), np.nonzero(mism & ~zero_sign_only)[0][:10]
    # The sign of zero codes follows the sign of the input.
    z = (codes & 0x7F) == 0
    assert np.array_equal(codes[z] >> 7, (np.signbit(y[z])).astype(np.uint8))


def test_quotient_is_ieee_fp32_division():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 65536, size=2000).astype(np.uint16)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    ok = np.isfinite(x)
    scales = rng.uniform(1e-3, 10, size=2000).astype(np.float32)
    L = oracle.lib()
    for b, s, good in zip(bits, scales, ok):
        if not good:
            continue
        q = L.oracle_fp8_quotient(int(b), float(s))
        ref = np.float32((np.uint32(b) << np.uint32(16)).view(np.float32) / s)
        assert np.float32(q) == ref


def _parse_golden():
    pts = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            val, code, *_ = line.split()
            v = float(eval(val, {"__builtins__": {}}))  # literals like 3*2**-10
            pts.append((np.float32(v), int(code, 16)))
    return pts


def test_golden_points():
    pts = _parse_golden()
    assert len(pts) >= 10
    for v, code in pts:
        got = int(oracle.e4m3_encode(np.array([v], np.float32))[0])
        assert got == code, (v, hex(got), hex(code))


def test_infinities_saturate_and_nan_maps_to_nan_code():
    y = np.array([np.inf, -np.inf, np.nan, -np.nan], np.float32)
    c = oracle.e4m3_encode(y)
    assert c[0] == 0x7E and c[1] == 0xFE
    assert (c[2] & 0x7F) == 0x7F and (c[3] & 0x7F) == 0x7F


def test_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


# ------------------------------------------------------------------- INT8
# Symmetric INT8 KV codes (concept page, "關鍵機制" quantisation bullet):
# nearest integer of the fp32 quotient, ties to even, clamped to +-127.
GOLDEN_INT8 = os.path.join(os.path.dirname(__file__), "golden", "int8_points.txt")


def test_int8_golden_points():
    pts = []
    for line in open(GOLDEN_INT8):
        line = line.strip()
        if line and not line.startswith("#"):
            val, code, *_ = line.split()
            pts.append((np.float32(float(val)), int(code)))
    assert len(pts) >= 12
    got = oracle.int8_encode(np.array([v for v, _ in pts], np.float32))
    assert got.tolist() == [c for _, c in pts]


@pytest.mark.parametrize("scale", [1.0, 0.37, 2.0**-4, 0.01])
def test_int8_quantize_exhaustive_bf16_vs_numpy(scale):
    # Library route: IEEE fp32 quotient, numpy's rint (round half to even),
    # clip to the symmetric range.
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    finite = np.isfinite(x)
    bits, x = bits[finite], x[finite]
    codes = oracle.int8_quantize(bits, np.float32(scale))
    with np.errstate(over="ignore"):
        y = (x / np.float32(scale)).astype(np.float32)
    ref = np.clip(np.rint(y.astype(np.float64)), -127, 127).astype(np.int8)
    assert np.array_equal(codes, ref)
    assert codes.min() >= -127  # -128 never stored


def test_int8_specials():
    c = oracle.int8_encode(np.array([np.inf, -np.inf, np.nan], np.float32))
    assert c.tolist() == [127, -127, 0]
    # every code round-trips through its value
    vals = np.arange(-127, 128, dtype=np.float32)
    assert oracle.int8_encode(vals).tolist() == list(range(-127, 128))
