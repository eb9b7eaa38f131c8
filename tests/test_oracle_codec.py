"""Pins for the oracle's FP8 (OCP E4M3) codec and the index-key cache write.

The codec is pinned to an independent library implementation of the OCP FP8
format (ml_dtypes) and to values fixed by the format definition; the cache
write (per-group scale = max|group| / 448, then the 8-bit cast, as in the
"Tiered Quantization" table and pseudocode of "Day-0 Inference Adaptation and
Performance Optimization for New-Architecture Large Language Models") is pinned
by its error bound and its special cases.
"""
import os

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lib_decode(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_decode_all_codes_match_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = _lib_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    # sign of zero survives
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


def test_decode_matches_golden_format_table():
    """Landmark values of the OCP 8-bit floating point E4M3 format."""
    path = os.path.join(GOLDEN, "e4m3_landmarks.txt")
    n = 0
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        code, value = line.split()
        code = int(code, 16)
        got = oracle.e4m3_decode(np.array([code], np.uint8))[0]
        if value == "nan":
            assert np.isnan(got)
        else:
            assert got == float.fromhex(value) if value.startswith(("0x", "-0x")) else got == float(value)
        n += 1
    assert n >= 8


def test_encode_matches_library_in_range():
    rng = np.random.default_rng(11)
    # random magnitudes across the whole exponent range, both signs
    mags = np.exp2(rng.uniform(-12, np.log2(447.9), 200_000)).astype(np.float32)
    x = (mags * rng.choice([-1, 1], mags.size)).astype(np.float32)
    # every exact grid point and every midpoint between neighbours (ties)
    grid = _lib_decode(np.arange(0x7F, dtype=np.uint8))  # 0 .. 448, finite, positive
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, grid.astype(np.float32), mids, -mids, np.float32([0.0, -0.0])])
    ours = oracle.e4m3_encode(x)
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, ref)


def test_encode_ties_go_to_even_code():
    grid = _lib_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    codes = oracle.e4m3_encode(mids)
    assert np.all(codes % 2 == 0)
    assert np.all((codes == np.arange(0x7E)) | (codes == np.arange(1, 0x7F)))


def test_encode_saturates_finite():
    x = np.float32([448.0, 449.0, 464.0, 480.0, 1e6, 3.4e38, -448.0, -500.0, -3.4e38])
    assert list(oracle.e4m3_encode(x)) == [0x7E] * 6 + [0xFE] * 3


def test_encode_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_quantize_special_cases():
    k = np.zeros((3, 128), np.float32)
    k[1, 5] = -2.5                      # single non-zero
    k[2] = np.linspace(-1, 1, 128, dtype=np.float32)
    codes, scales = oracle.quantize_keys(k, 128)
    assert scales[0, 0] == 0.0 and not codes[0].any()
    # the absmax element maps to +-448 exactly (satfinite), the rest to 0
    assert codes[1, 5] == 0xFE and np.count_nonzero(codes[1]) == 1
    assert scales[1, 0] == np.float32(2.5) / np.float32(448)
    assert codes[2, 0] == 0xFE and codes[2, -1] == 0x7E


def test_quantize_error_bound_and_group_independence():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((500, 128)).astype(np.float32)
    for group in (32, 64, 128):
        codes, scales = oracle.quantize_keys(k, group)
        deq = oracle.e4m3_decode(codes) * np.repeat(scales.astype(np.float64), group, axis=-1)
        # |x/s - code| <= half a grid step at |x/s| (plus the fp32 quotient rounding)
        s = np.repeat(scales.astype(np.float64), group, axis=-1)
        xs = np.abs(k / s)
        e = np.floor(np.log2(np.maximum(xs, 2.0 ** -6)))
        half_step = np.exp2(e - 4)
        err = np.abs(deq - k) / s
        assert np.all(err <= half_step * (1 + 1e-6) + 1e-6 * xs)
        # per-group absmax hits the top of the grid
        amax = np.abs(k.reshape(500, -1, group)).max(-1)
        assert np.allclose(scales, amax / 448.0, rtol=1e-7, atol=0)
    # changing one group leaves the others untouched
    k2 = k.copy()
    k2[:, :32] *= 3.0
    c1, s1 = oracle.quantize_keys(k, 32)
    c2, s2 = oracle.quantize_keys(k2, 32)
    assert np.array_equal(c1[:, 32:], c2[:, 32:]) and np.array_equal(s1[:, 1:], s2[:, 1:])


def test_dequantize_is_single_rounding_of_exact_product():
    rng = np.random.default_rng(6)
    k = (rng.standard_normal((64, 128)) * 3).astype(np.float32)
    codes, scales = oracle.quantize_keys(k, 32)
    out = oracle.dequantize_keys(codes, scales, 32)
    exact = _lib_decode(codes) * np.repeat(scales.astype(np.float64), 32, axis=-1)
    assert np.array_equal(out, exact.astype(np.float32))
