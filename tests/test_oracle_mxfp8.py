"""Pins of the oracle's MXFP8 quantisation of index queries and keys (Index
Q/K Uses MXFP8, section 4.2 of "Inference Adaptation and Performance
Optimization for New Large Language Model Architectures": per-group dynamic
quantisation, 32 elements per scale factor).

Reading pinned here: the scale is absmax / 448 rounded up to a power of two
2^e (an E8M0 byte e + 127), so no element saturates; codes are the E4M3 cast
of x / 2^e. The cast is pinned to an independent library (ml_dtypes), the
scale rule by brute force, the format by worked values.
"""
import ml_dtypes
import numpy as np

import oracle
from indexed_sparse_attention_relu_b200 import workloads as W


def test_worked_groups():
    x = np.zeros((4, 32), np.float32)
    x[0, :2] = [448.0, -1.0]       # absmax 448 = 448 * 2^0 -> e = 0, 448 -> code 0x7E
    x[1, :2] = [449.0, 3.0]        # just above: e = 1; 449 / 2 = 224.5 -> 224 (ties to even) -> 448 after scaling
    x[3, :2] = [1e-3, -7e-4]       # e = ceil(log2(1e-3 / 448)) = -18
    codes, sb = oracle.mx_quantize(x)
    e = sb.astype(np.int64)[:, 0] - 127
    assert list(e) == [0, 1, -127, -18]
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xB8          # -1 = 1 1000 000
    assert np.all(codes[2] == 0)
    deq = oracle.mx_dequantize(codes, sb)
    assert deq[0, 0] == 448.0 and deq[0, 1] == -1.0 and deq[1, 0] == 448.0 and deq[1, 1] == 3.0
    # 1e-3 * 2^18 = 262.1 -> 256 (E4M3 step 32 in [256, 512)); -7e-4 * 2^18 = -183.5 -> -176 (step 16)
    assert codes[3, 0] == 0x78 and codes[3, 1] == 0xF3
    assert deq[3, 0] == 2.0 ** -10 and deq[3, 1] == -176.0 * 2.0 ** -18


def test_scale_is_least_power_of_two_covering_absmax():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((200, 128)) * np.exp(rng.uniform(-20, 20, (200, 1)))).astype(np.float32)
    x[7, 32:64] = 448.0 * 2.0 ** 5          # exactly on a boundary: e = 5
    x[8, :32] = 0.0
    codes, sb = oracle.mx_quantize(x)
    e = sb.astype(np.int64) - 127
    amax = np.abs(x.astype(np.float64)).reshape(200, 4, 32).max(-1)
    nz = amax > 0
    assert np.all(448.0 * np.ldexp(1.0, e[nz]) >= amax[nz])
    assert np.all(448.0 * np.ldexp(1.0, e[nz] - 1) < amax[nz])
    assert e[7, 1] == 5 and e[8, 0] == -127 and np.all(codes[8, :32] == 0)


def test_codes_match_the_library_cast_and_never_saturate():
    rng = np.random.default_rng(6)
    x = W.bf16_round(rng.standard_normal((64, 128)).astype(np.float32) * 3.0)
    codes, sb = oracle.mx_quantize(x)
    s = np.repeat(np.ldexp(1.0, sb.astype(np.int64) - 127), 32, axis=-1)
    lib = (x.astype(np.float64) / s).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(lib, codes)
    assert np.all(np.abs(x / s) <= 448.0)


def test_dequantised_values_are_exact_in_bf16_and_within_half_a_step():
    rng = np.random.default_rng(7)
    x = W.bf16_round(rng.standard_normal((32, 128)).astype(np.float32))
    codes, sb = oracle.mx_quantize(x)
    deq = oracle.mx_dequantize(codes, sb)
    assert np.array_equal(W.bf16_round(deq.astype(np.float32)).astype(np.float64), deq)
    s = np.repeat(np.ldexp(1.0, sb.astype(np.int64) - 127), 32, axis=-1)
    m = np.abs(x.astype(np.float64)) / s
    step = 2.0 ** (np.floor(np.log2(np.maximum(m, 2.0 ** -6))) - 3)
    assert np.all(np.abs(deq - x) <= 0.5 * step * s + 1e-300)
