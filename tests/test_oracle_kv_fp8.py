"""Pins of the oracle's FP8 latent-KV cache (Block-Wise Quantization for
Key-Value Cache, section 4 of "Optimizing Inference for New Model
Architectures ..."; Tiered Quantization table of "Day-0 Inference Adaptation
..."): per token, the latent dims in 128-element tiles with scale =
absmax / 448 and an E4M3 code per element; the rope dims stay bf16 (a
reading: a 576-dim row is 4.5 tiles, and the rope part is kept exact).

The codec pins (ml_dtypes, the format table) live in test_oracle_codec.py;
here the KV layout on top of it is pinned by worked values, the per-tile
error bound, tile independence and the K = 1 attention identity.
"""
import ml_dtypes
import numpy as np

import oracle
from indexed_sparse_attention_relu_b200 import workloads as W


def test_hand_worked_tile_scales():
    # two tiles of 128 (dc = 256) + 4 rope dims; tile 0 peaks at 8.96, tile 1 is all zero
    kv = np.zeros((1, 260), np.float32)
    kv[0, 5] = -8.96
    kv[0, 7] = 4.48
    kv[0, 256:] = [1.5, -2.0, 0.25, 3.0]
    codes, scales, rope = oracle.quantize_kv(kv, dc=256)
    s0 = np.float32(8.96) / np.float32(448.0)         # fl32(absmax / 448)
    assert scales.shape == (1, 2) and scales[0, 0] == s0 and scales[0, 1] == 0.0
    # -8.96 / s0 rounds to -448 = -1.75 * 2^8 (code 1 1111 110 = 0xFE);
    # 4.48 / s0 rounds to 224 = 1.75 * 2^7 (code 0 1110 110 = 0x76)
    assert codes[0, 5] == 0xFE and codes[0, 7] == 0x76
    assert np.all(codes[0, 128:] == 0)                  # a zero tile has scale 0 and codes 0
    assert np.array_equal(rope, kv[:, 256:])
    deq = oracle.dequantize_kv(codes, scales, rope)
    assert deq[0, 5] == -448.0 * float(s0) and deq[0, 7] == 224.0 * float(s0)
    assert np.array_equal(deq[0, 256:], [1.5, -2.0, 0.25, 3.0])


def test_roundtrip_error_bound_per_tile():
    """|x - decode(code) * s| <= half an E4M3 step at |x| / s, times s: the
    step of E4M3 at magnitude m in [2^e, 2^(e+1)) is 2^(e-3), below 2^-6 it
    is 2^-9 (subnormals)."""
    rng = np.random.default_rng(1)
    kv = W.bf16_round(rng.standard_normal((64, 576)).astype(np.float32) * rng.uniform(0.01, 30, (64, 1)))
    codes, scales, rope = oracle.quantize_kv(kv, dc=512)
    deq = oracle.dequantize_kv(codes, scales, rope)
    s = np.repeat(scales.astype(np.float64), 128, axis=-1)
    m = np.abs(kv[:, :512].astype(np.float64)) / s
    e = np.floor(np.log2(np.maximum(m, 2.0 ** -6)))
    step = 2.0 ** (e - 3)
    err = np.abs(deq[:, :512] - kv[:, :512])
    assert np.all(err <= 0.5 * step * s * (1 + 1e-6) + 1e-300)
    assert np.array_equal(deq[:, 512:], kv[:, 512:].astype(np.float64))


def test_tiles_are_independent_and_match_the_library_cast():
    rng = np.random.default_rng(2)
    kv = W.bf16_round(rng.standard_normal((8, 576)).astype(np.float32))
    codes, scales, _ = oracle.quantize_kv(kv, dc=512)
    kv2 = kv.copy()
    kv2[:, 128:256] *= 1000.0                            # only tile 1 changes
    codes2, scales2, _ = oracle.quantize_kv(kv2, dc=512)
    keep = np.r_[0:128, 256:512]
    assert np.array_equal(codes[:, keep], codes2[:, keep])
    assert np.array_equal(scales[:, [0, 2, 3]], scales2[:, [0, 2, 3]])
    # each code is the library's round-to-nearest-even E4M3 cast of fl32(x / s)
    s = np.repeat(scales, 128, axis=-1)
    x = (kv[:, :512] / s).astype(np.float32)
    lib = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(lib, codes)


def test_small_latent_is_one_tile():
    """d_c = 64 (the tiny configuration): one tile of 64 elements."""
    rng = np.random.default_rng(3)
    kv = W.bf16_round(rng.standard_normal((5, 80)).astype(np.float32))
    codes, scales, rope = oracle.quantize_kv(kv, dc=64)
    assert codes.shape == (5, 64) and scales.shape == (5, 1) and rope.shape == (5, 16)
    want = (np.abs(kv[:, :64]).max(axis=1) / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(scales[:, 0], want)


def test_single_key_attention_returns_the_dequantised_value_row():
    """K = 1: softmax weight 1, so out = the selected row's dequantised latent
    part exactly and lse = its logit."""
    wl = W.scaled("c2", B=1, Lmax=300, lens=(300,), T_per_seq=3, K=1)
    codes, scales, rope = oracle.quantize_kv(wl.kv, dc=wl.dc)
    kv64 = oracle.dequantize_kv(codes, scales, rope)
    idx = np.array([[17], [250], [0]], np.int32)
    out, lse = oracle.sparse_mla(wl, idx, kv=kv64)
    for r in range(3):
        row = kv64[0, idx[r, 0]]
        assert np.array_equal(out[r], np.broadcast_to(row[:wl.dc], out[r].shape))
        z = wl.softmax_scale * (wl.q[r].astype(np.float64) @ row)
        assert np.allclose(lse[r], z, rtol=1e-12, atol=1e-12)
