"""Pins of the oracle's fp8 weight decoding (the quantised expert weights).

e4m3 codes against their definition at hand-picked patterns and against
torch's float8_e4m3fn conversion for all 256 codes; the block-scaled
dequantisation against closed forms that expose the scale layout (which
block, which row, the K-block-major transposition).
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import workloads as W


def test_e4m3_known_patterns():
    v = oracle.e4m3_to_f64(np.array([0x00, 0x38, 0x7E, 0x01, 0x08, 0xB8, 0x40, 0x3C], np.uint8))
    assert list(v) == [0.0, 1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -1.0, 2.0, 1.5]
    assert np.isnan(oracle.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours[~both_nan], ref[~both_nan]) and np.array_equal(np.isnan(ours), np.isnan(ref))


def test_dequant_scale_layout_closed_form():
    E, R, K = 2, 5, 96
    q = np.full((E, R, K), 0x38, np.uint8)                     # every value 1.0
    s = np.zeros((E, K // 32, R), np.uint8)
    for e in range(E):
        for b in range(K // 32):
            for r in range(R):
                s[e, b, r] = 120 + e + 2 * b + 3 * r          # distinct per (expert, block, row)
    w = oracle.dequant_mxfp8(q, s)
    for e in range(E):
        for r in range(R):
            for c in range(K):
                assert w[e, r, c] == 2.0 ** (120 + e + 2 * (c // 32) + 3 * r - 127)


def test_quantised_weights_round_trip_within_e4m3_precision():
    rng = np.random.default_rng(3)
    w = W.f32_to_bf16_bits((rng.standard_normal((3, 64, 128)) * 0.02).astype(np.float32))
    q, s = W.quantize_mxfp8(w)
    assert q.shape == (3, 64, 128) and s.shape == (3, 4, 64)
    back = oracle.dequant_mxfp8(q, s)
    ref = oracle.bf16_to_f64(w)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normal values,
    # and the block's scale puts its largest value in [224, 448]
    err = np.abs(back - ref)
    scale = np.exp2(np.repeat(np.swapaxes(s.astype(np.int64) - 127, -1, -2), 32, axis=-1))
    assert (err <= np.maximum(np.abs(ref) * 2.0 ** -4, scale * 2.0 ** -10) + 1e-30).all()
    blocks = np.abs(back).reshape(3, 64, 4, 32).max(axis=3)
    assert ((blocks >= 224 * np.exp2(s.transpose(0, 2, 1).astype(np.int64) - 127)) | (blocks == 0)).all()
