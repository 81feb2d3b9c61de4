"""Pins for the oracle's NVFP4 -> bf16 expansion (the W4A16 path of "decode
dynamic-scale NVFP4 H3 VAE tiles one at a time" -- FASTVIDEO_H3_ENCODER_FUSED_DEQUANT).

* Exact values: with a power-of-two global scale every E2M1 x E4M3 product divided by it
  is exact and fits bf16, so the expansion must return it bit for bit (checked against
  ml_dtypes / torch decoders and an independent 128x4 permutation).
* An independent restatement with any global scale: the same decoders, numpy fp32
  division (IEEE) and torch's round-to-nearest-even cast to bf16.
* Signed zeros, zero scales, and a quantize -> expand round trip that stays within
  the block scale's half step.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from test_oracle_gemm import pack_codes, swizzle_by_reshape
from nvfp4_block_scaled_17_b200 import workloads as W


def decode_f32(codes, sf_lin):
    vals = codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    sc = torch.from_numpy(sf_lin).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    return vals * np.repeat(sc, 16, axis=1)          # exact in fp32


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return W.to_u16(torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16))


@pytest.mark.parametrize("R,K", [(1, 16), (37, 80), (130, 256)])
def test_power_of_two_global_scale_is_exact(oracle, R, K):
    rng = np.random.default_rng(R * K)
    codes = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    sf_lin = rng.integers(0, 0x7F, size=(R, K // 16), dtype=np.uint8)
    gsf = 2.0 ** 7
    y = oracle.dequantize_bf16(pack_codes(codes), swizzle_by_reshape(sf_lin, R, K), R, K, gsf)
    exact = decode_f32(codes, sf_lin) / np.float32(gsf)
    assert np.array_equal(W.from_u16(y).float().numpy(), exact)      # no rounding happened


@pytest.mark.parametrize("gsf", [1.0, 3.0, 864.4824, 1e-3, 7.77e5])
def test_independent_restatement(oracle, gsf):
    rng = np.random.default_rng(int(gsf * 10) % 1000)
    R, K = 129, 192
    codes = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    sf_lin = rng.integers(0, 0x7F, size=(R, K // 16), dtype=np.uint8)
    y = oracle.dequantize_bf16(pack_codes(codes), swizzle_by_reshape(sf_lin, R, K), R, K, gsf)
    want = bf16_bits(decode_f32(codes, sf_lin) / np.float32(gsf))
    assert np.array_equal(y, want)


def test_zeros_and_signed_zero(oracle):
    R, K = 2, 32
    codes = np.zeros((R, K), dtype=np.uint8)
    codes[0, :] = 8                       # -0
    codes[1, :] = 7                       # 6, but under a zero scale
    sf_lin = np.array([[0x38, 0x38], [0x00, 0x00]], dtype=np.uint8)
    y = oracle.dequantize_bf16(pack_codes(codes), swizzle_by_reshape(sf_lin, R, K), R, K, 2.0)
    assert np.all(y[0] == 0x8000) and np.all(y[1] == 0x0000)


def test_round_trip_within_half_step(oracle):
    x = W.with_outliers((128, 256), 0.01, 20.0, W._gen(0, "cpu"), "cpu")
    xu = W.to_u16(x)
    packed, sf, gsf = oracle.quantize(xu)
    y = W.from_u16(oracle.dequantize_bf16(packed, sf, 128, 256, gsf)).double().numpy()
    xd = x.double().numpy()
    # per block: |x - y| <= half the largest E2M1 step (2) times the block scale, plus
    # the saturation excess and one bf16 rounding of y
    s = oracle.dequantize(packed, sf, 128, 256)          # code * scale, no global scale
    blk = np.abs(s).reshape(128, 16, 16).max(axis=2) / 6.0 / gsf   # block scale / gsf
    tol = np.repeat(blk, 16, axis=1) * 1.0 + np.abs(y) * 2.0 ** -8
    over = np.maximum(np.abs(xd) - 6.0 * np.repeat(blk, 16, axis=1), 0.0)
    assert np.all(np.abs(xd - y) <= tol + over + 1e-30)
