"""Pins for the oracle's fp64 GEMM over dequantized NVFP4 operands and for the
whole oracle path.

* closed forms (constant operands),
* an independent restatement on tiny random operands: codes and scale bytes are
  decoded by ml_dtypes / torch, the 128x4 offsets by a tensor permutation, the
  product by numpy matmul,
* the pages' printed figure: W4A4 relative error against the bf16 product on
  random N(0,1) rows is about 0.13 ("convert_minimax_h3_text_encoder_nvfp4.py",
  module docstring and probe_relative_error), with negative controls: a wrong
  scale layout, swapped nibbles and a zeroed output read far from it.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_17_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def pack_codes(codes: np.ndarray) -> np.ndarray:
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def swizzle_by_reshape(sf_lin, R, K):
    Rp, Cp = (R + 127) // 128 * 128, (K // 16 + 3) // 4 * 4
    p = np.zeros((Rp, Cp), dtype=np.uint8)
    p[:R, :K // 16] = sf_lin
    return p.reshape(Rp // 128, 4, 32, Cp // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)


def decode_independent(codes, sf_lin):
    vals = codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = torch.from_numpy(sf_lin).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.repeat(sc, 16, axis=1)


def test_gemm_closed_form(oracle):
    M, N, K = 3, 5, 64
    a = np.full((M, K // 2), 0x22, dtype=np.uint8)                  # every code 2 = 1.0
    b = np.full((N, K // 2), 0x22, dtype=np.uint8)
    sfa = swizzle_by_reshape(np.full((M, K // 16), 0x38, np.uint8), M, K)   # 1.0
    sfb = swizzle_by_reshape(np.full((N, K // 16), 0x40, np.uint8), N, K)   # 2.0
    bias = W.to_u16(torch.tensor([0.5, -1, 0, 2, 3], dtype=torch.bfloat16))
    y = oracle.gemm_f64(a, sfa, b, sfb, M, N, K, 0.25, bias)
    want = 0.25 * K * 2.0 + np.array([0.5, -1, 0, 2, 3])
    assert np.array_equal(y, np.broadcast_to(want, (M, N)))


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (7, 9, 48), (130, 33, 128), (5, 260, 320)])
def test_gemm_independent_restatement(oracle, M, N, K):
    rng = np.random.default_rng(M + N + K)
    ca = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    sa = rng.integers(0, 0x7F, size=(M, K // 16), dtype=np.uint8)    # finite E4M3 only
    sb = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    bias = W.to_u16(W.random_bf16((N,), seed=5))
    alpha = 0.0078125
    y = oracle.gemm_f64(pack_codes(ca), swizzle_by_reshape(sa, M, K), pack_codes(cb),
                        swizzle_by_reshape(sb, N, K), M, N, K, alpha, bias)
    ref = alpha * decode_independent(ca, sa) @ decode_independent(cb, sb).T \
        + W.from_u16(bias).double().numpy()
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-300)
    rows = np.array([M - 1, 0], dtype=np.int64)
    ysub = oracle.gemm_f64(pack_codes(ca), swizzle_by_reshape(sa, M, K), pack_codes(cb),
                           swizzle_by_reshape(sb, N, K), M, N, K, alpha, bias, rows=rows)
    assert np.array_equal(ysub, y[rows])


def test_dequantize_matches_restatement(oracle):
    rng = np.random.default_rng(3)
    R, K = 131, 96
    codes = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    sf_lin = rng.integers(0, 0x7F, size=(R, K // 16), dtype=np.uint8)
    d = oracle.dequantize(pack_codes(codes), swizzle_by_reshape(sf_lin, R, K), R, K)
    assert np.array_equal(d, decode_independent(codes, sf_lin))


def probe(oracle, weight: torch.Tensor, rows: int, seed: int, corrupt=None):
    """The pages' probe: random bf16 rows, unit activation scale, the weight with
    its own dynamic global scale; relative error against the bf16 product."""
    N, K = weight.shape
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    ref = x.double() @ weight.double().T
    wp, wsf, gsf_w = oracle.quantize(W.to_u16(weight))
    if corrupt is not None:
        wp, wsf = corrupt(wp, wsf)
    y, *_ = oracle.linear(W.to_u16(x), wp, wsf, gsf_w, N, None, gsf_x=1.0)
    return float(np.linalg.norm(y - ref.numpy()) / np.linalg.norm(ref.numpy()))


@pytest.fixture(scope="module")
def probe_weight():
    g = torch.Generator().manual_seed(1002)
    return (torch.randn(1024, 5120, generator=g) * 0.02).to(torch.bfloat16)   # k_proj shape


def test_probe_error_is_about_013(oracle, probe_weight):
    fig = json.load(open(GOLDEN))["probe_noise"]
    err = probe(oracle, probe_weight, 256, seed=0)
    assert abs(err - fig["value"]) < 0.02, err
    assert err < fig["max_probe_error_default"]


def test_probe_negative_controls(oracle, probe_weight):
    fig = json.load(open(GOLDEN))["probe_noise"]
    N, K = probe_weight.shape

    def linear_layout(wp, wsf):            # scale bytes left in plain row-major order
        lin = oracle.scale_unswizzle(wsf, N, K)
        out = np.zeros_like(wsf)
        out[:lin.size] = lin.reshape(-1)
        return wp, out

    def swap_nibbles(wp, wsf):
        return ((wp >> 4) | (wp << 4)).astype(np.uint8), wsf

    def zero(wp, wsf):
        return np.zeros_like(wp), wsf

    good = probe(oracle, probe_weight, 64, seed=1)
    wrong = probe(oracle, probe_weight, 64, seed=1, corrupt=linear_layout)
    swapped = probe(oracle, probe_weight, 64, seed=1, corrupt=swap_nibbles)
    zeroed = probe(oracle, probe_weight, 64, seed=1, corrupt=zero)
    assert good < 0.16
    assert wrong > 2.5 * good
    assert swapped > 1.2
    assert zeroed == fig["wrong_layout"]
