"""Pins for the oracle's quantizer: global scale, block encoding, packing, the
128x4 scale layout and the byte counts the pages print.

Brute force here means: for each block, search all 127 finite E4M3 scales and
all 16 E2M1 codes by their decoded values (decoded by torch / ml_dtypes, not by
the oracle), so the oracle's bisection and nearest-value loops are checked
against an exhaustive search on the same fp32 intermediate values.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_17_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")
E4M3_VALUES = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()                     # codes 0x00..0x7E
E2M1_VALUES = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def nearest_even(values: np.ndarray, v: float) -> int:
    """Index of the nearest value; an exact tie takes the even index."""
    d = np.abs(values - v)
    best = np.flatnonzero(d == d.min())
    even = [i for i in best if i % 2 == 0]
    return int(even[0] if even else best[0])


def brute_force_block(xf: np.ndarray, gsf: np.float32):
    """(scale byte, 16 codes) for one block by exhaustive search (R3 order)."""
    bmax = np.float32(np.max(np.abs(xf)))
    s_raw = np.float32(np.float32(gsf * bmax) / np.float32(6.0))
    s8 = 0x7E if s_raw >= 448.0 else nearest_even(E4M3_VALUES, float(s_raw))
    s = np.float32(E4M3_VALUES[s8])
    if s == 0:
        return s8, [0] * 16
    inv = np.float32(gsf / s)
    codes = []
    for v in xf:
        q = np.float32(v * inv)
        mag = min(abs(float(q)), 6.0)
        c = nearest_even(E2M1_VALUES[:8], mag)
        codes.append(c | (8 if np.signbit(q) else 0))
    return s8, codes


def bf16_rows(x: torch.Tensor) -> np.ndarray:
    return W.to_u16(x)


@pytest.mark.parametrize("case", ["normal", "outliers", "tiny", "huge", "zeros", "static_overflow"])
def test_block_quantize_brute_force(oracle, case):
    g = torch.Generator().manual_seed(7)
    R, K = 6, 64
    x = torch.randn(R, K, generator=g)
    if case == "outliers":
        x[torch.rand(R, K, generator=g) < 0.05] *= 40
    elif case == "tiny":
        x *= 1e-6
    elif case == "huge":
        x *= 1e4
    elif case == "zeros":
        x[:, 16:32] = 0
        x[2] = 0
    xb = x.to(torch.bfloat16)
    xu = bf16_rows(xb)
    amax = float(xb.float().abs().max())
    gsf = np.float32(2688.0) / np.float32(max(amax, 1e-12))
    if case == "static_overflow":          # calibrated amax below the data: saturation
        gsf = np.float32(gsf * np.float32(8.0))
    packed, sf_lin = oracle.quantize_rows(xu, float(gsf))
    xf = xb.float().numpy()
    for r in range(R):
        for j in range(K // 16):
            s8, codes = brute_force_block(xf[r, 16 * j:16 * j + 16], gsf)
            assert sf_lin[r, j] == s8, (r, j)
            got = packed[r, 8 * j:8 * j + 8]
            want = [codes[2 * i] | (codes[2 * i + 1] << 4) for i in range(8)]
            assert list(got) == want, (r, j)


def test_global_scale_closed_form(oracle):
    assert oracle.global_scale(2688.0) == 1.0
    assert oracle.global_scale(1.0) == 2688.0
    assert oracle.global_scale(448.0) == 6.0
    assert oracle.global_scale(0.0) == float(np.float32(2688.0) / np.float32(1e-12))
    x = W.random_bf16((33, 48), seed=3)
    assert oracle.amax_bf16(W.to_u16(x)) == float(x.float().abs().max())


def test_dynamic_scale_top_block_hits_448(oracle):
    """With the dynamic scale the block holding the tensor's amax gets s_raw = 448
    (up to one rounding) and its largest element the code for 6."""
    x = W.random_bf16((4, 128), seed=11)
    xu = W.to_u16(x)
    packed, sf, gsf = oracle.quantize(xu)
    xf = x.float().numpy()
    r, k = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    sf_lin = oracle.scale_unswizzle(sf, 4, 128)
    assert sf_lin[r, k // 16] == 0x7E                   # 448
    code = (packed[r, k // 2] >> (4 * (k % 2))) & 0xF
    assert code & 7 == 7


def test_all_zero_tensor(oracle):
    x = np.zeros((3, 32), dtype=np.uint16)
    packed, sf, gsf = oracle.quantize(x)
    assert not packed.any() and not sf.any()
    assert gsf == oracle.global_scale(0.0)


def test_nibble_order_even_element_low(oracle):
    """R5: element 2i in bits 0..3, element 2i+1 in bits 4..7."""
    x = torch.zeros(1, 16)
    x[0, 0], x[0, 1] = 6.0, -0.5        # with gsf such that the scale decodes to 1
    gsf = np.float32(1.0)
    packed, sf_lin = oracle.quantize_rows(W.to_u16(x.to(torch.bfloat16)), float(gsf))
    assert sf_lin[0, 0] == 0x38         # 6/6 = 1.0
    assert packed[0, 0] == (7 | (9 << 4))


def scale_layout_by_reshape(sf_lin: np.ndarray, R: int, K: int) -> np.ndarray:
    """The 128x4 layout restated as a tensor permutation of the padded
    [Rp, Cp] matrix: (Rp/128, 4, 32, Cp/4, 4) -> (Rp/128, Cp/4, 32, 4, 4)."""
    Rp, Cp = (R + 127) // 128 * 128, (K // 16 + 3) // 4 * 4
    padded = np.zeros((Rp, Cp), dtype=np.uint8)
    padded[:R, :K // 16] = sf_lin
    t = padded.reshape(Rp // 128, 4, 32, Cp // 4, 4).transpose(0, 3, 2, 1, 4)
    return t.reshape(-1)


@pytest.mark.parametrize("R,K", [(1, 16), (128, 64), (129, 80), (300, 1024), (5, 48), (256, 256)])
def test_scale_layout(oracle, R, K):
    rng = np.random.default_rng(R * 1000 + K)
    sf_lin = rng.integers(1, 255, size=(R, K // 16), dtype=np.uint8)
    sw = oracle.scale_swizzle(sf_lin, R, K)
    assert sw.size == oracle.scale_bytes(R, K)
    assert np.array_equal(sw, scale_layout_by_reshape(sf_lin, R, K))
    assert np.array_equal(oracle.scale_unswizzle(sw, R, K), sf_lin)
    offs = {oracle.scale_offset(r, c, K) for r in range(R) for c in range(K // 16)}
    assert len(offs) == R * (K // 16)                       # injective on the data
    assert int((sw == 0).sum()) == sw.size - R * (K // 16)  # the rest is zero padding


def test_byte_counts_match_pages(oracle):
    """50 Qwen3-VL layers: 24.4B values, 12.2 GB packed, 1.5 GB scales, 48.8 GB bf16;
    about 4.5 bits per weight, about 3.6x smaller than bf16."""
    fig = json.load(open(GOLDEN))
    shapes = fig["qwen3_vl_32b_layer_shapes"]["shapes"]
    tb = fig["text_encoder_bytes"]
    per_layer = sum(n * k for _, n, k in shapes)
    assert round(per_layer / 1e6, 1) == tb["values_per_layer"] / 1e6
    total = tb["layers"] * per_layer
    assert round(total / 1e9, 1) == tb["values_total"] / 1e9
    packed = tb["layers"] * sum(n * (k // 2) for _, n, k in shapes)
    scales = tb["layers"] * sum(oracle.scale_bytes(n, k) for _, n, k in shapes)
    assert round(packed / 1e9, 1) == tb["packed_gb"]
    assert round(scales / 1e9, 1) == tb["scales_gb"]
    assert round(total * 2 / 1e9, 1) == tb["bf16_gb"]
    bpw = fig["bits_per_weight"]
    assert (packed + scales) * 8 / total == pytest.approx(bpw["value"], abs=0.01)
    assert round(16 / bpw["value"], 1) == bpw["ratio_vs_bf16"]
