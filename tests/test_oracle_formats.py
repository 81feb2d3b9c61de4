"""Pins for the oracle's number formats (E2M1, E4M3, bf16 rounding).

Each check ties the oracle to something outside it: the bit-field definitions
of the formats, the ml_dtypes and torch casts (library routines), and the
magnitudes the pages print ("FastH3-QAD-v2 and NVFP4 VAE Decoders": 4-bit values
with a shared FP8 scale; "minimax_h3_nvfp4_decoder": E4M3 block scales).
"""
import ml_dtypes
import numpy as np
import pytest
import torch


def e2m1_from_fields(code: int) -> float:
    """E2M1: sign s, exponent e (2 bits, bias 1), mantissa m (1 bit)."""
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1 + m / 2)
    return -mag if s else mag


def test_e2m1_decode_matches_bitfields_and_pages(oracle):
    mags = [oracle.e2m1_decode(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        assert oracle.e2m1_decode(c) == e2m1_from_fields(c)
        assert np.signbit(oracle.e2m1_decode(c)) == bool(c & 8)


def test_e2m1_roundtrip_every_code(oracle):
    for c in range(16):
        v = oracle.e2m1_decode(c)
        v = -0.0 if c == 8 else v
        assert oracle.e2m1_encode(v) == c


def test_e2m1_ties_round_to_even(oracle):
    # midpoints between neighbouring magnitudes and the code they must take
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert oracle.e2m1_encode(v) == c
        assert oracle.e2m1_encode(-v) == c | 8
    assert oracle.e2m1_encode(6.5) == 7 and oracle.e2m1_encode(1e30) == 7
    assert oracle.e2m1_encode(float("inf")) == 7
    assert oracle.e2m1_encode(-0.1) == 8 and oracle.e2m1_encode(-0.0) == 8


def _fp32_sweep(seed=0, n_random=1 << 20):
    """fp32 bit patterns: every upper-20-bit prefix with a few low-bit endings,
    plus random patterns and every multiple of 1/256 in [-8, 8]."""
    hi = np.arange(1 << 20, dtype=np.uint32) << 12
    lows = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    pats = (hi[:, None] | lows[None, :]).reshape(-1)
    rng = np.random.default_rng(seed)
    pats = np.concatenate([pats, rng.integers(0, 1 << 32, n_random, dtype=np.uint64).astype(np.uint32)])
    v = pats.view(np.float32)
    v = v[np.isfinite(v)]
    grid = (np.arange(-8 * 256, 8 * 256 + 1) / 256.0).astype(np.float32)
    return np.concatenate([v, grid])


def test_e2m1_encode_matches_ml_dtypes(oracle):
    v = _fp32_sweep()
    ours = oracle.e2m1_encode_array(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first {v[bad[:5]]}: {ours[bad[:5]]} vs {ref[bad[:5]]}"


def test_e4m3_decode_matches_torch(oracle):
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_decode(i) for i in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2      # 0x7F, 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_roundtrip_every_finite_code(oracle):
    for b in range(0x7F):
        assert oracle.e4m3_encode(oracle.e4m3_decode(b)) == b


def test_e4m3_encode_matches_torch_in_range(oracle):
    v = np.abs(_fp32_sweep(seed=1))
    v = v[v <= 448.0]
    ours = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first {v[bad[:5]]}"


def test_e4m3_saturation_and_underflow(oracle):
    # satfinite: everything above 448 (where torch would give NaN) is 448 = 0x7E
    for v in (448.0, 449.0, 464.0, 480.0, 1e6, 3.0e38, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
    # subnormal grid 2^-9; the tie at 2^-10 goes to the even code 0
    assert oracle.e4m3_encode(2.0 ** -10) == 0
    assert oracle.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 1
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 2          # tie between codes 1 and 2
    assert oracle.e4m3_encode(0.0) == 0


def test_bf16_rounding_matches_torch(oracle):
    v = _fp32_sweep(seed=2, n_random=1 << 18)
    ours = oracle.f32_to_bf16_array(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    for h in (0x3F80, 0xC2F7, 0x0001, 0x7F7F):
        assert oracle.bf16_to_f32(h) == float(torch.tensor([h], dtype=torch.int32)
                                               .to(torch.int16).view(torch.bfloat16).float())
