"""Pins for the oracle's int8 per-row W8A8 linear ("FastH3-4-step-Preview-v1-r16-int8":
"What is inside" -- weight = round(W / scale) clamped to -127..127 with scale =
amax(|W[row]|) / 127, activations quantized per row at call time, int8 GEMM;
"Accuracy" -- 1.2 to 1.7 % mean and 2.7 % worst relative error on random rows).

* closed forms and round-half-to-even ties,
* an independent restatement with numpy (fp32 division, np.round, clip) and the integer
  GEMM by numpy int64 matmul,
* invariants: the row maximum maps to +-127, a zero row to zeros, the scheme halves the
  bf16 bytes (page: 42.4 GB -> 21.2 GB),
* the page's probe error band.
"""
import json
import os

import numpy as np
import pytest
import torch

from nvfp4_block_scaled_17_b200 import workloads as W

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def bf16(a):
    return W.to_u16(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16))


def test_closed_form_and_ties(oracle):
    # amax 127 -> scale 1: codes are round-half-even of the values themselves
    row = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -127.0] + [0.0] * 8], dtype=np.float32)
    q, s = oracle.int8_quantize_rows(bf16(row))
    assert s[0] == np.float32(1.0)
    assert q[0, :8].tolist() == [127, 2, 4, -2, 0, 0, 2, -127]


@pytest.mark.parametrize("R,K", [(1, 16), (9, 100), (64, 1024)])
def test_independent_restatement(oracle, R, K):
    x = W.with_outliers((R, K), 0.01, 20.0, W._gen(R * K, "cpu"), "cpu")
    xu = W.to_u16(x)
    q, s = oracle.int8_quantize_rows(xu)
    xf = W.from_u16(xu).float().numpy()
    s_ref = np.abs(xf).max(axis=1).astype(np.float32) / np.float32(127.0)
    assert np.array_equal(s, s_ref)
    q_ref = np.clip(np.round(xf / s_ref[:, None]), -127, 127).astype(np.int8)
    assert np.array_equal(q, q_ref)
    # every code is a nearest integer to x / s (within the clamp)
    err = np.abs(q.astype(np.float64) - xf.astype(np.float64) / s_ref[:, None].astype(np.float64))
    assert err.max() <= 0.5 + 1e-5       # the fp32 quotient carries a relative 2^-24


def test_row_max_zero_row_and_bytes(oracle):
    x = np.zeros((3, 32), dtype=np.float32)
    x[0, 5] = -3.0
    x[1, 7] = 1e-20
    q, s = oracle.int8_quantize_rows(bf16(x))
    assert q[0, 5] == -127 and q[1, 7] == 127
    assert s[2] == 0 and not q[2].any()
    g = GOLDEN["int8_scheme"]
    assert g["int8_bytes_gb"] == pytest.approx(g["bf16_bytes_of_seven_linears_gb"] / 2, rel=1e-3)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (17, 33, 96), (64, 40, 640)])
def test_gemm_restatement(oracle, M, N, K):
    rng = np.random.default_rng(M + N)
    qx = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    qw = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    sx = rng.random(M, dtype=np.float32) * 0.1
    sw = rng.random(N, dtype=np.float32) * 0.01
    b = bf16(rng.standard_normal(N))
    y = oracle.int8_gemm_f64(qx, sx, qw, sw, b)
    acc = qx.astype(np.int64) @ qw.astype(np.int64).T
    ref = acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64) \
        + W.from_u16(b).double().numpy()[None, :]
    assert np.allclose(y, ref, rtol=1e-14, atol=0)
    rows = np.array([M - 1, 0])
    assert np.array_equal(oracle.int8_gemm_f64(qx, sx, qw, sw, b, rows=rows), y[rows])


def test_probe_error_in_page_band(oracle):
    """Random N(0,1) rows against an N(0, 0.02) weight of a 5120-wide linear: the
    per-row int8 product's relative error sits in the page's 1.2-2.7 % band."""
    g = GOLDEN["int8_probe_error"]
    x = torch.randn(256, 5120, generator=W._gen(0, "cpu")).to(torch.bfloat16)
    w = W.normal((512, 5120), 0.02, W._gen(1, "cpu"), "cpu").to(torch.bfloat16)
    qx, sx = oracle.int8_quantize_rows(W.to_u16(x))
    qw, sw = oracle.int8_quantize_rows(W.to_u16(w))
    y = oracle.int8_gemm_f64(qx, sx, qw, sw)
    ref = (x.double() @ w.double().T).numpy()
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert g["mean_low"] * 0.8 <= rel <= g["worst"], rel
    # a wrong scale convention (amax / 255: codes saturate) leaves the band
    xf = W.from_u16(W.to_u16(x)).float().numpy()
    s_bad = (np.abs(xf).max(axis=1) / 255.0).astype(np.float32)
    q_bad = np.clip(np.round(xf / s_bad[:, None]), -127, 127).astype(np.int8)
    y_bad = oracle.int8_gemm_f64(q_bad, s_bad, qw, sw)
    assert np.linalg.norm(y_bad - ref) / np.linalg.norm(ref) > g["worst"]
