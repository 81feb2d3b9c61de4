"""GPU parity of the int8 per-row W8A8 linear against the oracle, through the C ABI
("FastH3-4-step-Preview-v1-r16-int8" -- "What is inside" and "Accuracy").

Quantizer: bit for bit (codes and fp32 row scales).  GEMM: the integer accumulator is
exact on both sides, so every output may differ from the oracle's fp64 value only by the
final bf16 rounding plus a few fp32 roundings of the scaling: |y - y64| <= one bf16 ulp of
y64 + 1e-6 * rms(y64), element by element.  The probe error against the bf16 product sits
in the page's band.
"""
import json
import os

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import bf16_ulp, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def assert_int8_close(y_gpu, y64, what):
    yg = y_gpu.float().cpu().double().numpy()
    bound = bf16_ulp(y64) + 1e-6 * np.sqrt(np.mean(y64 ** 2))
    excess = np.abs(yg - y64) - bound
    assert np.isfinite(yg).all(), what
    assert excess.max() <= 0, f"{what}: worst excess {excess.max():.3e} over one bf16 ulp"


@pytest.mark.parametrize("R,K", [(1, 16), (37, 80), (130, 1024), (512, 5120), (3, 25600)])
def test_quantize_rows_parity(oracle, R, K):
    x = W.with_outliers((R, K), 0.01, 20.0, W._gen(R + K, "cpu"), "cpu")
    if R > 2:
        x[1] = 0.0                                       # a zero row
        x[2, :16] = torch.tensor([127, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -127] * 2)   # ties
    q, s = nv.int8_quantize_rows(x.to(DEV))
    torch.cuda.synchronize()
    oq, os_ = oracle.int8_quantize_rows(W.to_u16(x))
    assert np.array_equal(to_np(q), oq)
    assert np.array_equal(to_np(s)[:R], os_)


def test_quantize_rows_every_bf16_value(oracle):
    """Each row holds every finite bf16 value up to its own maximum (the row's amax), so
    the per-value division x / s is checked, bit for bit against the oracle, for all bf16
    inputs under 48 different row scales (powers of two, wide range, subnormal scales)."""
    allv = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    allv = allv[torch.isfinite(allv)]
    rng = np.random.default_rng(5)
    amaxes = [1.0, 2.0, 0.5, 127.0, 448.0, 3.0, 1e-3, 6.5e4, 1.5e-30, 2.9e30, 1e-37, 3e-39] + \
        [float(v) for v in (10.0 ** rng.uniform(-6, 6, size=36))]
    rows = []
    for am in amaxes:
        am = float(torch.tensor(am).to(torch.bfloat16).float())
        keep = allv[allv.abs() <= am]
        row = torch.cat([torch.tensor([am]), keep])
        pad = (-row.numel()) % 16
        rows.append(torch.cat([row, torch.zeros(pad)]))
    K = max(r.numel() for r in rows)
    x = torch.zeros(len(rows), K)
    for i, r in enumerate(rows):
        x[i, :r.numel()] = r
    x = x.to(torch.bfloat16)
    q, s = nv.int8_quantize_rows(x.to(DEV))
    torch.cuda.synchronize()
    oq, os_ = oracle.int8_quantize_rows(W.to_u16(x))
    assert np.array_equal(to_np(s)[:len(rows)], os_)
    bad = np.argwhere(to_np(q) != oq)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:3]}"


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 8, 32), (100, 200, 96), (257, 513, 1024),
                                   (300, 640, 5120)])
@pytest.mark.parametrize("bias", [True, False])
def test_gemm_parity(oracle, M, N, K, bias):
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(M * 3 + K, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(N + K, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(N, "cpu"), "cpu").to(torch.bfloat16) if bias else None
    qx, sx = oracle.int8_quantize_rows(W.to_u16(x))
    qw, sw = oracle.int8_quantize_rows(W.to_u16(w))
    y = nv.int8_gemm(t(qx), t(sx), t(qw), t(sw), None if b is None else b.to(DEV))
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    y64 = oracle.int8_gemm_f64(qx, sx, qw, sw, None if b is None else W.to_u16(b))
    assert_int8_close(y, y64, f"int8 gemm {M}x{N}x{K}")


def test_linear_full_shape_and_probe(oracle):
    """A 5120-wide linear (FFN-like 5120 -> 25600) on 512 random rows: the GPU linear
    against the oracle on sampled rows, and the probe error against the bf16 product in the
    page's band."""
    M, N, K = 512, 25600, 5120
    x = torch.randn(M, K, generator=W._gen(0, "cpu")).to(torch.bfloat16)
    w = W.normal((N, K), 0.02, W._gen(1, "cpu"), "cpu").to(torch.bfloat16)
    wq, sw = nv.int8_quantize_rows(w.to(DEV))
    y = nv.int8_linear(x.to(DEV), wq, sw)
    torch.cuda.synchronize()
    oq, os_ = oracle.int8_quantize_rows(W.to_u16(w))
    assert np.array_equal(to_np(wq), oq)
    qx, sx = oracle.int8_quantize_rows(W.to_u16(x))
    rows = np.array([0, 1, 255, 511])
    y64 = oracle.int8_gemm_f64(qx, sx, oq, os_, rows=rows)
    assert_int8_close(y[torch.from_numpy(rows).to(DEV)], y64, "int8 linear")
    ref = (x.to(DEV).float() @ w.to(DEV).float().T)
    rel = ((y.float() - ref).norm() / ref.norm()).item()
    g = GOLDEN["int8_probe_error"]
    assert g["mean_low"] * 0.8 <= rel <= g["worst"], rel
