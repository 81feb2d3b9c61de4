"""GPU parity of the NVFP4 -> bf16 expansion (nvfp4_dequantize) against the oracle,
bit for bit, through the C ABI ("decode dynamic-scale NVFP4 H3 VAE tiles one at a
time" -- FASTVIDEO_H3_ENCODER_FUSED_DEQUANT)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def random_packed(rows, K, seed):
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, size=nv.nvfp4_scale_bytes(rows, K), dtype=np.uint8)
    return packed, sf


@pytest.mark.parametrize("rows,K", [(1, 16), (37, 80), (130, 256), (257, 1040), (64, 25600)])
@pytest.mark.parametrize("gsf", [1.0, 864.4824, 3.0e-4])
def test_dequantize_parity(oracle, rows, K, gsf):
    packed, sf = random_packed(rows, K, rows * K)
    g = torch.tensor([gsf], dtype=torch.float32, device=DEV)
    y = nv.nvfp4_dequantize(torch.from_numpy(packed).to(DEV), torch.from_numpy(sf).to(DEV), g, K)
    torch.cuda.synchronize()
    want = oracle.dequantize_bf16(packed, sf, rows, K, np.float32(gsf).item())
    got = W.to_u16(y)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:4]}: {got.reshape(-1)[bad[:4]]} vs {want.reshape(-1)[bad[:4]]}"


def test_round_trip_through_gpu_quantizer(oracle):
    """Weight as the converter stores it (quantized with its own dynamic scale), expanded
    back: bit-exact with the oracle's expansion of the same bytes."""
    w = W.qwen3_weight((1024, 5120), "cpu", W._gen(7, "cpu")).to(DEV)
    packed, sf, gsf = nv.nvfp4_quantize(w, 0, None)
    y = nv.nvfp4_dequantize(packed, sf, gsf, 5120)
    torch.cuda.synchronize()
    want = oracle.dequantize_bf16(to_np(packed), to_np(sf), 1024, 5120, float(gsf.item()))
    assert np.array_equal(W.to_u16(y), want)
    rel = ((y.float() - w.float()).norm() / w.float().norm()).item()
    assert rel < 0.15      # NVFP4 round-trip noise on Gaussian weights is about 0.1


def test_dequantize_full_size_weight(oracle):
    """A 5120 x 25600 projection (131 M values), checked on sampled rows."""
    rows, K = 5120, 25600
    packed, sf = random_packed(rows, K, 11)
    g = torch.tensor([1234.5], dtype=torch.float32, device=DEV)
    y = nv.nvfp4_dequantize(torch.from_numpy(packed).to(DEV), torch.from_numpy(sf).to(DEV), g, K)
    torch.cuda.synchronize()
    want = oracle.dequantize_bf16(packed, sf, rows, K, 1234.5)
    pick = np.array([0, 1, 127, 128, 2047, 4095, rows - 1])
    assert np.array_equal(W.to_u16(y)[pick], want[pick])
    assert np.array_equal(W.to_u16(y), want)


def test_zero_rows_and_errors():
    L = nv.lib()
    z = torch.zeros(64, dtype=torch.uint8, device=DEV)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    assert L.nvfp4_dequantize(nv._ptr(z), nv._ptr(z), nv._ptr(g), 0, 16, nv._ptr(z), None) == nv.OK
    assert L.nvfp4_dequantize(nv._ptr(z), nv._ptr(z), nv._ptr(g), 4, 24, nv._ptr(z), None) == nv.ERR_SHAPE
