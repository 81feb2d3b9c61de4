"""The GEMM whose epilogue emits the next linear's NVFP4 input (nvfp4_gemm_quantize_out),
through the C ABI ("minimax_h3_nvfp4_decoder" -- NVFP4FusedState / fused_state: static
global scale, no rotation; "FastH3-QAD-v2 and NVFP4 VAE Decoders" -- "Fused FP4
kernels": bit-exact with the unfused path).

* Against the oracle: operands quantized by the oracle; the expected encoding is the
  oracle's quantizer applied to its fp64 product rounded to bf16.  The GPU's bf16
  product can differ from that by one bf16 ulp (fp32 accumulation order), so scale
  bytes may differ by one E4M3 step and codes by one E2M1 step, on a small fraction.
* Against the unfused GPU path (nvfp4_gemm, then nvfp4_quantize of its bf16 output
  with the same static scale): bit for bit, the pages' own claim for their fused kernels.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6])


def t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def unpack(packed):
    return np.stack([packed & 15, packed >> 4], axis=-1).reshape(packed.shape[0], -1)


def operands(oracle, M, N, K, seed):
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(seed, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(seed + 1, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(seed + 2, "cpu"), "cpu").to(torch.bfloat16)
    xp, xsf, gx = oracle.quantize(W.to_u16(x))
    wp, wsf, gw = oracle.quantize(W.to_u16(w))
    return xp, xsf, wp, wsf, oracle.alpha(gx, gw), b


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 320, 128), (1, 64, 64),
                                   (257, 1024, 512), (130, 192, 1024)])
@pytest.mark.parametrize("bias", [True, False])
def test_fused_against_oracle(oracle, M, N, K, bias):
    xp, xsf, wp, wsf, al, b = operands(oracle, M, N, K, M + N + K)
    bu = W.to_u16(b) if bias else None
    y64 = oracle.gemm_f64(xp, xsf, wp, wsf, M, N, K, al, bu)
    y16 = oracle.f32_to_bf16_array(y64.astype(np.float32)).reshape(M, N)   # reference bf16 product
    g_out = oracle.global_scale(0.7 * float(np.abs(y64).max()))   # calibrated a bit low
    ref_p, ref_sf, _ = oracle.quantize(y16, gsf=g_out)
    gp, gsf_ = nv.nvfp4_gemm_quantize_out(
        t(xp), t(xsf), t(wp), t(wsf), torch.tensor([al], device=DEV), M, N, K,
        torch.tensor([g_out], device=DEV), bias=b.to(DEV) if bias else None)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    gp, gsf_ = to_np(gp), to_np(gsf_)
    # scale bytes: equal, or one E4M3 step apart where y differs by an ulp
    d = np.abs(gsf_.astype(int) - ref_sf.astype(int))
    assert d.max() <= 1 and (d == 0).mean() >= 0.98, (d.max(), (d == 0).mean())
    # codes: where the scale byte agrees, the value is within one E2M1 step
    cg, cr = unpack(gp), unpack(ref_p)
    same_scale = np.repeat(oracle.scale_unswizzle(gsf_, M, N) == oracle.scale_unswizzle(ref_sf, M, N),
                           16, axis=1)
    vg, vr = E2M1[cg], E2M1[cr]
    step = np.where(np.abs(vr) >= 4, 2.0, np.where(np.abs(vr) >= 2, 1.0, 0.5))
    assert np.all(np.abs(vg - vr)[same_scale] <= step[same_scale])
    assert (cg == cr).mean() >= 0.98


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (333, 640, 192), (4096, 4096, 1024)])
def test_fused_equals_unfused_gpu_path(oracle, M, N, K):
    xp, xsf, wp, wsf, al, b = operands(oracle, M, N, K, 7 * M + N)
    a_, sfa_, b_, sfb_ = t(xp), t(xsf), t(wp), t(wsf)
    alpha = torch.tensor([al], device=DEV)
    g_out = torch.tensor([40.0], device=DEV)
    y = nv.nvfp4_gemm(a_, sfa_, b_, sfb_, alpha, b.to(DEV), M, N, K)
    up, usf, _ = nv.nvfp4_quantize(y, 0, g_out)
    fp, fsf = nv.nvfp4_gemm_quantize_out(a_, sfa_, b_, sfb_, alpha, M, N, K, g_out, bias=b.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(fp, up)
    assert torch.equal(fsf, usf[:fsf.numel()])


def test_fused_vit_ffn_in_full_size(oracle):
    """FFN input projection of the ViT block at the 8-tile batch (32768 x 4096 x 1024),
    fused output against the unfused GPU path, bit for bit."""
    lin = W.vit_block("cpu")[2]
    M, N, K = lin.x.shape[0], lin.N, lin.K
    x = lin.x.to(DEV)
    wp, wsf, gw = nv.pack_weight(lin.weight.to(DEV), 0)
    xp, xsf, gx = nv.nvfp4_quantize(x, 0, None)
    alpha = 1.0 / (gx * gw)
    g_out = torch.tensor([30.0], device=DEV)
    y = nv.nvfp4_gemm(xp, xsf, wp, wsf, alpha, lin.bias.to(DEV), M, N, K)
    up, usf, _ = nv.nvfp4_quantize(y, 0, g_out)
    fp, fsf = nv.nvfp4_gemm_quantize_out(xp, xsf, wp, wsf, alpha, M, N, K, g_out,
                                         bias=lin.bias.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(fp, up) and torch.equal(fsf, usf[:fsf.numel()])
