"""GPU parity of the quantizer, the amax pass and the Hadamard rotation against
the CPU oracle, through the C ABI.  The bar is bit-exact: packed bytes, every
scale byte including the padding, and the global-scale bit pattern.

Pages: "minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference (dynamic scale, 128x4
layout), rotate_activation / from_linear (block Hadamard);
"convert_minimax_h3_text_encoder_nvfp4.py" -- quantize_language_linear.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_quantize(x: torch.Tensor, group: int, gsf, ws_bytes=None):
    """ws_bytes None: the binding's default workspace; otherwise a workspace of exactly
    that many bytes."""
    R, K = x.shape
    packed = torch.full((R, K // 2), 0xAB, dtype=torch.uint8, device=DEV)     # garbage first
    sf = torch.full((nv.nvfp4_scale_bytes(R, K),), 0xAB, dtype=torch.uint8, device=DEV)
    gsf_out = torch.full((1,), -7.0, dtype=torch.float32, device=DEV)
    g_in = None if gsf is None else torch.tensor([gsf], dtype=torch.float32, device=DEV)
    ws = None if ws_bytes is None else torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    nv.nvfp4_quantize(x, group, g_in, out=(packed, sf, gsf_out), workspace=ws)
    torch.cuda.synchronize()
    return to_np(packed), to_np(sf), np.float32(gsf_out.item())


def oracle_quantize(oracle, x: torch.Tensor, group: int, gsf):
    xu = W.to_u16(x)
    if group:
        xu = oracle.hadamard_rotate(xu, group)
    return oracle.quantize(xu, gsf)


def check(oracle, x, group, gsf, ws_bytes=None):
    p, s, g = gpu_quantize(x.to(DEV), group, gsf, ws_bytes)
    op, os_, og = oracle_quantize(oracle, x, group, gsf)
    assert np.float32(og).view(np.uint32) == g.view(np.uint32), (og, g)
    assert np.array_equal(s, os_), f"scale bytes differ at {np.flatnonzero(s != os_)[:8]}"
    bad = np.argwhere(p != op)
    assert bad.size == 0, f"{len(bad)} packed bytes differ, first {bad[:4].tolist()}"


SHAPES = [(1, 16), (7, 48), (128, 256), (129, 80), (300, 1024), (33, 1040), (256, 128), (5, 2048)]


@pytest.mark.parametrize("R,K", SHAPES)
@pytest.mark.parametrize("dynamic", [True, False])
def test_quantize_no_rotation(oracle, R, K, dynamic):
    x = W.with_outliers((R, K), 0.01, 20.0, W._gen(R * 7 + K, "cpu"), "cpu")
    gsf = None if dynamic else 2688.0 / 9.0
    check(oracle, x, 0, gsf)


@pytest.mark.parametrize("group", [16, 32, 64, 128])
@pytest.mark.parametrize("R,K", [(1, 128), (130, 256), (64, 1024), (3, 384)])
@pytest.mark.parametrize("dynamic", [True, False])
def test_quantize_rotated(oracle, group, R, K, dynamic):
    if K % group:
        pytest.skip("K % group")
    x = W.with_outliers((R, K), 0.005, 30.0, W._gen(R + K + group, "cpu"), "cpu")
    check(oracle, x, group, None if dynamic else 37.5)


def test_quantize_special_values(oracle):
    R, K = 130, 256
    x = torch.randn(R, K, generator=torch.Generator().manual_seed(5))
    x[0] = 0                                # all-zero row
    x[1, :16] = 0                           # all-zero block
    x[2] *= 1e-30                           # tiny values (scale underflow)
    x[3] *= 1e30                            # huge values
    x[4, 5] = -0.0
    x[5, :] = -1e-3                         # negative values rounding to zero codes
    x[6] *= 1e-38                           # subnormal bf16 values
    xb = x.to(torch.bfloat16)
    check(oracle, xb, 0, None)
    for g in (16, 64, 128):                 # the rotation on the same rows
        check(oracle, xb, g, None)
        check(oracle, xb, g, 1.0)
    check(oracle, xb, 0, 1.0)               # unit scale (the pages' probe)
    check(oracle, xb, 0, 1e6)               # static scale far too large: saturation
    check(oracle, torch.zeros(3, 64, dtype=torch.bfloat16), 0, None)


def test_quantize_vit_block_full_size(oracle):
    """The 8-tile ViT-decoder activation [32768, 1024], g = 128, dynamic and static."""
    lin = W.vit_block("cpu")[0]
    check(oracle, lin.x, 128, None)
    amax = float(oracle.amax_bf16(oracle.hadamard_rotate(W.to_u16(lin.x), 128)))
    check(oracle, lin.x, 128, oracle.global_scale(amax))
    check(oracle, lin.x, 0, None)


def test_weight_pack_qwen_shape(oracle):
    """Offline weight packing of one Qwen3-VL projection shape ([1024, 5120])."""
    w = W.qwen3_weight((1024, 5120), "cpu", W._gen(3, "cpu"))
    check(oracle, w, 0, None)


@pytest.mark.parametrize("group", [16, 32, 64, 128])
@pytest.mark.parametrize("R,K", [(1, 128), (129, 256), (64, 2048)])
def test_hadamard_rotate(oracle, group, R, K):
    x = W.random_bf16((R, K), seed=R * K + group)
    y = nv.hadamard_rotate(x.to(DEV), group)
    want = oracle.hadamard_rotate(W.to_u16(x), group)
    assert np.array_equal(W.to_u16(y), want)
    # in place
    xi = x.to(DEV).clone()
    nv.hadamard_rotate(xi, group, out=xi)
    assert np.array_equal(W.to_u16(xi), want)


def test_format_conversions_exhaustive(oracle):
    """The quantizer's device fp32 -> E2M1 and fp32 -> E4M3 conversions, and its
    block-scale step E4M3(rn(y / 6)), against the oracle's encoders (the quotient
    rounded by IEEE fp32 division) on all 2^32 fp32 bit patterns (NaNs excluded)."""
    n = 1 << 26
    e2 = torch.empty(n, dtype=torch.uint8, device=DEV)
    e4 = torch.empty(n, dtype=torch.uint8, device=DEV)
    sc = torch.empty(n, dtype=torch.uint8, device=DEV)
    L = nv.lib()
    for chunk in range(1 << 6):
        first = chunk * n
        assert L.nvfp4_debug_cvt_sweep(first, n, nv._ptr(e2), nv._ptr(e4), nv._ptr(sc),
                                       nv._stream()) == nv.OK
        v = (np.arange(n, dtype=np.uint32) + np.uint32(first)).view(np.float32)
        keep = ~np.isnan(v)
        vk = v[keep]
        g2, g4 = to_np(e2)[keep], to_np(e4)[keep]
        o2 = oracle.e2m1_encode_array(vk)
        bad2 = np.flatnonzero(g2 != o2)
        assert bad2.size == 0, f"E2M1 differs for {vk[bad2[:6]]}: {g2[bad2[:6]]} vs {o2[bad2[:6]]}"
        if first < (1 << 31):                 # E4M3 of |v|: the positive half covers it
            o4 = oracle.e4m3_encode_array(vk)
            bad4 = np.flatnonzero(g4 != o4)
            assert bad4.size == 0, f"E4M3 differs for {vk[bad4[:6]]}: {g4[bad4[:6]]} vs {o4[bad4[:6]]}"
            os_ = oracle.e4m3_encode_array(vk / np.float32(6.0))
            gs = to_np(sc)[keep]
            bads = np.flatnonzero(gs != os_)
            assert bads.size == 0, f"scale differs for {vk[bads[:6]]}: {gs[bads[:6]]} vs {os_[bads[:6]]}"


@pytest.mark.parametrize("group", [0, 128])
@pytest.mark.parametrize("rows", [4096, 14208, 14336])
def test_dynamic_streaming_sizes(oracle, group, rows):
    """Dynamic-scale calls of 4.2-14.7 M values run the streaming passes (g = 0: amax and
    encode phases in one cooperative kernel; g = 128: the amax pass, then the encode pass
    walking the items in reverse).  Bit for bit against the oracle."""
    K = 1024
    x = W.with_outliers((rows, K), 0.005, 30.0, W._gen(rows + group, "cpu"), "cpu")
    p, sf, g = nv.nvfp4_quantize(x.to(DEV), group, None)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    xr = oracle.hadamard_rotate(W.to_u16(x), group) if group else W.to_u16(x)
    op, osf, og = oracle.quantize(xr)
    assert float(g.item()) == og
    assert np.array_equal(to_np(p), op) and np.array_equal(to_np(sf), osf)


@pytest.mark.parametrize("group", [0, 16, 128])
@pytest.mark.parametrize("rows", [1, 47, 48, 49, 100])
def test_dynamic_single_pass_edge(oracle, group, rows):
    """A dynamic call of at most 12 items of 32 units (48 x 1024: 384 units) runs the
    one-CTA single pass, one item per warp; 49 rows need a 13th item and take the
    streaming passes (half-unit kernels for g <= 64).  Both bit for bit against the
    oracle."""
    K = 1024
    x = W.with_outliers((rows, K), 0.01, 20.0, W._gen(rows * 5 + group, "cpu"), "cpu")
    check(oracle, x, group, None)


@pytest.mark.parametrize("group", [16, 32, 64, 128])
def test_dynamic_two_pass_rotated(oracle, group):
    """A dynamic call of 16384 x 1024 (16.8 M values) runs the amax pass, then the encode
    pass (half-unit kernels for g <= 64, whole-unit ones for g = 128).  The amax pass stops before the last butterfly stage,
    keeps max(|a| + |b|) of its operand pairs, and scales and rounds that maximum once;
    the global scale must still equal the oracle's bit for bit."""
    rows, K = 16384, 1024
    x = W.with_outliers((rows, K), 0.005, 30.0, W._gen(rows * 3 + group, "cpu"), "cpu")
    check(oracle, x, group, None)


@pytest.mark.parametrize("sign", [1.0, -1.0])
@pytest.mark.parametrize("group,R,K", [(32, 3, 96), (32, 257, 160),
                                       (16, 3, 256), (32, 130, 256), (64, 3, 256), (128, 257, 256)])
def test_dynamic_amax_last_stage_branch(oracle, sign, group, R, K):
    """The largest rotated value comes out of the last stage's sum (sign +1) or its
    difference (sign -1): a g-group [1, 0 x (g/2 - 1), sign, 0 x (g/2 - 1)] gives halves of
    all ones and all `sign` before the last stage, so a + b or a - b is 2 and the other is
    0.  K % 128 != 0 runs the lane-pair kernels, K % 128 == 0 the one-thread-per-unit
    kernels; both take max(|a| + |b|) before the last stage in the amax pass."""
    g = torch.Generator().manual_seed(int(K + 10 * sign + group))
    x = torch.randn(R, K, generator=g) * 1e-3
    x[1, group] = 1.0
    x[1, group + group // 2] = sign
    xb = x.to(torch.bfloat16)
    check(oracle, xb, group, None)
    # the same rows repeated to 14.7 M values: the streaming route, amax pass then encode
    # pass, many items per warp
    if K % 128 == 0:
        rows = 14_700_000 // K + 1
        big = xb.repeat(rows // R + 1, 1)[:rows].contiguous()
        check(oracle, big, group, None)
