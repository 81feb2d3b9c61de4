"""GPU parity of the block-scaled FP4 GEMM and of the whole linear against the
fp64 oracle over the same dequantized operands, through the C ABI.

Bound: relative Frobenius error <= 2e-3 and max-abs error <= 1e-2 * rms(y) (+ one
bf16 ulp of the reference for the bf16 output).  Pages: "minimax_h3_nvfp4_decoder"
-- nvfp4_linear_inference (mm_fp4 with alpha = 1/(gsf_x*gsf_w), then the bias);
"convert_minimax_h3_text_encoder_nvfp4.py" -- probe_relative_error (W4A4 error about
0.13 on random N(0,1) rows with a unit activation scale).
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import assert_gemm_close, assert_gemm_strict, rounds_to, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def t(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    pick = {0, M - 1, min(127, M - 1), min(128, M - 1)}
    pick |= set(rng.integers(0, M, size=max(n - len(pick), 0)).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def run_gemm_case(oracle, M, N, K, bias: bool, seed: int, rows=None, cols=None):
    """GPU GEMM against the fp64 oracle on the rows `rows` (all when None) x all columns,
    and, when `cols` is given, also on all rows x the columns `cols`.  The column check
    runs the oracle on the transposed product: y^T[cols] = alpha deq(w[cols]) deq(x)^T,
    then adds the bias of those columns."""
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(seed, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(seed + 1, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(seed + 2, "cpu"), "cpu").to(torch.bfloat16) if bias else None
    xp, xsf, gx = oracle.quantize(W.to_u16(x))
    wp, wsf, gw = oracle.quantize(W.to_u16(w))
    al = oracle.alpha(gx, gw)
    y = nv.nvfp4_gemm(t(xp), t(xsf), t(wp), t(wsf), torch.tensor([al], device=DEV),
                      None if b is None else b.to(DEV), M, N, K)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    y64 = oracle.gemm_f64(xp, xsf, wp, wsf, M, N, K, al, None if b is None else W.to_u16(b),
                          rows=rows)
    yg = y if rows is None else y[torch.from_numpy(rows).to(DEV)]
    out = assert_gemm_close(yg, y64, f"gemm M={M} N={N} K={K}")
    if cols is not None:
        yt64 = oracle.gemm_f64(wp, wsf, xp, xsf, N, M, K, al, None, rows=cols)
        if b is not None:
            yt64 = yt64 + b.float().numpy().astype(np.float64)[cols][:, None]
        yc = y[:, torch.from_numpy(cols).to(DEV)].t().contiguous()
        assert_gemm_close(yc, yt64, f"gemm M={M} N={N} K={K}, all rows x {len(cols)} columns")
    return out


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 256),          # the tiny linear
    (1, 8, 64), (2, 16, 64), (100, 200, 192), (129, 300, 320), (257, 513, 1024),
    (300, 640, 576), (64, 128, 128), (256, 1000, 512), (384, 256, 2048),
])
@pytest.mark.parametrize("bias", [True, False])
def test_gemm_parity(oracle, M, N, K, bias):
    run_gemm_case(oracle, M, N, K, bias, seed=M * 31 + N * 7 + K)


@pytest.mark.parametrize("M,N,K,rows,cols", [
    (16, 5120, 5120, None, None),     # the M-sweep's decode shapes: 20 tiles on 148 SMs
    (128, 5120, 5120, 24, None),
    (7, 2050, 768, None, None),       # N % 4 != 0: element-wise stores of the reduced rows
    (1, 64, 4096, None, None),
    (130, 520, 1536, None, None),     # two row blocks, ragged N and M
    # one full wave plus a short second one of long tiles: the full wave runs
    # persistent, the leftover tiles split K (160 = 148 + 12 and 162 = 148 + 14 tiles)
    (1024, 5120, 5120, 192, 192),
    (1152, 4608, 4096, 128, 128),
])
def test_gemm_split_k(oracle, M, N, K, rows, cols):
    """Grids with at most half as many tiles as SMs split K over a cluster of CTAs and
    reduce the partial tiles over distributed shared memory; so does the short last
    wave of a larger grid."""
    sel = None if rows is None else sample_rows(M, rows, seed=M + N)
    csel = None if cols is None else sample_rows(N, cols, seed=N + K)
    run_gemm_case(oracle, M, N, K, bias=True, seed=M * 13 + N + K, rows=sel, cols=csel)


@pytest.mark.parametrize("prepared", [False, True], ids=["128x4", "prepared"])
@pytest.mark.parametrize("M,N,K", [
    (128, 256, 256), (1, 8, 64), (100, 200, 192), (129, 300, 320), (257, 513, 1024),
    (384, 256, 2048),
    (16, 5120, 5120), (7, 2050, 768), (130, 520, 1536),     # split-K over a cluster
    (1024, 5120, 5120),                                     # full wave + split last wave
    (2048, 3072, 1024),                                     # persistent, several waves
])
def test_gemm_f32_strict(oracle, M, N, K, prepared):
    """The unrounded output of the same GEMM (nvfp4_debug_gemm_f32) within both stated
    bounds without widening, and the bf16 output of nvfp4_gemm / nvfp4_gemm_prepared
    equal to it rounded to nearest even."""
    seed = M * 17 + N * 3 + K
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(seed, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(seed + 1, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(seed + 2, "cpu"), "cpu").to(torch.bfloat16)
    xp, xsf, gx = oracle.quantize(W.to_u16(x))
    wp, wsf, gw = oracle.quantize(W.to_u16(w))
    al = oracle.alpha(gx, gw)
    alpha = torch.tensor([al], device=DEV)
    wsf_d = t(wsf)
    if prepared:
        wsf_d = nv.prepare_weight_scales(wsf_d, N, K)
        y = nv.nvfp4_gemm_prepared(t(xp), t(xsf), t(wp), wsf_d, alpha, b.to(DEV), M, N, K)
    else:
        y = nv.nvfp4_gemm(t(xp), t(xsf), t(wp), wsf_d, alpha, b.to(DEV), M, N, K)
    y32 = nv.nvfp4_debug_gemm_f32(t(xp), t(xsf), t(wp), wsf_d, alpha, b.to(DEV), M, N, K,
                                  prepared=prepared)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert rounds_to(y32, y)
    rows = None if M <= 256 else sample_rows(M, 256, seed=M)
    y64 = oracle.gemm_f64(xp, xsf, wp, wsf, M, N, K, al, W.to_u16(b), rows=rows)
    yg = y32 if rows is None else y32[torch.from_numpy(rows).to(DEV)]
    assert_gemm_strict(yg, y64, f"gemm {M}x{N}x{K} {'prepared' if prepared else '128x4'}")


def test_gemm_split_k_deterministic_and_graph_capturable():
    """The split-K reduction adds the partial tiles in a fixed order, so repeated calls
    agree bit for bit; the call also replays from a CUDA graph with the same result."""
    M, N, K = 16, 5120, 5120
    g = torch.Generator(device="cpu").manual_seed(11)
    xp = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8).to(DEV)
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8).to(DEV)
    # scale bytes 0x30..0x3f (E4M3 0.5 .. 0.94): finite, positive
    xsf = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(M, K),), generator=g)).to(torch.uint8).to(DEV)
    wsf = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(N, K),), generator=g)).to(torch.uint8).to(DEV)
    al = torch.tensor([1e-3], device=DEV)
    bias = (torch.randn(N, generator=g) * 0.01).to(torch.bfloat16).to(DEV)
    y1 = nv.nvfp4_gemm(xp, xsf, wp, wsf, al, bias, M, N, K)
    y2 = nv.nvfp4_gemm(xp, xsf, wp, wsf, al, bias, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    y3 = torch.empty_like(y1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        nv.nvfp4_gemm(xp, xsf, wp, wsf, al, bias, M, N, K, out=y3)   # warm-up on the stream
        torch.cuda.synchronize()
        y3.zero_()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            nv.nvfp4_gemm(xp, xsf, wp, wsf, al, bias, M, N, K, out=y3)
    graph.replay()
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))
    del graph


def test_gemm_vit_qkv_full_size(oracle):
    """ViT block qkv projection: [32768, 1024] x [3072, 1024]^T, 256 sampled rows x all
    columns and all rows x 256 sampled columns."""
    run_gemm_case(oracle, 32768, 3072, 1024, True, seed=11, rows=sample_rows(32768, 256),
                  cols=sample_rows(3072, 256, seed=5))


def test_gemm_down_proj_full_size(oracle):
    """Qwen3-VL down_proj shape with the full K = 25600: [4096, 25600] x [5120, 25600]^T,
    256 sampled rows x all columns and all rows x 256 sampled columns."""
    run_gemm_case(oracle, 4096, 5120, 25600, False, seed=13, rows=sample_rows(4096, 256),
                  cols=sample_rows(5120, 256, seed=7))


def test_gemm_zero_sizes():
    z = torch.zeros(16, dtype=torch.uint8, device=DEV)
    a = torch.tensor([1.0], device=DEV)
    y = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    L = nv.lib()
    assert L.nvfp4_gemm(nv._ptr(z), nv._ptr(z), nv._ptr(z), nv._ptr(z), nv._ptr(a), None,
                        nv._ptr(y), 0, 8, 64, nv._stream()) == nv.OK
    assert L.nvfp4_gemm(nv._ptr(z), nv._ptr(z), nv._ptr(z), nv._ptr(z), nv._ptr(a), None,
                        nv._ptr(y), 8, 0, 64, nv._stream()) == nv.OK


@pytest.mark.parametrize("group", [0, 16, 128])
@pytest.mark.parametrize("dynamic", [True, False])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 384, 512), (33, 96, 1024)])
def test_linear_parity(oracle, group, dynamic, M, N, K):
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(M + N + K, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(M + N + K + 1, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(M + N + K + 2, "cpu"), "cpu").to(torch.bfloat16)
    # weight: rotated (fold) and packed offline on the GPU, checked bit-exact first
    wr_u16 = oracle.hadamard_rotate(W.to_u16(w), group) if group else W.to_u16(w)
    wp, wsf, gw = nv.pack_weight(w.to(DEV), group)
    owp, owsf, ogw = oracle.quantize(wr_u16)
    assert np.array_equal(to_np(wp), owp) and np.array_equal(to_np(wsf), owsf)
    gsf_x = None
    if not dynamic:
        xr = oracle.hadamard_rotate(W.to_u16(x), group) if group else W.to_u16(x)
        gsf_x = oracle.global_scale(0.5 * oracle.amax_bf16(xr))      # calibrated too low: saturates
    y = nv.nvfp4_linear(x.to(DEV), wp, wsf, gw, N, bias=b.to(DEV),
                        gsf_x=None if gsf_x is None else torch.tensor([gsf_x], device=DEV),
                        rotate_group=group)
    torch.cuda.synchronize()
    y64, *_ = oracle.linear(W.to_u16(x), owp, owsf, ogw, N, W.to_u16(b), gsf_x=gsf_x,
                            rotate_group=group)
    assert_gemm_close(y, y64, f"linear g={group} dynamic={dynamic}")


def test_probe_error_on_gpu():
    """The pages' probe through the GPU path: about 0.13 against the bf16 product."""
    g = W._gen(1002, "cpu")
    w = W.normal((1024, 5120), 0.02, g, "cpu").to(torch.bfloat16).to(DEV)
    x = torch.randn(512, 5120, generator=W._gen(0, "cpu")).to(torch.bfloat16).to(DEV)
    wp, wsf, gw = nv.pack_weight(w)
    y = nv.nvfp4_linear(x, wp, wsf, gw, 1024, gsf_x=1.0)
    ref = (x.double() @ w.double().T)
    err = float((y.double() - ref).norm() / ref.norm())
    assert abs(err - 0.13) < 0.02, err


# ---------------------------------------------------------------------------
# prepared weight scales (nvfp4_prepare_weight_scales + nvfp4_gemm_prepared)
# ---------------------------------------------------------------------------

def prepared_layout_np(sf: np.ndarray, N: int, K: int) -> np.ndarray:
    """The prepared order written out from its definition in the header: per 256-row
    block nb and K stage s of 256 values a 4 KiB block; bytes h*2048 + j*512 .. +511 of
    it are the 128x4 chunk (row tile 2 nb + h, step 4 s + j), zero past N or K/64."""
    kc, tiles, nb = K // 64, (N + 127) // 128, (N + 255) // 256
    ks = (kc + 3) // 4
    chunks = sf.reshape(-1)[: tiles * kc * 512].reshape(tiles, kc, 512)   # [tile, k, 512]
    out = np.zeros((nb, ks, 2, 4, 512), dtype=np.uint8)
    for blk in range(nb):
        for h in range(2):
            t = 2 * blk + h
            if t >= tiles:
                continue
            for k in range(kc):
                out[blk, k // 4, h, k % 4] = chunks[t, k]
    return out.reshape(-1)


def random_operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    ap = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    bp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    sa = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(M, K),), generator=g,
                               dtype=torch.int32)).to(torch.uint8)
    sb = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(N, K),), generator=g,
                               dtype=torch.int32)).to(torch.uint8)
    bias = (torch.randn(N, generator=g) * 0.01).to(torch.bfloat16)
    return ap.to(DEV), sa.to(DEV), bp.to(DEV), sb.to(DEV), bias.to(DEV)


@pytest.mark.parametrize("N,K", [(256, 64), (300, 576), (5120, 5120), (1000, 512), (128, 1024)])
def test_prepare_weight_scales_layout(N, K):
    g = torch.Generator().manual_seed(N + K)
    sf = torch.randint(0, 256, (nv.nvfp4_scale_bytes(N, K),), generator=g,
                       dtype=torch.int32).to(torch.uint8)
    out = torch.full((nv.nvfp4_prepared_scale_bytes(N, K),), 0xAB, dtype=torch.uint8, device=DEV)
    nv.prepare_weight_scales(sf.to(DEV), N, K, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(out), prepared_layout_np(sf.numpy(), N, K))


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 256), (100, 200, 192), (129, 300, 320), (257, 513, 1024), (300, 640, 576),
    (384, 256, 2048), (16, 5120, 5120), (1024, 5120, 5120), (2048, 3072, 1024), (7, 2050, 768),
])
@pytest.mark.parametrize("bias", [True, False])
def test_gemm_prepared_bit_exact_with_128x4(M, N, K, bias):
    """Same operands, the weight scales in either order: identical bf16 outputs (the same
    bytes reach the same tensor-memory columns), through the persistent, split-K and
    split-last-wave schedules."""
    ap, sa, bp, sb, b = random_operands(M, N, K, M * 7 + N + K)
    al = torch.tensor([1e-3], device=DEV)
    b = b if bias else None
    y0 = nv.nvfp4_gemm(ap, sa, bp, sb, al, b, M, N, K)
    y1 = nv.nvfp4_gemm_prepared(ap, sa, bp, nv.prepare_weight_scales(sb, N, K), al, b, M, N, K)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_gemm_prepared_vit_qkv_full_size(oracle):
    """ViT qkv projection through the prepared weight scales against the fp64 oracle:
    256 sampled rows x all columns and all rows x 256 sampled columns."""
    M, N, K = 32768, 3072, 1024
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(21, "cpu"), "cpu")
    w = W.normal((N, K), 0.02, W._gen(22, "cpu"), "cpu").to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(23, "cpu"), "cpu").to(torch.bfloat16)
    xp, xsf, gx = oracle.quantize(W.to_u16(x))
    wp, wsf, gw = oracle.quantize(W.to_u16(w))
    al = oracle.alpha(gx, gw)
    y = nv.nvfp4_gemm_prepared(t(xp), t(xsf), t(wp), nv.prepare_weight_scales(t(wsf), N, K),
                               torch.tensor([al], device=DEV), b.to(DEV), M, N, K)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    rows = sample_rows(M, 256)
    y64 = oracle.gemm_f64(xp, xsf, wp, wsf, M, N, K, al, W.to_u16(b), rows=rows)
    assert_gemm_close(y[torch.from_numpy(rows).to(DEV)], y64, "prepared qkv rows")
    cols = sample_rows(N, 256, seed=9)
    yt64 = oracle.gemm_f64(wp, wsf, xp, xsf, N, M, K, al, None, rows=cols)
    yt64 = yt64 + b.float().numpy().astype(np.float64)[cols][:, None]
    assert_gemm_close(y[:, torch.from_numpy(cols).to(DEV)].t().contiguous(), yt64,
                      "prepared qkv columns")


@pytest.mark.parametrize("group,dynamic", [(0, True), (128, True), (16, False)])
def test_linear_prepared_bit_exact(group, dynamic):
    M, N, K = 200, 384, 512
    x = W.with_outliers((M, K), 0.005, 30.0, W._gen(31 + group, DEV), DEV)
    w = W.normal((N, K), 0.02, W._gen(32, DEV), DEV).to(torch.bfloat16)
    b = W.normal((N,), 0.01, W._gen(33, DEV), DEV).to(torch.bfloat16)
    wp, wsf, gw = nv.pack_weight(w, group)
    gx = None if dynamic else 37.5
    y0 = nv.nvfp4_linear(x, wp, wsf, gw, N, b, gx, group)
    y1 = nv.nvfp4_linear(x, wp, nv.prepare_weight_scales(wsf, N, K), gw, N, b, gx, group,
                         prepared=True)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(16, 5120, 5120), (128, 5120, 5120), (512, 8192, 1024)])
def test_linear_sees_weights_written_just_before(M, N, K):
    """The linear's GEMM starts loading the weights before it waits for the activation
    quantizer, which is safe only because the quantizer itself waits for all earlier
    work.  Overwrite the weight buffers with another weight on the same stream, with no
    synchronisation, and call the linear right after: the result must be the second
    weight's, bit for bit (swapped-operand, split-K and persistent GEMM builds)."""
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(M + 7, DEV), DEV)
    w1 = W.normal((N, K), 0.02, W._gen(N + 8, DEV), DEV).to(torch.bfloat16)
    w2 = W.normal((N, K), 0.05, W._gen(N + 9, DEV), DEV).to(torch.bfloat16)
    wp2, wsf2, gw2 = nv.pack_weight(w2, 0)
    ref = nv.nvfp4_linear(x, wp2, wsf2, gw2, N)
    torch.cuda.synchronize()
    wp, wsf, gw = nv.pack_weight(w1, 0)
    y1 = nv.nvfp4_linear(x, wp, wsf, gw, N)
    nv.nvfp4_quantize(w2, 0, None, out=(wp, wsf, gw))   # the same buffers, no sync
    y2 = nv.nvfp4_linear(x, wp, wsf, gw, N)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert not torch.equal(y1.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), ref.view(torch.int16))
