"""GPU parity of the whole path on every workload of the pages, through the C ABI:
the packed weight and the quantized activation bit-exact against the CPU oracle, then
the linear's bf16 output and the GEMM's unrounded fp32 output against the fp64 oracle
over the same dequantized operands (bounds in gpu_util), and the bf16 output equal,
bit for bit, to the fp32 output rounded to nearest even.

Large outputs are compared on sampled rows x all columns and on all rows x sampled
columns; the quantizer is compared on every byte.

Workloads (seeded; nvfp4_block_scaled_17_b200.workloads):
  tiny        x [128, 256] with 1 % outliers x20, dynamic scale, bias, no rotation;
  ViT block   the four linears at 8 tiles x 4096 tokens, g = 128, dynamic and static
              scale ("minimax_h3_nvfp4_decoder" -- NVFP4DecoderLinear, rotate_activation;
              "decode dynamic-scale NVFP4 H3 VAE tiles one at a time" -- tile batching);
  Qwen3-VL    the seven projections of one text-encoder layer at M = 512, dynamic
              scale, no bias ("convert_minimax_h3_text_encoder_nvfp4.py" --
              quantize_language_linear);
  down_proj   SwiGLU input with Student-t(3) factors, [4096, 25600] x [5120, 25600],
              g in {none, 16, 128} ("convert_minimax_h3_text_encoder_nvfp4.py" -- the
              widest outliers; "minimax_h3_nvfp4_decoder" -- rotate_activation);
  M-sweep     K = N = 5120, M in {16, 128, 1024, 8192, 65536}, dynamic scale.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W
from gpu_util import assert_gemm_close, assert_gemm_strict, rounds_to, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample(n: int, k: int, seed: int) -> np.ndarray:
    """k distinct indices of range(n) including the first, the last and the row-block
    edges 127 / 128 (all of them when n <= k)."""
    if n <= k:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pick = {0, n - 1, min(127, n - 1), min(128, n - 1)}
    rest = rng.choice(np.setdiff1d(np.arange(n), list(pick)), size=k - len(pick), replace=False)
    return np.array(sorted(pick | set(rest.tolist())), dtype=np.int64)


def run_case(oracle, what, x, w, b, group, static, n_rows=256, n_cols=256, prepared=False):
    """x, w, b: bf16 tensors on the GPU (drawn by the seeded generators); the oracle gets
    host copies of the same tensors."""
    M, K = x.shape
    N = w.shape[0]
    bias_u16 = None if b is None else W.to_u16(b)

    # oracle: weight folded and packed, activation rotated and quantized, alpha
    wu, xu = W.to_u16(w), W.to_u16(x)
    wr = oracle.hadamard_rotate(wu, group) if group else wu
    owp, owsf, ogw = oracle.quantize(wr)
    xr = oracle.hadamard_rotate(xu, group) if group else xu
    gsf_x = oracle.global_scale(oracle.amax_bf16(xr)) if static else None
    oxp, oxsf, ogx = oracle.quantize(xr, gsf_x)
    al = oracle.alpha(ogx, ogw)

    # GPU: packing and quantization bit-exact
    wp, wsf, gw = nv.pack_weight(w, group)
    gx_in = None if gsf_x is None else torch.tensor([gsf_x], dtype=torch.float32, device=DEV)
    xp, xsf, gx = nv.nvfp4_quantize(x, group, gx_in)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(wp), owp), f"{what}: packed weight differs from the oracle"
    assert np.array_equal(to_np(wsf), owsf), f"{what}: weight scales differ from the oracle"
    assert np.float32(gw.item()) == np.float32(ogw)
    assert np.array_equal(to_np(xp), oxp), f"{what}: activation codes differ from the oracle"
    assert np.array_equal(to_np(xsf), oxsf), f"{what}: activation scales differ from the oracle"
    assert np.float32(gx.item()) == np.float32(ogx)

    # the linear (bf16) and the unrounded GEMM on the same operands
    wsf_use = nv.prepare_weight_scales(wsf, N, K) if prepared else wsf
    y = nv.nvfp4_linear(x, wp, wsf_use, gw, N, bias=b, gsf_x=gx_in, rotate_group=group,
                        prepared=prepared)
    y32 = nv.nvfp4_debug_gemm_f32(xp, xsf, wp, wsf_use,
                                  torch.tensor([al], dtype=torch.float32, device=DEV), b, M, N, K,
                                  prepared=prepared)
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert rounds_to(y32, y), f"{what}: bf16 output is not the fp32 output rounded"

    rows = sample(M, n_rows, seed=M + N)
    y64 = oracle.gemm_f64(oxp, oxsf, owp, owsf, M, N, K, al, bias_u16, rows=rows)
    ridx = torch.from_numpy(rows).to(DEV)
    assert_gemm_close(y[ridx], y64, f"{what} rows")
    assert_gemm_strict(y32[ridx], y64, f"{what} [{len(rows)} rows x {N}]")
    if M > n_rows:
        cols = sample(N, n_cols, seed=N + K)
        yt64 = oracle.gemm_f64(owp, owsf, oxp, oxsf, N, M, K, al, None, rows=cols)
        if b is not None:
            yt64 = yt64 + b.float().cpu().numpy().astype(np.float64)[cols][:, None]
        cidx = torch.from_numpy(cols).to(DEV)
        assert_gemm_close(y[:, cidx].t().contiguous(), yt64, f"{what} columns")
        assert_gemm_strict(y32[:, cidx].t().contiguous(), yt64, f"{what} [{M} x {len(cols)} cols]")


def test_tiny(oracle):
    lin = W.tiny(DEV)
    run_case(oracle, "tiny 128x256x256", lin.x, lin.weight, lin.bias, 0, False)


@pytest.fixture(scope="module")
def vit():
    return W.vit_block(DEV)


@pytest.mark.parametrize("static", [False, True], ids=["dynamic", "static"])
@pytest.mark.parametrize("idx", range(4), ids=[s[0] for s in W.VIT_SHAPES])
def test_vit_block(oracle, vit, idx, static):
    lin = vit[idx]
    run_case(oracle, f"ViT {lin.name} M={lin.x.shape[0]} g=128 {'static' if static else 'dynamic'}",
             lin.x, lin.weight, lin.bias, 128, static, prepared=not static)


@pytest.fixture(scope="module")
def qwen3():
    return W.qwen3_layer(DEV)


@pytest.mark.parametrize("idx", range(7), ids=[s[0] for s in W.QWEN3_SHAPES])
def test_qwen3_layer(oracle, qwen3, idx):
    lin = qwen3[idx]
    run_case(oracle, f"Qwen3-VL {lin.name} 512x{lin.N}x{lin.K}", lin.x, lin.weight, None, 0,
             False)


@pytest.fixture(scope="module")
def down_proj():
    return W.down_proj_swiglu(DEV)


@pytest.mark.parametrize("group", [0, 16, 128])
def test_down_proj_swiglu(oracle, down_proj, group):
    lin = down_proj
    run_case(oracle, f"down_proj SwiGLU 4096x5120x25600 g={group}", lin.x, lin.weight, None,
             group, False)


@pytest.mark.parametrize("M", W.M_SWEEP)
def test_m_sweep_linear(oracle, M):
    lin = W.m_sweep(M, DEV)
    run_case(oracle, f"M-sweep {M}x5120x5120", lin.x, lin.weight, None, 0, False,
             prepared=M >= 8192)
