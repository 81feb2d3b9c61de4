"""The C ABI library without a GPU: it loads, exports every symbol the header
declares, computes sizes on the host, and rejects bad arguments before touching
the device (the checks mirror "minimax_h3_nvfp4_decoder" -- NVFP4DecoderLinear.
__init__ / from_packed and "convert_minimax_h3_text_encoder_nvfp4.py" --
quantize_language_linear).  No compute call runs here.
"""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_17_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")
A = ctypes.c_void_p(1 << 20)          # a 16-byte aligned address that is never dereferenced
MIS = ctypes.c_void_p((1 << 20) + 4)  # a misaligned one
S = ctypes.c_void_p(None)


@pytest.fixture(scope="module")
def L():
    from nvfp4_block_scaled_17_b200 import _build
    _build.build()
    return nv.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(nv.SIGNATURES), "binding and header disagree"
    assert L.nvfp4_abi_version() == 1


def test_status_strings(L):
    for code, name in nv.STATUS.items():
        assert L.nvfp4_status_string(code).decode() == name


def test_sizes_match_oracle(L, oracle):
    for rows, K in [(1, 16), (128, 256), (129, 80), (32768, 1024), (5120, 25600), (25600, 5120)]:
        assert L.nvfp4_scale_bytes(rows, K) == oracle.scale_bytes(rows, K)
        assert L.nvfp4_packed_bytes(rows, K) == rows * K // 2
    assert L.nvfp4_scale_bytes(0, 64) == 0 and L.nvfp4_scale_bytes(5, 0) == 0
    assert L.nvfp4_quantize_workspace_bytes() >= 1024 * 4
    ws = L.nvfp4_linear_workspace_bytes(4096, 5120)
    assert ws >= 4096 * 5120 // 2 + oracle.scale_bytes(4096, 5120) + 8
    assert ws % 256 == 0
    # prepared weight scales: one 4 KiB block per 256-row block and 256-value K stage
    assert L.nvfp4_prepared_scale_bytes(5120, 5120) == 20 * 20 * 4096
    assert L.nvfp4_prepared_scale_bytes(300, 576) == 2 * 3 * 4096
    assert L.nvfp4_prepared_scale_bytes(0, 64) == 0 and L.nvfp4_prepared_scale_bytes(8, 48) == 0


def test_quantize_argument_errors(L):
    q = L.nvfp4_quantize
    assert q(None, 4, 64, 0, A, A, A, A, None, None, A, 4096, S) == nv.ERR_INVALID_ARG
    assert q(A, -1, 64, 0, A, A, A, A, None, None, A, 4096, S) == nv.ERR_INVALID_ARG
    assert q(A, 4, 64, 8, A, A, A, A, None, None, A, 4096, S) == nv.ERR_INVALID_ARG      # group 8
    assert q(A, 4, 64, 0, None, None, A, A, None, None, A, 4096, S) == nv.ERR_INVALID_ARG  # no scale at all
    assert q(A, 4, 24, 0, A, A, A, A, None, None, A, 4096, S) == nv.ERR_SHAPE            # K % 16
    assert q(A, 4, 0, 0, A, A, A, A, None, None, A, 4096, S) == nv.ERR_SHAPE
    assert q(A, 4, 96, 64, A, A, A, A, None, None, A, 4096, S) == nv.ERR_SHAPE           # K % group
    assert q(MIS, 4, 64, 0, A, A, A, A, None, None, A, 4096, S) == nv.ERR_ALIGN
    assert q(A, 4, 64, 0, None, A, A, A, None, None, None, 0, S) == nv.ERR_WORKSPACE     # dynamic, no scratch
    assert q(A, 4, 64, 0, None, A, A, A, None, None, A, 16, S) == nv.ERR_WORKSPACE
    assert q(A, 4, 64, 0, A, A, A, A, A, None, None, 0, S) == nv.ERR_INVALID_ARG  # gsf_w alone


def test_gemm_and_linear_argument_errors(L):
    g = L.nvfp4_gemm
    assert g(A, A, A, A, A, None, A, 4, 4, 48, S) == nv.ERR_SHAPE             # K % 64
    assert g(A, A, A, A, None, None, A, 4, 4, 64, S) == nv.ERR_INVALID_ARG    # no alpha
    assert g(A, A, A, A, A, None, A, -1, 4, 64, S) == nv.ERR_INVALID_ARG
    assert g(A, A, MIS, A, A, None, A, 4, 4, 64, S) == nv.ERR_ALIGN
    lin = L.nvfp4_linear
    assert lin(A, 4, 64, A, A, A, 8, None, None, 0, A, 16, A, S) == nv.ERR_WORKSPACE
    assert lin(A, 4, 96, A, A, A, 8, None, None, 0, A, 1 << 20, A, S) == nv.ERR_SHAPE
    assert lin(A, 4, 128, A, A, A, 8, None, None, 48, A, 1 << 20, A, S) == nv.ERR_INVALID_ARG
    assert lin(A, 4, 128, A, A, None, 8, None, None, 0, A, 1 << 20, A, S) == nv.ERR_INVALID_ARG
    gq = L.nvfp4_gemm_quantize_out
    assert gq(A, A, A, A, A, None, A, A, A, 4, 96, 64, S) == nv.ERR_SHAPE      # N % 64
    assert gq(A, A, A, A, A, None, None, A, A, 4, 64, 64, S) == nv.ERR_INVALID_ARG
    assert gq(A, A, A, A, A, None, A, MIS, A, 4, 64, 64, S) == nv.ERR_ALIGN
    dq = L.nvfp4_dequantize
    assert dq(None, A, A, 4, 64, A, S) == nv.ERR_INVALID_ARG
    assert dq(A, A, A, 4, 24, A, S) == nv.ERR_SHAPE
    assert dq(A, A, A, -1, 64, A, S) == nv.ERR_INVALID_ARG
    assert dq(A, A, A, 4, 64, MIS, S) == nv.ERR_ALIGN
    fx = L.nvfp4_linear_fixed_scratch
    assert fx(A, 16384, 1024, A, A, A, 8, None, None, 0, A, S) == nv.ERR_WORKSPACE  # > 8 MiB
    assert fx(A, 4, 96, A, A, A, 8, None, None, 0, A, S) == nv.ERR_SHAPE
    assert fx(A, 4, 128, A, A, None, 8, None, None, 0, A, S) == nv.ERR_INVALID_ARG
    h = L.hadamard_rotate
    assert h(A, A, 4, 64, 0, S) == nv.ERR_INVALID_ARG
    assert h(A, A, 4, 96, 64, S) == nv.ERR_SHAPE
    gp = L.nvfp4_gemm_prepared
    assert gp(A, A, A, A, A, None, A, 4, 4, 48, S) == nv.ERR_SHAPE            # K % 64
    assert gp(A, A, A, None, A, None, A, 4, 4, 64, S) == nv.ERR_INVALID_ARG   # no B scales
    assert gp(A, A, A, MIS, A, None, A, 4, 4, 64, S) == nv.ERR_ALIGN
    pw = L.nvfp4_prepare_weight_scales
    assert pw(None, 256, 64, A, S) == nv.ERR_INVALID_ARG
    assert pw(A, -1, 64, A, S) == nv.ERR_INVALID_ARG
    assert pw(A, 256, 96, A, S) == nv.ERR_SHAPE
    assert pw(A, 256, 64, MIS, S) == nv.ERR_ALIGN
    df = L.nvfp4_debug_gemm_f32
    assert df(A, A, A, A, 0, A, None, A, 4, 4, 48, S) == nv.ERR_SHAPE         # K % 64
    assert df(A, A, A, A, 2, A, None, A, 4, 4, 64, S) == nv.ERR_INVALID_ARG   # prepared flag
    assert df(A, A, A, A, 1, None, None, A, 4, 4, 64, S) == nv.ERR_INVALID_ARG
    assert df(A, A, A, A, 0, A, None, MIS, 4, 4, 64, S) == nv.ERR_ALIGN
    lp = L.nvfp4_linear_prepared
    assert lp(A, 4, 64, A, A, A, 8, None, None, 0, A, 16, A, S) == nv.ERR_WORKSPACE
    assert lp(A, 4, 96, A, A, A, 8, None, None, 0, A, 1 << 20, A, S) == nv.ERR_SHAPE


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly(L):
    st = L.nvfp4_gemm(A, A, A, A, A, None, A, 4, 4, 64, S)
    assert st in (nv.ERR_CUDA, nv.ERR_DEVICE)
