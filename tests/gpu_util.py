"""Helpers shared by the GPU parity tests (comparison rules only; no method
arithmetic).

The GEMM bound is the one stated for this path: relative Frobenius error <= 2e-3
and max-abs error <= 1e-2 * rms(y), both against the fp64 oracle over the same
dequantized operands.
  * strict  -- both bounds as stated, applied to the GEMM's unrounded fp32 output
               (nvfp4_debug_gemm_f32: the same mainloop, no bf16 rounding);
  * bf16    -- the production output is bf16, whose own rounding is up to half an
               ulp of |y|; for it the max-abs bound is widened by one bf16 ulp of the
               reference value, element by element.
"""
import numpy as np
import torch

REL_FRO = 2e-3
MAX_ABS_RMS = 1e-2

# (what, relative Frobenius error, max-abs / rms) of every strict check that ran,
# printed at the end of the session (tests/conftest.py)
STRICT_RESULTS = []


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-300)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def gemm_errors(y_gpu: torch.Tensor, y64: np.ndarray):
    yg = y_gpu.detach().float().cpu().double().numpy()
    diff = np.abs(yg - y64)
    rel = float(np.linalg.norm(yg - y64) / max(np.linalg.norm(y64), 1e-300))
    rms = float(np.sqrt(np.mean(y64 ** 2)))
    excess = diff - (MAX_ABS_RMS * rms + bf16_ulp(y64))
    return rel, rms, float(diff.max()), float(excess.max())


def assert_gemm_close(y_gpu: torch.Tensor, y64: np.ndarray, what: str = ""):
    """The bf16-output bound: relative Frobenius as stated, max-abs widened by one bf16
    ulp of the reference per element."""
    rel, rms, maxabs, excess = gemm_errors(y_gpu, y64)
    assert np.isfinite(y_gpu.float().cpu().numpy()).all(), f"{what}: non-finite output"
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert excess <= 0, f"{what}: max-abs {maxabs:.3e} exceeds 1e-2*rms ({rms:.3e}) + ulp"
    return rel, maxabs / max(rms, 1e-300)


def assert_gemm_strict(y32: torch.Tensor, y64: np.ndarray, what: str = ""):
    """Both bounds as stated, no widening, on an fp32 output."""
    assert y32.dtype == torch.float32, "the strict bound applies to the unrounded fp32 output"
    yg = y32.detach().cpu().double().numpy()
    assert np.isfinite(yg).all(), f"{what}: non-finite output"
    rel = float(np.linalg.norm(yg - y64) / max(np.linalg.norm(y64), 1e-300))
    rms = float(np.sqrt(np.mean(y64 ** 2)))
    mar = float(np.abs(yg - y64).max() / max(rms, 1e-300))
    STRICT_RESULTS.append((what, rel, mar))
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mar <= MAX_ABS_RMS, f"{what}: max-abs / rms {mar:.3e} > {MAX_ABS_RMS}"
    return rel, mar


def rounds_to(y32: torch.Tensor, y16: torch.Tensor) -> bool:
    """True when the bf16 output is the fp32 output rounded to nearest even, bit for bit."""
    return torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
