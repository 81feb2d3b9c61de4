"""Helpers shared by the GPU parity tests (comparison rules only; no method
arithmetic).  The GEMM bound is the one stated for this path: relative
Frobenius error <= 2e-3 and max-abs error <= 1e-2 * rms(y), the latter widened by
one bf16 ulp of the reference because the output itself is bf16."""
import numpy as np
import torch

REL_FRO = 2e-3
MAX_ABS_RMS = 1e-2


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
    rel, rms, maxabs, excess = gemm_errors(y_gpu, y64)
    assert np.isfinite(y_gpu.float().cpu().numpy()).all(), f"{what}: non-finite output"
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert excess <= 0, f"{what}: max-abs {maxabs:.3e} exceeds 1e-2*rms ({rms:.3e}) + ulp"
    return rel, maxabs / max(rms, 1e-300)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
