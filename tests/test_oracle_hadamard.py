"""Pins for the oracle's block Hadamard rotation.

"minimax_h3_nvfp4_decoder" (module docstring, from_linear): a block Hadamard
rotation, orthonormal and symmetric, folded into the weight along the input
dimension and applied to the activation at run time, exact in full precision:
y = x W^T = (x H)(W H)^T.  The reading is the Sylvester matrix scaled by
1/sqrt(g), which scipy.linalg.hadamard builds independently.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

from nvfp4_block_scaled_17_b200 import workloads as W

GROUPS = (16, 32, 64, 128)


@pytest.mark.parametrize("g", GROUPS)
def test_rotation_equals_scipy_hadamard_exactly(oracle, g):
    """Small-integer inputs make every butterfly sum exact in fp32, so the only
    roundings are the one multiply by rn(1/sqrt(g)) and the bf16 rounding; the
    result must then equal scipy's H_g applied in exact arithmetic, bit for bit.
    A wrong sign, index or stage order fails this."""
    rng = np.random.default_rng(g)
    R, K = 7, 2 * g
    xi = rng.integers(-8, 9, size=(R, K)).astype(np.float32)
    x = torch.from_numpy(xi).to(torch.bfloat16)
    y = oracle.hadamard_rotate(W.to_u16(x), g)
    H = scipy.linalg.hadamard(g).astype(np.float64)
    c = np.float32(1.0 / np.sqrt(g))
    assert oracle.hadamard_scale(g) == float(c)
    exact = np.concatenate([xi[:, j:j + g].astype(np.float64) @ H for j in range(0, K, g)], axis=1)
    want = torch.from_numpy((exact.astype(np.float32) * c).astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(y, W.to_u16(want))


def test_scipy_hadamard_is_orthonormal_and_symmetric():
    for g in GROUPS:
        H = scipy.linalg.hadamard(g) / np.sqrt(g)
        assert np.allclose(H @ H, np.eye(g), atol=1e-14)
        assert np.array_equal(H, H.T)


@pytest.mark.parametrize("g", GROUPS)
def test_fold_invariant(oracle, g):
    """rot(x) rot(W)^T = x W^T.  In fp64 with the exact H the identity holds to
    rounding; through the oracle (fp32 butterfly, bf16 outputs) it holds to the
    bf16 rounding of the two rotated operands."""
    x = W.random_bf16((64, 4 * g), seed=100 + g)
    w = W.random_bf16((48, 4 * g), seed=200 + g, std=0.02)
    H = scipy.linalg.hadamard(g) / np.sqrt(g)
    Hb = np.kron(np.eye(4), H)
    xf, wf = x.double().numpy(), w.double().numpy()
    ref = xf @ wf.T
    assert np.linalg.norm((xf @ Hb) @ (wf @ Hb).T - ref) / np.linalg.norm(ref) < 1e-12
    xr = W.from_u16(oracle.hadamard_rotate(W.to_u16(x), g)).double().numpy()
    wr = W.from_u16(oracle.hadamard_rotate(W.to_u16(w), g)).double().numpy()
    rel = np.linalg.norm(xr @ wr.T - ref) / np.linalg.norm(ref)
    assert rel < 4e-3
    # and the oracle's rotation is H applied to each group up to bf16 rounding
    assert np.allclose(xr, xf @ Hb, rtol=2 ** -8, atol=1e-30)


def test_rotation_spreads_an_outlier(oracle):
    """One large entry in a group becomes g entries of magnitude |v|/sqrt(g)."""
    g = 128
    x = torch.zeros(1, g)
    x[0, 5] = 64.0
    y = W.from_u16(oracle.hadamard_rotate(W.to_u16(x.to(torch.bfloat16)), g)).float()
    assert torch.allclose(y.abs(), torch.full((1, g), 64.0 / np.sqrt(g)), rtol=2 ** -8)
