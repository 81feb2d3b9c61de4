"""Seeded synthetic inputs for the NVFP4 W4A4 linear.

This module draws random tensors with the shapes and value distributions of
the pages' workloads and holds none of the method's arithmetic: no scale, no
rounding to FP4/FP8, no rotation.  It is shared by the tests, the smoke check
and ``bench.py``; both the CUDA path and the CPU oracle receive its tensors.

Workloads (shapes from the pages):
  * tiny      -- x [128, 256] ~ N(0,1) with exactly 1% of entries x20, W [256, 256]
                 ~ N(0, 0.02), bias [256] ~ N(0, 0.01); seed 0.
  * vit_block -- one H3 ViT decoder block with 8 spatial tiles of 4096 tokens batched
                 ("minimax_h3_nvfp4_decoder" and the tile-batch change "decode
                 dynamic-scale NVFP4 H3 VAE tiles one at a time"): x [32768, 1024]
                 ~ N(0,1) with 0.5% of entries x30; qkv [3072,1024], attn-out
                 [1024,1024], FFN-in [4096,1024], FFN-out [1024,4096] ~ N(0,0.02);
                 biases ~ N(0,0.01); FFN-out input [32768, 4096] drawn the same way.
  * qwen3_layer -- one Qwen3-VL-32B text-encoder layer ("convert_minimax_h3_text_
                 encoder_nvfp4.py": 487.6M values per layer): q [8192,5120], k/v
                 [1024,5120], o [5120,8192], gate/up [25600,5120], down [5120,25600];
                 W ~ N(0,0.02); x [512, K] ~ N(0,1); no bias.
  * down_proj_swiglu -- x = silu(a)*b with a, b ~ 0.5*Student-t(3), [4096, 25600];
                 W [5120, 25600] ~ N(0,0.02).
  * m_sweep   -- K = N = 5120, M in {16, 128, 1024, 8192, 65536}.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

BF16 = torch.bfloat16


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * std


def with_outliers(shape, frac: float, factor: float, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) fp32 with exactly round(frac * numel) entries, chosen by a seeded
    permutation, multiplied by ``factor``; returned as bf16."""
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    n = x.numel()
    k = int(round(frac * n))
    if k:
        idx = torch.randperm(n, generator=gen, device=device)[:k]
        x.view(-1)[idx] *= factor
    return x.to(BF16)


def student_t(shape, df: int, gen: torch.Generator, device) -> torch.Tensor:
    """Student-t(df) as z / sqrt(chi2_df / df) from df+1 independent normals."""
    z = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(df):
        e = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
        chi2 += e * e
    return z / torch.sqrt(chi2 / df)


def swiglu_input(shape, gen: torch.Generator, device) -> torch.Tensor:
    a = 0.5 * student_t(shape, 3, gen, device)
    b = 0.5 * student_t(shape, 3, gen, device)
    return (torch.nn.functional.silu(a) * b).to(BF16)


@dataclass
class Linear:
    name: str
    N: int
    K: int
    weight: torch.Tensor          # bf16 [N, K] (not rotated)
    bias: torch.Tensor | None     # bf16 [N] or None
    x: torch.Tensor               # bf16 [M, K]


def tiny(device="cpu", seed: int = 0) -> Linear:
    g = _gen(seed, device)
    x = with_outliers((128, 256), 0.01, 20.0, g, device)
    w = normal((256, 256), 0.02, g, device).to(BF16)
    b = normal((256,), 0.01, g, device).to(BF16)
    return Linear("tiny", 256, 256, w, b, x)


VIT_SHAPES = (("qkv", 3072, 1024), ("attn_out", 1024, 1024), ("ffn_in", 4096, 1024),
              ("ffn_out", 1024, 4096))


def vit_block(device="cpu", seed: int = 1001, tokens: int = 8 * 4096,
              shared_x: bool = False) -> list[Linear]:
    """The four block linears.  Each gets its own input of the right width drawn
    from the same outlier distribution (``shared_x`` reuses one [M,1024] input for
    the three K=1024 linears)."""
    g = _gen(seed, device)
    out = []
    x1024 = with_outliers((tokens, 1024), 0.005, 30.0, g, device) if shared_x else None
    for name, N, K in VIT_SHAPES:
        w = normal((N, K), 0.02, g, device).to(BF16)
        b = normal((N,), 0.01, g, device).to(BF16)
        if shared_x and K == 1024:
            x = x1024
        else:
            x = with_outliers((tokens, K), 0.005, 30.0, g, device)
        out.append(Linear(name, N, K, w, b, x))
    return out


QWEN3_SHAPES = (("q_proj", 8192, 5120), ("k_proj", 1024, 5120), ("v_proj", 1024, 5120),
                ("o_proj", 5120, 8192), ("gate_proj", 25600, 5120), ("up_proj", 25600, 5120),
                ("down_proj", 5120, 25600))


def qwen3_weight(shape, device, gen) -> torch.Tensor:
    return normal(shape, 0.02, gen, device).to(BF16)


def qwen3_layer(device="cpu", seed: int = 1002, M: int = 512) -> list[Linear]:
    g = _gen(seed, device)
    out = []
    for name, N, K in QWEN3_SHAPES:
        w = qwen3_weight((N, K), device, g)
        x = normal((M, K), 1.0, g, device).to(BF16)
        out.append(Linear(name, N, K, w, None, x))
    return out


def down_proj_swiglu(device="cpu", seed: int = 1003, M: int = 4096) -> Linear:
    g = _gen(seed, device)
    x = swiglu_input((M, 25600), g, device)
    w = normal((5120, 25600), 0.02, g, device).to(BF16)
    return Linear("down_proj", 5120, 25600, w, None, x)


M_SWEEP = (16, 128, 1024, 8192, 65536)


def m_sweep(M: int, device="cpu", seed: int = 1004) -> Linear:
    g = _gen(seed + M, device)
    w = normal((5120, 5120), 0.02, g, device).to(BF16)
    x = normal((M, 5120), 1.0, g, device).to(BF16)
    return Linear(f"m{M}", 5120, 5120, w, None, x)


def random_bf16(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    return normal(shape, std, _gen(seed, device), device).to(BF16)


def to_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_u16(a, device="cpu") -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(BF16).to(device)
