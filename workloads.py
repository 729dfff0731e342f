"""Seeded synthetic inputs for the FP4 quantization + block-scaled GEMM path.

This module only draws random tensors.  It holds none of the quantization
arithmetic, so both the CPU oracle (``oracle/``) and the CUDA path
(``fp4_quantization_block_b200``) can take their inputs from it without sharing
any of the method's code.

Workloads (all bf16, row-major, contiguous):

* ``tiny``: X[256, 512] ~ N(0, 1), seed 0.
* ``sweep``: 0.5 * Student-t(nu=3) with 1% of the columns scaled by 50.
  The Student-t draw is Z / sqrt(chi2_3 / 3), where chi2_3 is the sum of three
  squared normals from the same generator; a seeded permutation picks the
  outlier columns.
* ``act``: activations X ~ N(0, 1) with 0.5% of the channels scaled by 20
  (Llama-3-8B-shaped linear inputs).
* ``weight``: W[Cout, Cin] ~ N(0, 0.02).
* ``grad``: dY[T, Cout] = N(0, 1e-3) times a per-row lognormal(0, 1) factor.

Every generator takes a ``device`` so that large benchmark inputs can be drawn
directly in device memory; parity tests draw on the CPU and copy.
"""
from __future__ import annotations

import math

import torch

# Llama-3-8B-shaped linears: name -> (Cin, Cout); 8192 tokens per step.
LLAMA8B_LINEARS = {
    "qkv": (4096, 6144),
    "o": (4096, 4096),
    "gate_up": (4096, 28672),
    "down": (14336, 4096),
}
LLAMA8B_TOKENS = 8192
SWEEP_SHAPES = [(4096, 4096), (8192, 4096), (8192, 14336)]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def tiny(seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(256, 512, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def normal(rows: int, cols: int, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def _outlier_columns(cols: int, frac: float, seed: int) -> torch.Tensor:
    n = max(1, int(round(cols * frac)))
    g = _gen(seed + 7919, "cpu")
    return torch.randperm(cols, generator=g)[:n]


def sweep(rows: int, cols: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """0.5 * t_3 values with 1% outlier columns x50."""
    g = _gen(seed, device)
    z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(3):
        n = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(n, n)
    x = z.div_(torch.sqrt(chi2.div_(3.0))).mul_(0.5)
    del chi2
    cols_idx = _outlier_columns(cols, 0.01, seed).to(device)
    x[:, cols_idx] *= 50.0
    return x.to(torch.bfloat16)


def act(tokens: int, channels: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """N(0,1) activations with 0.5% outlier channels x20."""
    g = _gen(seed, device)
    x = torch.randn(tokens, channels, generator=g, device=device, dtype=torch.float32)
    cols_idx = _outlier_columns(channels, 0.005, seed).to(device)
    x[:, cols_idx] *= 20.0
    return x.to(torch.bfloat16)


def weight(cout: int, cin: int, seed: int = 0, device="cpu") -> torch.Tensor:
    return normal(cout, cin, seed, std=0.02, device=device)


def grad(tokens: int, cout: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """dY rows: N(0, 1e-3) times a lognormal(0, 1) factor per row."""
    g = _gen(seed, device)
    x = torch.randn(tokens, cout, generator=g, device=device, dtype=torch.float32).mul_(1e-3)
    row = torch.randn(tokens, 1, generator=g, device=device, dtype=torch.float32).exp_()
    return x.mul_(row).to(torch.bfloat16)


def with_specials(x: torch.Tensor, seed: int = 0) -> torch.Tensor:
    """Plant edge cases into a bf16 tensor: an all-zero block row segment,
    signed zeros, bf16 extremes and subnormals, exact E2M1 ties after scaling.

    Returns a copy; the input is unchanged.
    """
    y = x.clone()
    rows, cols = y.shape
    g = _gen(seed + 104729, "cpu")
    # a run of zeros long enough to cover a 32-wide block somewhere
    r = int(torch.randint(0, rows, (1,), generator=g))
    y[r, 0:64] = 0.0
    # negative zeros
    r2 = (r + 1) % rows
    y[r2, 0:32] = -0.0
    # bf16 extremes on one block
    r3 = (r + 2) % rows
    big = torch.tensor([3.3895313892515355e38, -3.3895313892515355e38], dtype=torch.float32)
    y[r3, 32:34] = big.to(torch.bfloat16)
    # bf16 subnormals on one block
    r4 = (r + 3) % rows
    y[r4, 64:96] = torch.full((32,), 9.183549615799121e-41, dtype=torch.float32).to(torch.bfloat16)
    # small integers: scaled values hit E2M1 grid points and midpoints
    r5 = (r + 4) % rows
    vals = torch.tensor([8.0, 0.5, 1.0, 1.5, 2.5, 3.0, 3.5, 5.0, 7.0, 0.25, 0.75, 1.25,
                         1.75, 6.0, 4.0, 2.0], dtype=torch.float32)
    y[r5, 0:16] = vals.to(torch.bfloat16)
    y[r5, 16:32] = (-vals).to(torch.bfloat16)
    return y


def ragged_like(rows: int, cols: int, seed: int) -> torch.Tensor:
    return normal(rows, cols, seed)


def llama8b_stack_flops_per_token() -> float:
    """Linear-layer FLOPs per token of one Llama-3-8B-shaped block, fwd only."""
    return sum(2.0 * cin * cout for cin, cout in LLAMA8B_LINEARS.values())


def describe() -> dict:
    return {
        "tiny": "X[256,512] ~ N(0,1), seed 0",
        "sweep": "0.5*t_3 (t_3 = Z/sqrt(chi2_3/3)), 1% columns x50, seeded permutation",
        "act": "N(0,1), 0.5% channels x20",
        "weight": "N(0,0.02)",
        "grad": "N(0,1e-3) x lognormal(0,1) per row",
    }


assert math.isclose(llama8b_stack_flops_per_token(), 2 * (4096 * 6144 + 4096 * 4096 + 4096 * 28672 + 14336 * 4096))
