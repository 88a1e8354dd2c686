"""Seeded synthetic inputs shaped like a 27B-class hybrid layer.

This module holds random draws only -- none of the method's arithmetic -- and
is the one module both the CUDA path's tests/benchmark and the CPU oracle's
tests take inputs from.  Every tensor is drawn with a ``torch.Generator``
seeded explicitly; the same seed on the same device gives the same bytes.
Both sides of a parity check always consume the identical bytes (the oracle
gets a host copy), so the device the draw runs on does not matter.

Recipes (shapes from the pages' model: hidden size 5120, the Gated DeltaNet
input projection q/k/v/z plus the a/b gate projections, an MLP of width
17408; the pages report GDN inputs as outlier-laden as attention inputs,
max/RMS 63.5 and kurtosis ~1,564 -- evolve.pub review, Strengths, Table 2):

* heavy-tailed activations: Student-t with nu = 3, i.e. a standard normal
  divided by sqrt(chi2_3 / 3), plus 8 fixed outlier channels (the first 8 of
  a seeded permutation of the columns) scaled by 200; cast to BF16.
* weights: N(0, sigma) per module, cast to BF16.
* the tiny case: X ~ N(0, 1) with 1 % of entries times 50, W ~ N(0, 0.02),
  both rounded once to BF16.
* Gated DeltaNet decay-gate parameters per head: A ~ U(1, 16), A_log = log A;
  dt log-uniform in [1e-3, 1e-1], dt_bias its softplus preimage (FP32).
"""
from __future__ import annotations

import math

import torch

HIDDEN = 5120
MLP_WIDTH = 17408

# Fused GDN input projection: (name, rows, sigma).  The a/b gate projections
# have tiny widths and sigmas ~100x apart, so their global scales differ ~100x.
GDN_MODULES = (("q", 4096, 0.02), ("k", 4096, 0.02), ("v", 8192, 0.015),
               ("z", 8192, 0.015), ("b", 64, 0.2), ("a", 64, 0.002))
# The decode-shaped variant of the same projection with 32-wide gates.
GDN_MODULES_DECODE = (("q", 4096, 0.02), ("k", 4096, 0.02), ("v", 8192, 0.015),
                      ("z", 8192, 0.015), ("b", 32, 0.2), ("a", 32, 0.002))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def student_t_activations(rows: int, cols: int = HIDDEN, seed: int = 1,
                          outlier_seed: int = 2, n_outliers: int = 8,
                          outlier_scale: float = 200.0, nu: int = 3,
                          device="cpu") -> torch.Tensor:
    """BF16 [rows, cols] heavy-tailed activations with fixed outlier channels."""
    g = _gen(seed, device)
    z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(rows, cols, device=device, dtype=torch.float32)
    for _ in range(nu):
        e = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(e, e)
        del e
    x = z.div_(chi2.div_(nu).sqrt_())
    del chi2
    go = _gen(outlier_seed, "cpu")
    ch = torch.randperm(cols, generator=go)[:n_outliers].to(device)
    x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def gaussian_weights(rows: int, cols: int, sigma: float, seed: int,
                     device="cpu") -> torch.Tensor:
    """BF16 [rows, cols] weights ~ N(0, sigma)."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    return w.mul_(sigma).to(torch.bfloat16)


def tiny_inputs(M: int = 64, K: int = 256, N: int = 128, seed: int = 0, device="cpu"):
    """The tiny single linear: X ~ N(0,1) with 1 % entries x50, W ~ N(0, 0.02).

    Both are drawn in FP32 from one generator (X first, then the outlier mask,
    then W) and rounded once to BF16.
    """
    g = _gen(seed, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(M, K, generator=g, device=device) < 0.01
    x = torch.where(mask, x * 50.0, x)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * 0.02
    return x.to(torch.bfloat16), w.to(torch.bfloat16), x, w


def gdn_weights(modules=GDN_MODULES, cols: int = HIDDEN, first_seed: int = 10,
                device="cpu"):
    """List of (name, BF16 [rows, cols]) per module, seeds first_seed, +1, ..."""
    return [(name, gaussian_weights(rows, cols, sigma, first_seed + i, device))
            for i, (name, rows, sigma) in enumerate(modules)]


def gdn_gate_params(heads: int, seed: int = 40, device="cpu"):
    """FP32 per-head decay-gate parameters (A_log, dt_bias) in the usual
    Mamba-style initialisation: A ~ U(1, 16), A_log = log A; dt log-uniform in
    [1e-3, 1e-1] and dt_bias the softplus preimage of dt.  Input generation
    only -- seeded, float64 on the CPU, then cast."""
    g = _gen(seed, "cpu")
    a = 1.0 + 15.0 * torch.rand(heads, generator=g, dtype=torch.float64)
    u = torch.rand(heads, generator=g, dtype=torch.float64)
    dt = torch.exp(math.log(1e-3) + u * (math.log(1e-1) - math.log(1e-3)))
    dt_bias = dt + torch.log(-torch.expm1(-dt))
    return (torch.log(a).to(torch.float32).to(device), dt_bias.to(torch.float32).to(device))


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a BF16 tensor's bit patterns (for the oracle)."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
