"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (derived from the arithmetic, stated once here):

* Codes, scale bytes, global scales: bit-exact.  Both sides take every
  quantization decision in binary32 with IEEE round-to-nearest-even division,
  so there is exactly one correct byte.
* GEMM output, element-wise.  The GPU accumulates in FP32 on the tensor
  cores in an order of its own, multiplies by alpha = fl32(gA*gW) and rounds to
  BF16; the oracle sums exactly-representable products in FP64.  With
  S = |alpha| * sum_k |a_k w_k| (the sum of magnitudes), FP32 accumulation over
  K terms errs by at most K * 2^-24 * S (2^-22 used: margin for the unknown
  internal order), the alpha product and scaling by 2 * 2^-24 * |y|, and BF16
  rounding by 2^-8 * |y| (8 significant bits).  Hence
      |y_gpu - y64| <= (2^-8 + 2^-22) |y64| + K * 2^-22 * S.
* GEMM output, row-normalised (the target's own reading): per row m,
  max_n |y_gpu - y64| / ||y64[m, :]||_2 <= 2e-3.  "Row norm" is read as the
  Euclidean norm of the FP64 reference row.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_w4a4_quantized_09_b200.synth import bf16_bits

ROW_NORM_TOL = 2e-3


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().astype(np.uint8)


def np_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float32)


def oracle_quant(x_host_bits: np.ndarray, g=None):
    """(codes, sf_linear, g) from the oracle; g from the whole tensor if None."""
    if g is None:
        g, _ = oracle.global_scale(x_host_bits)
    codes, sf = oracle.quantize(x_host_bits, g)
    return codes, sf, np.float32(g)


def assert_gemm_matches(y_gpu_bits: np.ndarray, A: np.ndarray, W: np.ndarray, alpha: np.ndarray,
                        row_ids=None, label=""):
    """y_gpu_bits: BF16 bit patterns [rows(sel), N]; A, W dequantized without
    global scales (FP64); alpha per column (FP64)."""
    y64 = oracle.gemm_f64(A, W, alpha, row_ids)
    rid = np.arange(A.shape[0]) if row_ids is None else np.asarray(row_ids)
    S = (np.abs(A[rid]) @ np.abs(W).T) * np.abs(alpha)[None, :]
    K = A.shape[1]
    yg = oracle.bf16_bits_to_f64(y_gpu_bits)
    err = np.abs(yg - y64)
    bound = (2.0 ** -8 + 2.0 ** -22) * np.abs(y64) + K * 2.0 ** -22 * S + 1e-37
    bad = err > bound
    assert not bad.any(), (
        f"{label}: {bad.sum()} elements beyond the derived bound; worst ratio "
        f"{(err / bound).max():.3g} at {np.unravel_index(np.argmax(err / bound), err.shape)}")
    norms = np.linalg.norm(y64, axis=1)
    rel = np.max(err, axis=1) / np.where(norms > 0, norms, 1.0)
    assert rel.max() <= ROW_NORM_TOL, f"{label}: row-normalised error {rel.max():.3g}"
    ref_bits = oracle.bf16_from_double(y64)
    exact = float(np.mean(ref_bits == y_gpu_bits))
    return {"max_row_rel": float(rel.max()), "bf16_exact_fraction": exact,
            "max_elem_over_bound": float((err / bound).max())}


def dequant(codes, sf):
    return oracle.dequantize_noglobal(codes, sf)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return bf16_bits(t)


def assert_gates_match(y_gpu_bits, y64, S, K, kind, a_log=None, dt_bias=None, label=""):
    """Gate outputs of one segment against the oracle's gate functions on the
    FP64 GEMM values y64 [rows, n]; S = |alpha| sum_k |a_k w_k| per element.
    Bound (derived in tests/test_gpu_gates.py): L (e_v + 2^-24 |y + b|) +
    (2^-7 + 2^-18) |r| + 2^-126 with e_v = 2^-23 |y64| + K 2^-22 S and L the
    gate's Lipschitz constant (e^A_log for the decay gate, 1/4 for the sigmoid).
    Returns the fraction equal to the oracle's BF16 value."""
    ref_bits = oracle.gdn_gates(y64, kind, a_log, dt_bias)
    ref = oracle.bf16_bits_to_f64(ref_bits)
    e_v = 2.0 ** -23 * np.abs(y64) + K * 2.0 ** -22 * S
    if kind == oracle.GATE_DECAY:
        lip = np.exp(np.asarray(a_log, np.float64))[None, :]
        zabs = np.abs(y64 + np.asarray(dt_bias, np.float64)[None, :])
    else:
        lip, zabs = 0.25, np.abs(y64)
    bound = lip * (e_v + 2.0 ** -24 * zabs) + (2.0 ** -7 + 2.0 ** -18) * np.abs(ref) + 2.0 ** -126
    err = np.abs(oracle.bf16_bits_to_f64(y_gpu_bits) - ref)
    assert np.all(err <= bound), f"{label}: worst ratio {float((err / bound).max()):.3g}"
    return float((y_gpu_bits == ref_bits).mean())


def assert_silu_matches(h_gpu_bits, g64, u64, Sg, Su, K, label=""):
    """h = SiLU(gate) * up against the oracle on the FP64 GEMM values.
    Bound (derived in tests/test_gpu_mlp_fused.py): 1.1 e_g |u| + |SiLU(g)| e_u
    + 1.1 e_g e_u + (2^-7 + 2^-18) |h_ref| + 2^-126.  Returns the fraction equal
    to the oracle's BF16 value."""
    ref_bits = oracle.silu_mul_f64(g64, u64)
    ref = oracle.bf16_bits_to_f64(ref_bits)
    e_g = 2.0 ** -23 * np.abs(g64) + K * 2.0 ** -22 * Sg
    e_u = 2.0 ** -23 * np.abs(u64) + K * 2.0 ** -22 * Su
    silu = np.abs(g64 / (1.0 + np.exp(-g64)))
    bound = (1.1 * e_g * np.abs(u64) + silu * e_u + 1.1 * e_g * e_u +
             (2.0 ** -7 + 2.0 ** -18) * np.abs(ref) + 2.0 ** -126)
    err = np.abs(oracle.bf16_bits_to_f64(h_gpu_bits) - ref)
    assert np.all(err <= bound), f"{label}: worst ratio {float((err / bound).max()):.3g}"
    return float((h_gpu_bits == ref_bits).mean())
