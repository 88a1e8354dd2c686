"""Sensitivity of the GEMM parity check, on the CPU: the comparison the GPU
tests use accepts the oracle's own BF16 result and rejects results carrying
a plausible kernel mistake -- a wrong module scale, swapped nibbles, a scale
row taken from the neighbouring row, a dropped k-block, a transposed operand
tile.  Every mistake is planted in oracle-side data (no GPU involved)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, oracle_quant

M, N, K = 24, 40, 256


@pytest.fixture(scope="module")
def case():
    x = synth.student_t_activations(M, K, seed=77)
    w = synth.gaussian_weights(N, K, 0.02, seed=78)
    ca, sa, ga = oracle_quant(host_bits(x))
    cw, sw, gw = oracle_quant(host_bits(w))
    A, W = dequant(ca, sa), dequant(cw, sw)
    alpha = oracle.segment_alpha(ga, [(0, 16, gw), (16, N - 16, np.float32(gw * 3.0))])
    y_bits = oracle.bf16_from_double(oracle.gemm_f64(A, W, alpha))
    return dict(ca=ca, sa=sa, cw=cw, sw=sw, A=A, W=W, alpha=alpha, y_bits=y_bits, ga=ga, gw=gw)


def _fails(y_bits, c):
    with pytest.raises(AssertionError):
        assert_gemm_matches(y_bits, c["A"], c["W"], c["alpha"], label="planted")


def test_accepts_the_oracle_result(case):
    stats = assert_gemm_matches(case["y_bits"], case["A"], case["W"], case["alpha"])
    assert stats["bf16_exact_fraction"] == 1.0


def test_rejects_one_module_with_the_wrong_scale(case):
    alpha = case["alpha"].copy()
    alpha[16:] = alpha[0]                          # the single-scale mismatch
    _fails(oracle.bf16_from_double(oracle.gemm_f64(case["A"], case["W"], alpha)), case)


def test_rejects_swapped_nibbles(case):
    ca = case["ca"].copy()
    ca[:, 3] = ((ca[:, 3] & 0x0F) << 4) | (ca[:, 3] >> 4)     # one byte per row, nibbles swapped
    A = dequant(ca, case["sa"])
    _fails(oracle.bf16_from_double(oracle.gemm_f64(A, case["W"], case["alpha"])), case)


def test_rejects_a_scale_row_from_the_neighbour(case):
    sw = case["sw"].copy()
    sw[5] = sw[6]                                   # scale layout off by one row
    W = dequant(case["cw"], sw)
    _fails(oracle.bf16_from_double(oracle.gemm_f64(case["A"], W, case["alpha"])), case)


def test_rejects_a_dropped_k_block(case):
    A = case["A"].copy()
    A[:, 64:80] = 0.0                               # one 16-element block of K skipped
    _fails(oracle.bf16_from_double(oracle.gemm_f64(A, case["W"], case["alpha"])), case)


def test_rejects_a_transposed_tile(case):
    W = case["W"].copy()
    W[:16, :16] = W[:16, :16].T.copy()              # a 16 x 16 operand tile transposed
    _fails(oracle.bf16_from_double(oracle.gemm_f64(case["A"], W, case["alpha"])), case)
