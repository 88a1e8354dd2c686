"""Sensitivity of the parity checks, on the CPU: the comparisons the GPU tests
use accept the oracle's own BF16 result and reject results carrying a
plausible kernel mistake -- for the GEMM a wrong module scale, swapped
nibbles, a scale row taken from the neighbouring row, a dropped k-block, a
transposed operand tile; for the gate and SiLU epilogues a dropped parameter,
a sign error, a swapped operand or a small scale error.  Every mistake is
planted in oracle-side data (no GPU involved)."""
import numpy as np
import pytest

import oracle
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import (assert_gates_match, assert_gemm_matches, assert_silu_matches, dequant,
                            host_bits, oracle_quant)

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


# ---------------------------------------------------------------------------
# the derived tolerances of the gate epilogue and the fused SiLU epilogue
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def gate_case():
    Mg, Ng, Kg = 32, 64, 512
    x = synth.student_t_activations(Mg, Kg, seed=81)
    w = synth.gaussian_weights(Ng, Kg, 0.05, seed=82)
    ca, sa, ga = oracle_quant(host_bits(x))
    cw, sw, gw = oracle_quant(host_bits(w))
    A, W = dequant(ca, sa), dequant(cw, sw)
    alpha = oracle.segment_alpha(ga, [(0, Ng, gw)])
    y64 = oracle.gemm_f64(A, W, alpha)
    S = (np.abs(A) @ np.abs(W).T) * np.abs(alpha)[None, :]
    a_log, dt_bias = (t.numpy() for t in synth.gdn_gate_params(Ng, seed=83))
    return dict(y64=y64, S=S, K=Kg, a_log=a_log, dt_bias=dt_bias)


def test_gate_bound_accepts_the_oracle_and_rejects_mistakes(gate_case):
    c = gate_case
    for kind in (oracle.GATE_DECAY, oracle.GATE_SIGMOID):
        ok = oracle.gdn_gates(c["y64"], kind, c["a_log"], c["dt_bias"])
        assert assert_gates_match(ok, c["y64"], c["S"], c["K"], kind, c["a_log"], c["dt_bias"]) == 1.0
    bad = [
        # decay gate without dt_bias
        (oracle.GATE_DECAY, oracle.gdn_gates(c["y64"], oracle.GATE_DECAY, c["a_log"],
                                             np.zeros_like(c["dt_bias"]))),
        # decay gate without the exp(A_log) factor
        (oracle.GATE_DECAY, oracle.gdn_gates(c["y64"], oracle.GATE_DECAY, np.zeros_like(c["a_log"]),
                                             c["dt_bias"])),
        # sigmoid of the negated value
        (oracle.GATE_SIGMOID, oracle.gdn_gates(-c["y64"], oracle.GATE_SIGMOID)),
        # gate computed from a value with a 1 % scale error (a wrong alpha)
        (oracle.GATE_SIGMOID, oracle.gdn_gates(1.01 * c["y64"], oracle.GATE_SIGMOID)),
    ]
    for kind, bits in bad:
        with pytest.raises(AssertionError):
            assert_gates_match(bits, c["y64"], c["S"], c["K"], kind, c["a_log"], c["dt_bias"])


def test_silu_bound_accepts_the_oracle_and_rejects_mistakes(gate_case):
    c = gate_case
    g64, u64 = c["y64"][:, :32], c["y64"][:, 32:]
    Sg, Su = c["S"][:, :32], c["S"][:, 32:]
    ok = oracle.silu_mul_f64(g64, u64)
    assert assert_silu_matches(ok, g64, u64, Sg, Su, c["K"]) == 1.0
    for bits in (oracle.silu_mul_f64(u64, g64),            # gate and up swapped
                 oracle.bf16_from_double(g64 * u64),        # the SiLU dropped
                 oracle.silu_mul_f64(g64, 1.02 * u64)):     # a 2 % scale error on up
        with pytest.raises(AssertionError):
            assert_silu_matches(bits, g64, u64, Sg, Su, c["K"])
