"""GPU parity of the gate_up GEMM with the SiLU(gate) * up epilogue (the MLP
intermediate computed from the FP32 accumulators; W4A4 on every linear layer,
chatpaper.ai abstract) and of the global scale of h it returns.

Tolerance, derived from the arithmetic.  The kernel holds gate and up as
fl32(acc * alpha), each within e = 2^-23 |y64| + K 2^-22 S of the exact
value (S = |alpha| sum_k |a_k w_k|).  |SiLU'| <= 1.1, so SiLU(g) u moves by at
most 1.1 e_g |u| + |SiLU(g)| e_u (+ the product of the two errors); the FP32
evaluation (expf, one add, one division, one multiply) errs by at most
2^-20 |h|; the kernel's and the oracle's BF16 roundings add 2^-8 |h| each:
    |h_gpu - h_ref| <= 1.1 e_g |u| + |SiLU(g)| e_u + 1.1 e_g e_u + (2^-7 + 2^-18) |h_ref| + 2^-126.
The returned global scale equals nvfp4_global_scale of the h written, bit for
bit, so the requantization of h is exact."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_silu_matches, dequant, host_bits, np_f32, oracle_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("M,F,K", [(300, 256, 256), (1000, 384, 512), (513, 128, 5120)])
def test_gemm_silu_mul_matches_oracle(M, F, K):
    x = synth.student_t_activations(M, K, seed=M + 3, device=DEV)
    w = synth.gaussian_weights(2 * F, K, 0.015, seed=F + 7, device=DEV)
    a = nv.quantize_tensor(x)
    wi = nv.quantize_tensor(nv.interleave_gate_up(w))
    h, g_h, amax_h = nv.gemm_silu_mul(a, wi)
    g_chk, amax_chk = nv.global_scale(h)
    torch.cuda.synchronize()
    # global scale of h: exactly what the standalone kernel and the oracle give
    assert np_f32(g_h)[0] == np_f32(g_chk)[0] and np_f32(amax_h)[0] == np_f32(amax_chk)[0]
    g_or, amax_or = oracle.global_scale(host_bits(h))
    assert np_f32(g_h)[0] == g_or and np_f32(amax_h)[0] == amax_or
    # h against SiLU(gate) * up of the exact GEMM (non-interleaved oracle weight)
    ca, sa, ga = oracle_quant(host_bits(x))
    cw, sw, gw = oracle_quant(host_bits(w))
    A, W = dequant(ca, sa), dequant(cw, sw)
    alpha = oracle.segment_alpha(ga, [(0, 2 * F, gw)])
    y64 = oracle.gemm_f64(A, W, alpha)
    S = (np.abs(A) @ np.abs(W).T) * np.abs(alpha)[None, :]
    exact = assert_silu_matches(host_bits(h), y64[:, :F], y64[:, F:], S[:, :F], S[:, F:], K,
                                label=f"M={M} F={F} K={K}")
    print(f"M={M} F={F} K={K}: {exact:.4f} of h equal the oracle's BF16 exactly")
    assert exact > 0.9


def test_gemm_silu_mul_then_requantize_is_the_unfused_quantizer():
    # the fused h requantized with the returned scale is byte-identical to the
    # quantizer run on h with its own freshly computed global scale
    M, F, K = 384, 256, 512
    x = synth.student_t_activations(M, K, seed=5, device=DEV)
    w = synth.gaussian_weights(2 * F, K, 0.015, seed=6, device=DEV)
    a = nv.quantize_tensor(x)
    wi = nv.quantize_tensor(nv.interleave_gate_up(w))
    h, g_h, _ = nv.gemm_silu_mul(a, wi)
    c1, s1 = nv.quantize(h, g_h)
    q2 = nv.quantize_tensor(h)
    torch.cuda.synchronize()
    assert torch.equal(c1, q2.codes) and torch.equal(s1, q2.sf)


def test_mlp_interleaved_is_the_fused_three_launch_path():
    # nv.mlp(interleaved=True): fused gate_up + SiLU epilogue, requantization of
    # h with the returned scale, down GEMM -- bit for bit the composed calls
    M, H, F = 300, 512, 256
    x = synth.student_t_activations(M, H, seed=41, device=DEV)
    w_gu = synth.gaussian_weights(2 * F, H, 0.015, seed=42, device=DEV)
    w_dn = synth.gaussian_weights(H, F, 0.01, seed=43, device=DEV)
    wi = nv.quantize_tensor(nv.interleave_gate_up(w_gu))
    wd = nv.quantize_tensor(w_dn)
    y = nv.mlp(x, wi, wd, interleaved=True)
    h, g_h, _ = nv.gemm_silu_mul(nv.quantize_tensor(x), wi)
    codes, sf = nv.quantize(h, g_h)
    y_ref = nv.gemm(nv.QuantizedTensor(codes, sf, g_h, M, F), wd)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
