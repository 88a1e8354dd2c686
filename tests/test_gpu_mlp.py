"""GPU parity of the W4A4 MLP (gate_up GEMM -> SiLU(gate)*up -> global scale +
quantization -> down GEMM) against the oracle, stage by stage: each stage is
checked on the bytes the GPU's previous stage produced, so a mismatch points
at one kernel."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def ulp_distance(a_bits, b_bits):
    def key(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(key(a_bits) - key(b_bits))


def test_silu_mul_within_one_ulp():
    rng = np.random.default_rng(3)
    g = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float32)
    u = (rng.standard_normal((64, 256)) * 2).astype(np.float32)
    g[0, :8] = [0.0, -0.0, 1e-30, -1e-30, 60.0, -60.0, 88.0, -88.0]
    g[1, :8] = [-80.0, -81.0, -90.0, -95.0, -100.0, -120.0, -200.0, -1e6]
    u[1, :8] = [1.0, 3.0, 7.0, 1000.0, 1e30, 1e35, 1e38, 1.0]
    gu = torch.from_numpy(np.concatenate([g, u], axis=1)).to(torch.bfloat16).to(DEV)
    h = nv.silu_mul(gu)
    torch.cuda.synchronize()
    ref = oracle.silu_mul(host_bits(gu))
    d = ulp_distance(host_bits(h), ref)
    assert d.max() <= 1
    assert np.mean(d == 0) > 0.97


def test_mlp_stage_by_stage():
    M, H, F = 300, 512, 384
    x = synth.student_t_activations(M, H, seed=31, device=DEV)
    w_gu = synth.gaussian_weights(2 * F, H, 0.02, seed=32, device=DEV)
    w_dn = synth.gaussian_weights(H, F, 0.02, seed=33, device=DEV)
    a = nv.quantize_tensor(x)
    wq_gu = nv.quantize_tensor(w_gu)
    wq_dn = nv.quantize_tensor(w_dn)
    gu = nv.gemm(a, wq_gu)
    h = nv.silu_mul(gu)
    hq = nv.quantize_tensor(h)
    y = nv.gemm(hq, wq_dn)
    torch.cuda.synchronize()
    # 1. gate_up GEMM
    xb = host_bits(x)
    ga, _ = oracle.global_scale(xb)
    ca, sa = oracle.quantize(xb, ga)
    gw, _ = oracle.global_scale(host_bits(w_gu))
    cw, sw = oracle.quantize(host_bits(w_gu), gw)
    assert_gemm_matches(host_bits(gu), dequant(ca, sa), dequant(cw, sw),
                        oracle.segment_alpha(ga, [(0, 2 * F, gw)]), label="gate_up")
    # 2. SiLU * up on the GPU's gate_up output
    assert ulp_distance(host_bits(h), oracle.silu_mul(host_bits(gu))).max() <= 1
    # 3. requantization of the GPU's h: bit-exact
    hb = host_bits(h)
    gh, _ = oracle.global_scale(hb)
    assert np_f32(hq.g)[0] == gh
    ch, sh = oracle.quantize(hb, gh)
    assert np.array_equal(np_u8(hq.codes), ch)
    assert np.array_equal(np_u8(hq.sf), oracle.sf_to_tcgen05(sh))
    # 4. down GEMM
    gd, _ = oracle.global_scale(host_bits(w_dn))
    cd, sd = oracle.quantize(host_bits(w_dn), gd)
    assert_gemm_matches(host_bits(y), dequant(ch, sh), dequant(cd, sd),
                        oracle.segment_alpha(gh, [(0, H, gd)]), label="down")
    # the public composite gives the same bytes
    y2 = nv.mlp(x, wq_gu, wq_dn)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
