"""GPU parity of the block-scaled FP4 GEMM and the fused multi-module GEMM
against the oracle (FP64 sums of the dequantized operands), within the
tolerance derived in parity_helpers; fused == per-module bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, np_f32, oracle_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_linear(xb, wb):
    a = nv.quantize_tensor(xb)
    w = nv.quantize_tensor(wb)
    out = nv.gemm(a, w)
    torch.cuda.synchronize()
    return a, w, out


def oracle_reference(xb, wb):
    ca, sa, ga = oracle_quant(host_bits(xb))
    cw, sw, gw = oracle_quant(host_bits(wb))
    A, W = dequant(ca, sa), dequant(cw, sw)
    alpha = oracle.segment_alpha(ga, [(0, wb.shape[0], gw)])
    return A, W, alpha


def test_tiny_config_full():
    xb, wb, x32, w32 = synth.tiny_inputs(device=DEV)
    a, w, y = run_linear(xb, wb)
    A, W, alpha = oracle_reference(xb, wb)
    stats = assert_gemm_matches(host_bits(y), A, W, alpha, label="tiny")
    assert stats["bf16_exact_fraction"] > 0.9
    # sanity (reported, not a target): quantized vs unquantized GEMM error
    ref = x32.double().cpu().numpy() @ w32.double().cpu().numpy().T
    yq = y.double().cpu().numpy()
    rel = np.linalg.norm(yq - ref) / np.linalg.norm(ref)
    print(f"tiny: quantized-vs-fp32 relative error {rel:.4f}; {stats}")
    assert rel < 0.25


@pytest.mark.parametrize("M,N,K", [
    (200, 600, 768),     # small-M configuration, ragged M and N
    (333, 520, 320),     # large-M configuration, K % 256 == 64
    (130, 136, 96),      # K % 64 == 32, ragged everything
    (512, 1024, 1024),   # several full tiles each way
    (257, 264, 5120),    # long K
    (300, 136, 160),     # large-M configuration, K % 64 == 32 (half an MMA in the last step)
    (513, 392, 2080),    # large-M, K % 256 == 32, one row into a third 256-row tile
    (1, 128, 256),
    (7, 40, 64),
])
def test_gemm_shapes(M, N, K):
    xb = synth.student_t_activations(M, K, seed=M + N + K, device=DEV)
    wb = synth.gaussian_weights(N, K, 0.02, seed=N * 3 + K, device=DEV)
    a, w, y = run_linear(xb, wb)
    A, W, alpha = oracle_reference(xb, wb)
    assert_gemm_matches(host_bits(y), A, W, alpha, label=f"{M}x{N}x{K}")


def test_output_row_stride_and_canary():
    M, N, K, ldy = 150, 200, 256, 216
    xb = synth.student_t_activations(M, K, seed=1, device=DEV)
    wb = synth.gaussian_weights(N, K, 0.05, seed=2, device=DEV)
    a = nv.quantize_tensor(xb)
    w = nv.quantize_tensor(wb)
    buf = torch.full((M + 1, ldy), -7.0, dtype=torch.bfloat16, device=DEV)
    y = buf[:M, :N]
    nv.gemm(a, w, y)
    torch.cuda.synchronize()
    assert torch.all(buf[:M, N:] == -7.0) and torch.all(buf[M] == -7.0)
    A, W, alpha = oracle_reference(xb, wb)
    assert_gemm_matches(host_bits(y.contiguous()), A, W, alpha, label="strided")


@pytest.mark.parametrize("M", [64, 384])
def test_one_hot_layout_and_nibble_order(M):
    # one nonzero per row of A, at a position that moves through every nibble,
    # 16-block and 64-wide MMA step: the output is a closed form that pins the
    # scale layout, the nibble order and the K-step addressing on the hardware
    K, N = 512, 256
    xa = np.zeros((M, K), np.float32)
    rng = np.random.default_rng(1)
    ks = np.arange(M) * 37 % K
    xa[np.arange(M), ks] = rng.choice([-1, 1], M) * np.exp(rng.uniform(-3, 3, M))
    xw = (rng.standard_normal((N, K)) * 0.1).astype(np.float32)
    xb = torch.from_numpy(xa).to(torch.bfloat16).to(DEV)
    wb = torch.from_numpy(xw).to(torch.bfloat16).to(DEV)
    a, w, y = run_linear(xb, wb)
    A, W, alpha = oracle_reference(xb, wb)
    assert_gemm_matches(host_bits(y), A, W, alpha, label="one-hot")


def gdn_like_modules(K, rows=(256, 256, 128, 64, 64), sig=(0.02, 0.02, 0.015, 0.2, 0.002)):
    return [synth.gaussian_weights(n, K, s, seed=60 + i, device=DEV) for i, (n, s) in
            enumerate(zip(rows, sig))]


@pytest.mark.parametrize("M", [100, 300])
def test_fused_equals_per_module_bitwise_and_oracle(M):
    K = 512
    ws = gdn_like_modules(K)
    xb = synth.student_t_activations(M, K, seed=11, device=DEV)
    fw = nv.FusedWeight.from_modules(ws)
    a = nv.quantize_tensor(xb)
    y_fused = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    torch.cuda.synchronize()
    off = 0
    for wmod in ws:
        wq = nv.quantize_tensor(wmod)
        y_mod = nv.gemm(a, wq)
        torch.cuda.synchronize()
        n = wmod.shape[0]
        assert torch.equal(y_fused[:, off:off + n].view(torch.int16), y_mod.view(torch.int16)), \
            f"fused != per-module for rows [{off}, {off + n})"
        off += n
    # against the oracle, per-segment alphas
    ca, sa, ga = oracle_quant(host_bits(xb))
    segs, cws, sws, o = [], [], [], 0
    for wmod in ws:
        c, s, g = oracle_quant(host_bits(wmod))
        cws.append(c)
        sws.append(s)
        segs.append((o, wmod.shape[0], g))
        o += wmod.shape[0]
    A = dequant(ca, sa)
    W = dequant(np.concatenate(cws), np.concatenate(sws))
    alpha = oracle.segment_alpha(ga, segs)
    assert_gemm_matches(host_bits(y_fused), A, W, alpha, label="fused")


def test_single_global_scale_is_the_mismatch():
    # the negative control: serving the fused weight with ONE global scale
    # (the first module's) mis-scales every other module by its scale ratio
    K, M = 256, 64
    ws = gdn_like_modules(K)
    xb = synth.student_t_activations(M, K, seed=12, device=DEV)
    fw = nv.FusedWeight.from_modules(ws)
    a = nv.quantize_tensor(xb)
    good = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    wrong = nv.fused_gemm(a, fw.codes, fw.sf, [(0, fw.rows, fw.g_list[0])])
    torch.cuda.synchronize()
    off = 0
    for n, g in zip(fw.sizes, fw.g_list):
        ratio = float(np_f32(fw.g_list[0])[0] / np_f32(g)[0])
        gseg = good[:, off:off + n].double()
        wseg = wrong[:, off:off + n].double()
        mask = gseg.abs() > gseg.abs().max() * 1e-2
        r = (wseg[mask] / gseg[mask]).cpu().numpy()
        assert np.allclose(r, ratio, rtol=2e-2), (off, ratio, r[:4])
        off += n
    assert float(np_f32(fw.g_list[0])[0] / np_f32(fw.g_list[4])[0]) > 3


def test_device_status_timeout_path():
    assert nv.last_device_status() == 0
    nv.debug_wait_timeout(2_000_000)          # 2 ms bounded wait that must give up
    assert nv.last_device_status() == 5       # NVFP4_ERR_TIMEOUT, context still usable
    assert nv.last_device_status() == 0       # cleared
    xb, wb, _, _ = synth.tiny_inputs(device=DEV)
    a, w, y = run_linear(xb, wb)
    assert nv.last_device_status() == 0
    A, W, alpha = oracle_reference(xb, wb)
    assert_gemm_matches(host_bits(y), A, W, alpha, label="after-timeout")


def test_zero_sized_gemm():
    a = nv.quantize_tensor(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV))
    w = nv.quantize_tensor(torch.ones(32, 64, dtype=torch.bfloat16, device=DEV))
    y = nv.gemm(a, w)
    torch.cuda.synchronize()
    assert y.shape == (0, 32)
