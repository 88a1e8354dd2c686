"""GPU parity of the few-token GEMM path (M <= 128: weights on the MMA's M
side, K split over a cluster of 1, 2, 4 or 8 CTAs and reduced through
distributed shared memory) against the oracle, and fused == per-module bit for
bit on that path.

The shapes are chosen so that every split size, a shared-memory ring that
wraps several times, a last k-step with one scale atom, K % 64 == 32, every
padded token width class (16 .. 128) and ragged N all occur."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, oracle_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"


def k_split(K):
    """Cluster size the library picks for K (a function of K alone: the largest
    of 1, 2, 4, 8 that leaves every CTA at least 8 k-steps of 256)."""
    ks, s = (K + 255) // 256, 1
    while s < 8 and ks // (2 * s) >= 8:
        s *= 2
    return s


@pytest.mark.parametrize("M,N,K", [
    (64, 130, 96),       # one k-step, K % 64 == 32, split 1
    (3, 200, 2048),      # split 1, one full ring
    (17, 264, 4160),     # split 2, 8..9 steps in a ring of 4, last step one atom
    (9, 392, 8224),      # split 4, K % 64 == 32, 8..9 steps per CTA
    (128, 384, 2304),    # token width 128, ring of 3 wraps, split 1
    (100, 520, 5120),    # token width 112, split 2
    (45, 136, 17440),    # split 8, K % 64 == 32, ring wraps twice
    (1, 5, 7168),        # one token, five outputs, split 2
    (2, 300, 5120),      # split 2, two tokens
    (8, 136, 17440),     # split 8, eight tokens, ragged N
])
def test_decode_shapes(M, N, K):
    assert k_split(K) in (1, 2, 4, 8)
    xb = synth.student_t_activations(M, K, seed=M * 7 + K, device=DEV)
    wb = synth.gaussian_weights(N, K, 0.02, seed=N + K, device=DEV)
    a = nv.quantize_tensor(xb)
    w = nv.quantize_tensor(wb)
    # the output row stride must be a multiple of 8 elements: pad it
    ldy = (N + 7) // 8 * 8
    y = torch.empty(M, ldy, dtype=torch.bfloat16, device=DEV)[:, :N]
    nv.gemm(a, w, y)
    torch.cuda.synchronize()
    assert nv.last_device_status() == 0
    ca, sa, ga = oracle_quant(host_bits(xb))
    cw, sw, gw = oracle_quant(host_bits(wb))
    alpha = oracle.segment_alpha(ga, [(0, N, gw)])
    assert_gemm_matches(host_bits(y.contiguous()), dequant(ca, sa), dequant(cw, sw), alpha,
                        label=f"decode {M}x{N}x{K} split {k_split(K)}")


def test_decode_splits_cover_1_2_4_8():
    assert sorted({k_split(K) for K in (96, 4160, 8224, 17440)}) == [1, 2, 4, 8]


@pytest.mark.parametrize("M", [1, 24, 128])
def test_decode_fused_equals_per_module_bitwise(M):
    # segment boundaries inside 128-row tiles, sizes not multiples of 16,
    # per-module scales ~100x apart
    K = 4096
    rows = [200, 56, 72, 8, 296]
    sig = [0.02, 0.2, 0.002, 0.05, 0.015]
    ws = [synth.gaussian_weights(n, K, s, seed=40 + i, device=DEV)
          for i, (n, s) in enumerate(zip(rows, sig))]
    xb = synth.student_t_activations(M, K, seed=50 + M, device=DEV)
    a = nv.quantize_tensor(xb)
    fw = nv.FusedWeight.from_modules(ws)
    y_fused = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    torch.cuda.synchronize()
    off = 0
    for wmod in ws:
        y_mod = nv.gemm(a, nv.quantize_tensor(wmod))
        torch.cuda.synchronize()
        n = wmod.shape[0]
        assert torch.equal(y_fused[:, off:off + n].view(torch.int16), y_mod.view(torch.int16)), \
            f"fused != per-module for rows [{off}, {off + n})"
        off += n
    ca, sa, ga = oracle_quant(host_bits(xb))
    segs, cws, sws, o = [], [], [], 0
    for wmod in ws:
        c, s, g = oracle_quant(host_bits(wmod))
        cws.append(c)
        sws.append(s)
        segs.append((o, wmod.shape[0], g))
        o += wmod.shape[0]
    alpha = oracle.segment_alpha(ga, segs)
    assert_gemm_matches(host_bits(y_fused), dequant(ca, sa),
                        dequant(np.concatenate(cws), np.concatenate(sws)), alpha,
                        label=f"decode fused M={M}")


def test_decode_repeatable_bitwise():
    # the split-K reduction order is fixed: two runs give the same bits
    M, N, K = 32, 1000, 5120
    xb = synth.student_t_activations(M, K, seed=5, device=DEV)
    wb = synth.gaussian_weights(N, K, 0.02, seed=6, device=DEV)
    a, w = nv.quantize_tensor(xb), nv.quantize_tensor(wb)
    y1 = nv.gemm(a, w)
    y2 = nv.gemm(a, w)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_decode_output_stride_and_canary():
    # y written through a row stride wider than N; nothing outside [M, N) touched
    M, N, K, ldy = 9, 136, 1024, 152
    xb = synth.student_t_activations(M, K, seed=8, device=DEV)
    wb = synth.gaussian_weights(N, K, 0.02, seed=9, device=DEV)
    a, w = nv.quantize_tensor(xb), nv.quantize_tensor(wb)
    buf = torch.full((M + 1, ldy), -7.0, dtype=torch.bfloat16, device=DEV)
    y = buf[:M, :N]
    nv.gemm(a, w, y)
    torch.cuda.synchronize()
    assert torch.all(buf[:M, N:] == -7.0) and torch.all(buf[M] == -7.0)
    ca, sa, ga = oracle_quant(host_bits(xb))
    cw, sw, gw = oracle_quant(host_bits(wb))
    alpha = oracle.segment_alpha(ga, [(0, N, gw)])
    assert_gemm_matches(host_bits(y.contiguous()), dequant(ca, sa), dequant(cw, sw), alpha,
                        label="decode strided")
