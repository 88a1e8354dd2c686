"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the quantizer on the whole [32768, 5120] activation
(bit-exact), the fused GDN input projection at 8192 x 24704 x 5120 (codes and
scales bit-exact everywhere, GEMM on sampled rows against the oracle, fused ==
per-module bit for bit), and the decode-shaped sweep."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    rows = set([0, M - 1]) | set(rng.choice(M, min(n, M), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


def test_quantizer_full_activation_bitexact():
    x = synth.student_t_activations(32768, 5120, seed=1, device=DEV)
    q = nv.quantize_tensor(x)
    torch.cuda.synchronize()
    bits = host_bits(x)
    g, amax = oracle.global_scale(bits)
    assert np_f32(q.g)[0] == g
    codes, sf = oracle.quantize(bits, g)
    assert np.array_equal(np_u8(q.codes), codes)
    assert np.array_equal(np_u8(q.sf), oracle.sf_to_tcgen05(sf))


def quantize_modules_oracle(ws):
    cs, ss, segs, off = [], [], [], 0
    for w in ws:
        b = host_bits(w)
        g, _ = oracle.global_scale(b)
        c, s = oracle.quantize(b, g)
        cs.append(c)
        ss.append(s)
        segs.append((off, w.shape[0], np.float32(g)))
        off += w.shape[0]
    return np.concatenate(cs), np.concatenate(ss), segs


def test_fused_gdn_prefill_full_size():
    x = synth.student_t_activations(8192, 5120, seed=3, device=DEV)
    ws = [w for _, w in synth.gdn_weights(synth.GDN_MODULES, device=DEV)]
    fw = nv.FusedWeight.from_modules(ws)
    a = nv.quantize_tensor(x)
    y = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    torch.cuda.synchronize()
    assert y.shape == (8192, 24704)
    # operands bit-exact everywhere
    cw, sw, segs = quantize_modules_oracle(ws)
    assert np.array_equal(np_u8(fw.codes), cw)
    assert np.array_equal(np_u8(fw.sf), oracle.sf_to_tcgen05(sw))
    xb = host_bits(x)
    ga, _ = oracle.global_scale(xb)
    rows = sample_rows(8192, 14, 0)
    ca, sa = oracle.quantize(xb[rows], ga)
    assert np.array_equal(np_u8(a.codes)[rows], ca)
    # GEMM on sampled rows against the FP64 oracle
    A = dequant(ca, sa)
    W = dequant(cw, sw)
    alpha = oracle.segment_alpha(ga, segs)
    stats = assert_gemm_matches(host_bits(y[torch.from_numpy(rows).to(DEV)]), A, W, alpha,
                                label="gdn-prefill")
    print("gdn prefill sampled rows:", stats)
    # fused == per-module GEMMs, bit for bit
    for (off, n, _), w in zip(fw.segments(), ws):
        ym = nv.gemm(a, nv.quantize_tensor(w))
        torch.cuda.synchronize()
        assert torch.equal(y[:, off:off + n].view(torch.int16), ym.view(torch.int16))


_decode_cache = {}


def decode_weights(which):
    """GPU weights and the oracle's quantization of them, built once per
    weight set for the whole sweep."""
    if which not in _decode_cache:
        if which == "gdn24640":
            ws = [w for _, w in synth.gdn_weights(synth.GDN_MODULES_DECODE, device=DEV)]
        else:
            N = 5120 if which == "dense5120" else 34816
            ws = [synth.gaussian_weights(N, 5120, 0.015, seed=20, device=DEV)]
        cw, sw, segs = quantize_modules_oracle(ws)
        _decode_cache[which] = (ws, cw, dequant(cw, sw), segs)
    return _decode_cache[which]


@pytest.mark.parametrize("which", ["dense5120", "gdn24640", "gateup34816"])
@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_decode_sweep(which, M):
    K = 5120
    ws, cw, W, segs = decode_weights(which)
    x = synth.student_t_activations(M, K, seed=100 + M, device=DEV)
    a = nv.quantize_tensor(x)
    if which == "gdn24640":
        fw = nv.FusedWeight.from_modules(ws)
        assert np.array_equal(np_u8(fw.codes), cw)
        y = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    else:
        wq = nv.quantize_tensor(ws[0])
        y = nv.gemm(a, wq)
    torch.cuda.synchronize()
    xb = host_bits(x)
    ga, _ = oracle.global_scale(xb)
    rows = sample_rows(M, 6, M)
    ca, sa = oracle.quantize(xb[rows], ga)
    A = dequant(ca, sa)
    alpha = oracle.segment_alpha(ga, segs)
    assert_gemm_matches(host_bits(y[torch.from_numpy(rows).to(DEV)]), A, W, alpha,
                        label=f"decode M={M} {which}")
