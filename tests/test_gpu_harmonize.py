"""GPU parity of checkpoint-side scale harmonisation (the single-scale repair
of the fused-module global-scale mismatch, chatpaper.ai abstract): the
rewritten scale bytes are bit-exact against the oracle in both layouts, the
single-scale GEMM on them matches the oracle, and against the per-segment
epilogue the module holding the common scale is bit-identical while the
other modules lose precision (reported)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import _lib, synth
from parity_helpers import assert_gemm_matches, dequant, host_bits, np_f32, np_u8, oracle_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"

# GDN-like modules: per-module scales about 100x apart, sizes not multiples of 128
ROWS = [200, 136, 264, 72, 24, 40]
SIGMA = [0.02, 0.02, 0.015, 0.015, 0.2, 0.002]


def modules(K, seed0=60):
    return [synth.gaussian_weights(n, K, s, seed=seed0 + i, device=DEV)
            for i, (n, s) in enumerate(zip(ROWS, SIGMA))]


def oracle_harmonized(ws):
    """Oracle: per-module quantization, then harmonisation of the linear scales."""
    cs, ss, segs, off = [], [], [], 0
    for w in ws:
        c, s, g = oracle_quant(host_bits(w))
        cs.append(c)
        ss.append(s)
        segs.append((off, w.shape[0], g))
        off += w.shape[0]
    gc, sf_lin = oracle.harmonize_scales(np.concatenate(ss), segs)
    return np.concatenate(cs), sf_lin, gc, segs, np.concatenate(ss)


@pytest.mark.parametrize("K", [512, 96])
def test_harmonize_tcgen05_layout_bitexact(K):
    ws = modules(K)
    fw = nv.FusedWeight.from_modules(ws)
    h = nv.harmonize(fw)
    torch.cuda.synchronize()
    codes, sf_lin, gc, _, _ = oracle_harmonized(ws)
    assert np.array_equal(np_u8(h.codes), codes)                 # codes untouched
    assert np.array_equal(np_u8(h.sf), oracle.sf_to_tcgen05(sf_lin))
    assert np_f32(h.g)[0] == gc
    assert max(float(np_f32(g)[0]) for g in fw.g_list) == gc


@pytest.mark.parametrize("K", [160, 32])
def test_harmonize_linear_layout_bitexact(K):
    # 10 scales per row: 16-byte chunks span two rows; 2 per row: a chunk spans eight
    ws = modules(K, seed0=70)
    N = sum(ROWS)
    codes = torch.empty(N, K // 2, dtype=torch.uint8, device=DEV)
    sf = torch.empty(nv.sf_bytes(N, K, nv.SF_LINEAR), dtype=torch.uint8, device=DEV)
    segs, off = [], 0
    for w in ws:
        g, _ = nv.global_scale(w)
        nv.quantize_into(w, g, codes, sf, off, N, nv.SF_LINEAR)
        segs.append((off, w.shape[0], g))
        off += w.shape[0]
    arr = (_lib.Segment * len(segs))()
    for i, (o, n, g) in enumerate(segs):
        arr[i].n_offset, arr[i].n_size, arr[i].w_gscale = o, n, g.data_ptr()
    gc_dev = torch.empty(1, dtype=torch.float32, device=DEV)
    _lib.check("nvfp4_harmonize_scales", _lib.lib().nvfp4_harmonize_scales(
        ctypes.c_void_p(sf.data_ptr()), K, arr, len(segs), nv.SF_LINEAR,
        ctypes.c_void_p(gc_dev.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
    torch.cuda.synchronize()
    _, sf_lin, gc, _, _ = oracle_harmonized(ws)
    assert np.array_equal(np_u8(sf).reshape(N, K // 16), sf_lin)
    assert np_f32(gc_dev)[0] == gc


@pytest.mark.parametrize("M", [7, 300])
def test_single_scale_gemm_on_harmonized_weight(M):
    # parity of the single-scale GEMM on the harmonized scales, and the error
    # against the per-segment repair: identical on the common-scale module
    K = 512
    ws = modules(K, seed0=80)
    fw = nv.FusedWeight.from_modules(ws)
    h = nv.harmonize(fw)
    xb = synth.student_t_activations(M, K, seed=81 + M, device=DEV)
    a = nv.quantize_tensor(xb)
    y_h = nv.gemm(a, h)
    y_seg = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    torch.cuda.synchronize()
    codes, sf_lin, gc, segs, _ = oracle_harmonized(ws)
    ca, sa, ga = oracle_quant(host_bits(xb))
    assert_gemm_matches(host_bits(y_h), dequant(ca, sa), dequant(codes, sf_lin),
                        oracle.segment_alpha(ga, [(0, fw.rows, gc)]), label=f"harmonized M={M}")
    imax = int(np.argmax([float(np_f32(g)[0]) for g in fw.g_list]))
    errs = []
    for i, (off, n, _) in enumerate(segs):
        ref = y_seg[:, off:off + n].double()
        got = y_h[:, off:off + n].double()
        if i == imax:
            assert torch.equal(y_h[:, off:off + n].view(torch.int16),
                               y_seg[:, off:off + n].view(torch.int16))
        errs.append(float((got - ref).norm() / ref.norm()))
    print("harmonized vs per-segment relative error per module:", [f"{e:.2e}" for e in errs])
    # every other module's scales are re-rounded to E4M3's 3 mantissa bits
    # (at most 2^-4 relative per block scale): a non-zero, bounded loss
    for i, e in enumerate(errs):
        if i != imax:
            assert 0 < e < 0.1, (i, e)
