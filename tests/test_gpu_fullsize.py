"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the quantizer on the whole [32768, 5120] activation
(bit-exact), the fused GDN input projection at 8192 x 24704 x 5120 (codes and
scales bit-exact everywhere, GEMM on 256 seeded rows against the oracle, fused ==
per-module bit for bit), the decode-shaped sweep (every row), and the 32K MLP
(64 seeded rows through every stage)."""
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
    rows = sample_rows(8192, 254, 0)                     # 256 rows with the first and last
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
    rows = sample_rows(M, M, M)                          # every row (M <= 128)
    ca, sa = oracle.quantize(xb[rows], ga)
    A = dequant(ca, sa)
    alpha = oracle.segment_alpha(ga, segs)
    assert_gemm_matches(host_bits(y[torch.from_numpy(rows).to(DEV)]), A, W, alpha,
                        label=f"decode M={M} {which}")


def test_mlp_32k_prefill_sampled():
    # the 32K-token MLP: gate_up [34816, 5120], SiLU(gate)*up, requantization of
    # h [32768, 17408], down [5120, 17408]; every stage on sampled rows
    M, H, F = 32768, 5120, 17408
    x = synth.student_t_activations(M, H, seed=1, device=DEV)
    w_gu = synth.gaussian_weights(2 * F, H, 0.015, seed=20, device=DEV)
    w_dn = synth.gaussian_weights(H, F, 0.01, seed=21, device=DEV)
    a = nv.quantize_tensor(x)
    wq_gu = nv.quantize_tensor(w_gu)
    wq_dn = nv.quantize_tensor(w_dn)
    gu = nv.gemm(a, wq_gu)
    h = nv.silu_mul(gu)
    hq = nv.quantize_tensor(h)
    y = nv.gemm(hq, wq_dn)
    torch.cuda.synchronize()
    rows = sample_rows(M, 62, 7)
    rid = torch.from_numpy(rows).to(DEV)
    xb = host_bits(x)
    ga, _ = oracle.global_scale(xb)
    ca, sa = oracle.quantize(xb[rows], ga)
    wgb = host_bits(w_gu)
    gw, _ = oracle.global_scale(wgb)
    cw, sw = oracle.quantize(wgb, gw)
    assert np.array_equal(np_u8(wq_gu.codes), cw)
    assert_gemm_matches(host_bits(gu[rid]), dequant(ca, sa), dequant(cw, sw),
                        oracle.segment_alpha(ga, [(0, 2 * F, gw)]), label="gate_up 32K")
    del cw, sw
    hb_rows = host_bits(h[rid])
    ref_h = oracle.silu_mul(host_bits(gu[rid]))
    assert np.max(np.abs(hb_rows.astype(np.int32) - ref_h.astype(np.int32))) <= 1
    hb = host_bits(h)
    gh, _ = oracle.global_scale(hb)
    assert np_f32(hq.g)[0] == gh
    ch, sh = oracle.quantize(hb_rows, gh)
    assert np.array_equal(np_u8(hq.codes)[rows], ch)
    del hb
    wdb = host_bits(w_dn)
    gd, _ = oracle.global_scale(wdb)
    cd, sd = oracle.quantize(wdb, gd)
    assert_gemm_matches(host_bits(y[rid]), dequant(ch, sh), dequant(cd, sd),
                        oracle.segment_alpha(gh, [(0, H, gd)]), label="down 32K")


def test_mlp_32k_fused_silu_sampled():
    # the fused MLP intermediate at the 32K prefill size the benchmark times:
    # gate_up [34816, 5120] (rows interleaved gate/up in 128-row blocks) with
    # h = SiLU(gate) * up and its global scale in the epilogue.  h on 64 seeded
    # rows against SiLU(gate) * up of the exact GEMM; the returned scale equals
    # the standalone global scale of the whole h and the oracle's; the
    # requantization with it equals the unfused quantizer's bytes.
    from parity_helpers import assert_silu_matches
    M, H, F = 32768, 5120, 17408
    x = synth.student_t_activations(M, H, seed=1, device=DEV)
    w_gu = synth.gaussian_weights(2 * F, H, 0.015, seed=20, device=DEV)
    a = nv.quantize_tensor(x)
    wi = nv.quantize_tensor(nv.interleave_gate_up(w_gu))
    h, g_h, amax_h = nv.gemm_silu_mul(a, wi)
    g_chk, amax_chk = nv.global_scale(h)
    c1, s1 = nv.quantize(h, g_h)
    q2 = nv.quantize_tensor(h)
    torch.cuda.synchronize()
    assert nv.last_device_status() == 0
    assert np_f32(g_h)[0] == np_f32(g_chk)[0] and np_f32(amax_h)[0] == np_f32(amax_chk)[0]
    assert torch.equal(c1, q2.codes) and torch.equal(s1, q2.sf)
    del c1, s1, q2
    g_or, amax_or = oracle.global_scale(host_bits(h))
    assert np_f32(g_h)[0] == g_or and np_f32(amax_h)[0] == amax_or
    rows = sample_rows(M, 62, 11)
    rid = torch.from_numpy(rows).to(DEV)
    xb = host_bits(x)
    ga, _ = oracle.global_scale(xb)
    ca, sa = oracle.quantize(xb[rows], ga)
    wgb = host_bits(w_gu)
    gw, _ = oracle.global_scale(wgb)
    cw, sw = oracle.quantize(wgb, gw)
    A, W = dequant(ca, sa), dequant(cw, sw)
    del cw, sw
    alpha = oracle.segment_alpha(ga, [(0, 2 * F, gw)])
    y64 = oracle.gemm_f64(A, W, alpha)
    S = (np.abs(A) @ np.abs(W).T) * np.abs(alpha)[None, :]
    exact = assert_silu_matches(host_bits(h[rid]), y64[:, :F], y64[:, F:], S[:, :F], S[:, F:], H,
                                label="fused SiLU 32K")
    assert exact > 0.9
