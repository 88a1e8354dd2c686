"""GPU parity of the gate epilogue of the fused Gated DeltaNet input
projection (evolve.pub, Key claims under review, second bullet: log-space
softplus/exponential decay gate and sigmoid write strength), in all three
GEMM kernels (M = 1 and 7: few-token kernel; 200: one-CTA kernel; 300: CTA
pairs).

Tolerance, derived from the arithmetic.  Before the gate function the kernel
holds v = fl32(acc * alpha) with |v - y64| <= e_v = 2^-23 |y64| + K 2^-22 S
(S = |alpha| sum_k |a_k w_k|: FP32 accumulation in any order, the alpha
product and the scaling rounding).  The decay gate f(y) = -e^A softplus(y + b)
has |f'| = e^A sigmoid(y + b) <= e^A; the sigmoid has |f'| <= 1/4.  The FP32
evaluation (one add, expf, log1pf, one multiply, or expf, one add, one
division) errs by at most 2^-20 |f| plus the add's 2^-24 |y + b| times the
slope; the kernel's BF16 rounding and the oracle's (FP64, rounded once) each
add 2^-8 |f|.  Hence, against the oracle's BF16 value r:
    |gpu - r| <= L (e_v + 2^-24 |y64 + b|) + (2^-7 + 2^-18) |r| + 2^-126.
Columns outside the gate segments are bit-identical to the plain fused GEMM."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import assert_gates_match, dequant, host_bits, oracle_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"

LAYOUTS = {
    # name, rows, sigma, gate kind; GDN order q, k, v, z, b (sigmoid), a (decay)
    "gdn": [("q", 256, 0.02, 0), ("k", 256, 0.02, 0), ("v", 512, 0.015, 0), ("z", 512, 0.015, 0),
            ("b", 64, 0.2, nv.ACT_SIGMOID), ("a", 64, 0.002, nv.ACT_DECAY_GATE)],
    # segment edges inside 4-column groups and 32-column chunks
    "ragged": [("x", 200, 0.02, 0), ("b", 56, 0.2, nv.ACT_SIGMOID), ("a", 40, 0.05, nv.ACT_DECAY_GATE),
               ("y", 72, 0.015, 0)],
}


def build(layout, K, seed0):
    mods = LAYOUTS[layout]
    ws = [synth.gaussian_weights(n, K, s, seed=seed0 + i, device=DEV) for i, (_, n, s, _) in enumerate(mods)]
    fw = nv.FusedWeight.from_modules(ws)
    acts, params = [], []
    for i, (_, n, _, kind) in enumerate(mods):
        if kind == nv.ACT_DECAY_GATE:
            a_log, dt_bias = synth.gdn_gate_params(n, seed=seed0 + 50 + i, device=DEV)
            acts.append((kind, a_log, dt_bias))
            params.append((a_log.cpu().numpy(), dt_bias.cpu().numpy()))
        else:
            acts.append((kind, None, None))
            params.append((None, None))
    return ws, fw, acts, params


@pytest.mark.parametrize("M", [1, 7, 200, 300])
@pytest.mark.parametrize("layout", ["gdn", "ragged"])
def test_gate_epilogue_matches_oracle(M, layout):
    K = 512
    ws, fw, acts, params = build(layout, K, seed0=90)
    xb = synth.student_t_activations(M, K, seed=91 + M, device=DEV)
    a = nv.quantize_tensor(xb)
    y_act = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments(), acts=acts)
    y_plain = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    torch.cuda.synchronize()
    # oracle GEMM (FP64) on the same operands
    ca, sa, ga = oracle_quant(host_bits(xb))
    A = dequant(ca, sa)
    segs, cws, sws, off = [], [], [], 0
    for w in ws:
        c, s, g = oracle_quant(host_bits(w))
        cws.append(c)
        sws.append(s)
        segs.append((off, w.shape[0], g))
        off += w.shape[0]
    W = dequant(np.concatenate(cws), np.concatenate(sws))
    alpha = oracle.segment_alpha(ga, segs)
    y64 = oracle.gemm_f64(A, W, alpha)
    S = (np.abs(A) @ np.abs(W).T) * np.abs(alpha)[None, :]
    yp = host_bits(y_plain)
    exact = total = 0
    for (off, n, _), (kind, _, _), (a_log, dt_bias) in zip(segs, acts, params):
        cols = slice(off, off + n)
        if kind == nv.ACT_NONE:
            assert np.array_equal(host_bits(y_act)[:, cols], yp[:, cols]), "identity segment changed"
            continue
        frac = assert_gates_match(host_bits(y_act)[:, cols], y64[:, cols], S[:, cols], K, kind,
                                  a_log, dt_bias, label=f"{layout} M={M} kind={kind}")
        exact += int(round(frac * M * n))
        total += M * n
    print(f"{layout} M={M}: {exact}/{total} gate outputs equal the oracle's BF16 exactly")
    assert exact >= 0.9 * total


def test_gate_epilogue_fused_equals_per_module():
    # the gate segment alone, as its own GEMM, gives the same bits
    K, M = 512, 64
    ws, fw, acts, _ = build("gdn", K, seed0=120)
    xb = synth.student_t_activations(M, K, seed=121, device=DEV)
    a = nv.quantize_tensor(xb)
    y = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments(), acts=acts)
    off = 0
    for w, act in zip(ws, acts):
        q = nv.quantize_tensor(w)
        y1 = nv.fused_gemm(a, q.codes, q.sf, [(0, w.shape[0], q.g)], acts=[act])
        torch.cuda.synchronize()
        n = w.shape[0]
        assert torch.equal(y[:, off:off + n].view(torch.int16), y1.view(torch.int16))
        off += n
