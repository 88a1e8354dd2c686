"""GPU parity of the FP8 E4M3 KV-cache quantizer with a calibrated per-tensor
scale (evolve.pub, Key claims under review): every byte equals the oracle's
(one binary32 division, RNE, saturation at 448, sign of zero kept), over every
finite BF16 value under several scales, ragged and strided shapes, and the
calibration s = fl32(amax / 448)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import host_bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def all_finite_bf16(cols=512):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    bits = bits[np.isfinite(vals)]
    pad = (-bits.size) % cols
    bits = np.concatenate([bits, np.zeros(pad, np.uint16)]).reshape(-1, cols)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("s", [1.0, 0.37, 3.1e-3, 41.0, 2.0 ** -126, 2.0 ** 126,
                               2.0 ** -92, 1.37 * 2.0 ** -90, 2.0 ** 100, 1.5 * 2.0 ** 100])
def test_kv_every_bf16_value_bitexact(s):
    # includes scales outside [2^-92, 2^100] (division path) and the edges of
    # that range, where large x overflow the quotient (the group divides)
    x = all_finite_bf16()
    scale = torch.tensor([s], dtype=torch.float32, device=DEV)
    out = nv.kv_quantize(x, scale)
    torch.cuda.synchronize()
    assert np.array_equal(np_u8(out), oracle.kv_quantize(host_bits(x), np.float32(s)))


def test_kv_exact_ties_behind_an_inexact_reciprocal():
    # s = 1.75: the quotients 1.5625, 1.8125 and 3.125 are exact E4M3 ties and
    # 1/1.75 is not a float32; the even codes must come out
    x = torch.tensor([[2.734375, 3.171875, 5.46875, -2.734375, 0, 0, 0, 0]],
                     dtype=torch.bfloat16, device=DEV)
    out = nv.kv_quantize(x, torch.tensor([1.75], dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    want = oracle.kv_quantize(host_bits(x), np.float32(1.75))
    assert [int(v) for v in want[0, :4]] == [0x3C, 0x3E, 0x44, 0xBC]
    assert np.array_equal(np_u8(out), want)


@pytest.mark.parametrize("rows,cols,ld,ldo", [(1, 8, 8, 8), (33, 136, 152, 144), (257, 1024, 1024, 1032),
                                               (4096, 2048, 2048, 2048)])
def test_kv_shapes_calibrated_bitexact(rows, cols, ld, ldo):
    calib = synth.student_t_activations(512, cols, seed=rows + 1, device=DEV)
    s = nv.kv_scale(calib)
    buf = synth.student_t_activations(rows, ld, seed=rows + 2, device=DEV)
    x = buf[:, :cols]
    obuf = torch.full((rows + 1, ldo), 0xA5, dtype=torch.uint8, device=DEV)
    out = obuf[:rows, :cols]
    nv.kv_quantize(x, s, out)
    torch.cuda.synchronize()
    xb = host_bits(x.contiguous())
    _, amax = oracle.global_scale(host_bits(calib))
    s_ref = oracle.kv_scale(amax)
    assert np_f32(s)[0] == s_ref
    assert np.array_equal(np_u8(out.contiguous()), oracle.kv_quantize(xb, s_ref))
    assert torch.all(obuf[:rows, cols:] == 0xA5) and torch.all(obuf[rows] == 0xA5)   # canary


def test_kv_scale_of_zero_tensor_is_one():
    s = nv.kv_scale(torch.zeros(16, 64, dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert np_f32(s)[0] == np.float32(1.0)
