"""A quantized weight written by save_quantized and read back onto the GPU
serves the same GEMM bit for bit: the fused GDN-shaped weight with its
per-module scales, and a harmonised single-scale copy of it."""
import pytest
import torch

import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

MODULES = [(256, 0.02), (128, 0.015), (64, 0.2), (64, 0.002)]


def test_fused_weight_file_serves_the_same_gemm(tmp_path):
    K = 512
    ws = [synth.gaussian_weights(n, K, s, seed=300 + i, device=DEV) for i, (n, s) in enumerate(MODULES)]
    fw = nv.FusedWeight.from_modules(ws)
    path = str(tmp_path / "fused.pt")
    nv.save_quantized(path, fw)
    fr = nv.load_quantized(path, device=DEV)
    a = nv.quantize_tensor(synth.student_t_activations(300, K, seed=301, device=DEV))
    y0 = nv.fused_gemm(a, fw.codes, fw.sf, fw.segments())
    y1 = nv.fused_gemm(a, fr.codes, fr.sf, fr.segments())
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_harmonized_weight_file_serves_the_same_gemm(tmp_path):
    K = 256
    ws = [synth.gaussian_weights(n, K, s, seed=310 + i, device=DEV) for i, (n, s) in enumerate(MODULES)]
    hq = nv.harmonize(nv.FusedWeight.from_modules(ws))
    path = str(tmp_path / "harmonized.pt")
    nv.save_quantized(path, hq)
    hr = nv.load_quantized(path, device=DEV)
    assert hr.layout == hq.layout and torch.equal(hr.g, hq.g)
    a = nv.quantize_tensor(synth.student_t_activations(7, K, seed=311, device=DEV))
    y0, y1 = nv.gemm(a, hq), nv.gemm(a, hr)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
