"""Host-side pieces of the Python binding that need no GPU: the offline
gate/up row interleave the fused-SiLU GEMM reads, and argument checks that
raise before the library is called."""
import pytest
import torch

import nvfp4_w4a4_quantized_09_b200 as nv


def test_interleave_gate_up_is_the_block_permutation():
    F, K = 384, 16
    w = torch.arange(2 * F * K, dtype=torch.float32).reshape(2 * F, K).to(torch.bfloat16)
    wi = nv.interleave_gate_up(w)
    assert wi.shape == w.shape and wi.is_contiguous()
    for b in range(F // 128):
        assert torch.equal(wi[256 * b:256 * b + 128], w[128 * b:128 * b + 128])          # gate block b
        assert torch.equal(wi[256 * b + 128:256 * b + 256], w[F + 128 * b:F + 128 * b + 128])  # up block b
    # a permutation of the rows: nothing lost or duplicated
    assert torch.equal(torch.sort(wi.float().sum(1)).values, torch.sort(w.float().sum(1)).values)


def test_interleave_gate_up_rejects_bad_widths():
    with pytest.raises(ValueError):
        nv.interleave_gate_up(torch.zeros(2 * 100, 16, dtype=torch.bfloat16))   # F not a multiple of 128
    with pytest.raises(ValueError):
        nv.interleave_gate_up(torch.zeros(257, 16, dtype=torch.bfloat16))       # odd row count


def test_fused_gemm_act_table_length_checked_before_the_library():
    g = torch.ones(1)
    a = nv.QuantizedTensor(torch.zeros(4, 32, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                           g, 4, 64)
    with pytest.raises(ValueError):
        nv.fused_gemm(a, torch.zeros(8, 32, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                      [(0, 4, g), (4, 4, g)], acts=[(nv.ACT_SIGMOID, None, None)])


def test_gemm_requires_tensor_core_layout():
    g = torch.ones(1)
    a = nv.QuantizedTensor(torch.zeros(4, 32, dtype=torch.uint8), torch.zeros(16, dtype=torch.uint8),
                           g, 4, 64, nv.SF_LINEAR)
    with pytest.raises(ValueError):
        nv.gemm(a, a)
