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


# ---------------------------------------------------------------------------
# buffer checks: the C ABI cannot see how large a caller's buffer is, so the
# binding checks dtype, shape and size first and the device last.  Each case
# below is malformed in one way and must be rejected for that reason (the
# message is matched), before any tensor reaches the library.
# ---------------------------------------------------------------------------
def _q(rows, cols, layout=nv.SF_TCGEN05):
    return nv.QuantizedTensor(torch.zeros(rows, cols // 2, dtype=torch.uint8),
                              torch.zeros(nv.sf_bytes(rows, cols, layout), dtype=torch.uint8),
                              torch.ones(1), rows, cols, layout)


X = torch.zeros(8, 64, dtype=torch.bfloat16)
G = torch.ones(1)


@pytest.mark.parametrize("kwargs,match", [
    (dict(codes=torch.zeros(8, 16, dtype=torch.uint8)), r"codes must have shape \(8, 32\)"),
    (dict(codes=torch.zeros(8, 32, dtype=torch.int8)), "codes must be a contiguous uint8"),
    (dict(codes=torch.zeros(32, 8, dtype=torch.uint8).t()), "codes must be a contiguous uint8"),
    (dict(sf=torch.zeros(16, dtype=torch.uint8)), r"sf holds 16 bytes, 512 needed"),
])
def test_quantize_rejects_bad_outputs(kwargs, match):
    with pytest.raises(ValueError, match=match):
        nv.quantize(X, G, **kwargs)


def test_quantize_rejects_a_non_f32_global_scale():
    with pytest.raises(ValueError, match="g must be a contiguous float32"):
        nv.quantize(X, torch.ones(1, dtype=torch.float64))


def test_quantize_into_checks_the_row_range_and_the_full_buffers():
    codes = torch.zeros(16, 32, dtype=torch.uint8)
    sf = torch.zeros(nv.sf_bytes(16, 64), dtype=torch.uint8)
    with pytest.raises(ValueError, match=r"rows \[12, 20\) outside \[0, 16\)"):
        nv.quantize_into(X, G, codes, sf, 12, 16)
    with pytest.raises(ValueError, match=r"codes must have shape \(24, 32\)"):
        nv.quantize_into(X, G, codes, sf, 0, 24)


def test_global_scale_rejects_small_workspace():
    with pytest.raises(ValueError, match="workspace holds 8 bytes"):
        nv.global_scale(X, workspace=torch.zeros(8, dtype=torch.uint8))


@pytest.mark.parametrize("y,match", [
    (torch.zeros(8, 40, dtype=torch.bfloat16), r"y must have shape \(8, 48\)"),
    (torch.zeros(8, 48, dtype=torch.float16), "y must be a torch.bfloat16"),
    (torch.zeros(48, 8, dtype=torch.bfloat16).t(), "y must be row-major"),
])
def test_gemm_rejects_bad_outputs(y, match):
    with pytest.raises(ValueError, match=match):
        nv.gemm(_q(8, 64), _q(48, 64), y)


def test_gemm_rejects_operands_that_disagree_with_their_sizes():
    a = _q(8, 64)
    a.codes = torch.zeros(4, 32, dtype=torch.uint8)          # fewer rows than a.rows says
    with pytest.raises(ValueError, match=r"a.codes must have shape \(8, 32\)"):
        nv.gemm(a, _q(48, 64))
    w = _q(48, 64)
    w.sf = w.sf[:100]                                         # scales of too few rows
    with pytest.raises(ValueError, match=r"w.sf holds 100 bytes, 512 needed"):
        nv.gemm(_q(8, 64), w)


def test_fused_gemm_checks_segments_weights_and_gate_parameters():
    a = _q(8, 64)
    wc, ws = torch.zeros(48, 32, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8)
    with pytest.raises(ValueError, match=r"segment 1 = \[36, 48\) does not continue at 32"):
        nv.fused_gemm(a, wc, ws, [(0, 32, G), (36, 12, G)])
    with pytest.raises(ValueError, match=r"1\.\.16 segments"):
        nv.fused_gemm(a, wc, ws, [(3 * i, 3, G) for i in range(17)])
    with pytest.raises(ValueError, match=r"w_codes must have shape \(40, 32\)"):
        nv.fused_gemm(a, wc, ws, [(0, 32, G), (32, 8, G)])
    segs = [(0, 32, G), (32, 16, G)]
    short = torch.zeros(8)
    with pytest.raises(ValueError, match=r"acts\[1\].a_log must hold at least 16"):
        nv.fused_gemm(a, wc, ws, segs, acts=[(nv.ACT_NONE, None, None),
                                             (nv.ACT_DECAY_GATE, short, torch.zeros(16))])
    with pytest.raises(ValueError, match="the decay gate needs a_log and dt_bias"):
        nv.fused_gemm(a, wc, ws, segs, acts=[(nv.ACT_DECAY_GATE, None, None),
                                             (nv.ACT_NONE, None, None)])
    with pytest.raises(ValueError, match=r"segments\[0\] global scale must be a contiguous float32"):
        nv.fused_gemm(a, wc, ws, [(0, 32, torch.ones(1, dtype=torch.float64)), (32, 16, G)])


def test_gemm_silu_mul_and_silu_mul_check_their_widths():
    with pytest.raises(ValueError, match="even number of columns"):
        nv.silu_mul(torch.zeros(4, 63, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match=r"h must have shape \(4, 32\)"):
        nv.silu_mul(torch.zeros(4, 64, dtype=torch.bfloat16), torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match=r"h must have shape \(8, 128\)"):
        nv.gemm_silu_mul(_q(8, 64), _q(256, 64), torch.zeros(8, 256, dtype=torch.bfloat16))


def test_kv_quantize_checks_scale_and_output():
    with pytest.raises(ValueError, match="scale must be a contiguous float32"):
        nv.kv_quantize(X, torch.ones(1, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must be a torch.uint8"):
        nv.kv_quantize(X, G, torch.zeros(8, 64, dtype=torch.int16))


def test_well_formed_host_tensors_stop_at_the_device_check():
    # everything else is right: the call is refused because the tensors are
    # on the host, before any pointer reaches the library
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        nv.gemm(_q(8, 64), _q(48, 64), torch.zeros(8, 48, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        nv.fused_gemm(_q(8, 64), torch.zeros(48, 32, dtype=torch.uint8),
                      torch.zeros(512, dtype=torch.uint8), [(0, 32, G), (32, 16, G)])
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        nv.quantize(X, G)


def test_linear_host_checks_its_arguments_before_the_library():
    w = _q(48, 64)
    with pytest.raises(ValueError, match="x_host must be a contiguous 2-D bfloat16 host tensor"):
        nv.linear_host(torch.zeros(8, 64, dtype=torch.float32), w)
    with pytest.raises(ValueError, match="x_host must be"):
        nv.linear_host(torch.zeros(64, 8, dtype=torch.bfloat16).t(), w)
    with pytest.raises(TypeError):
        nv.linear_host(X, torch.zeros(4))
    with pytest.raises(ValueError, match="x_host has 64 columns, the weight 96"):
        nv.linear_host(X, _q(48, 96))
    with pytest.raises(ValueError, match=r"y_host must be a contiguous bfloat16 host tensor of shape \(8, 48\)"):
        nv.linear_host(X, w, torch.zeros(8, 40, dtype=torch.bfloat16))
    scratch = nv.HostLinearScratch.__new__(nv.HostLinearScratch)
    scratch.shape = (8, 64, 40)
    with pytest.raises(ValueError, match=r"scratch is for \(8, 64, 40\)"):
        nv.linear_host(X, w, torch.zeros(8, 48, dtype=torch.bfloat16), scratch=scratch)
