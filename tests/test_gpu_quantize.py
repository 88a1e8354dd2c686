"""GPU parity of the global scale and the 16-block quantizer against the
oracle: bit-exact codes, scale bytes (tensor-core layout including its zero
padding, and the linear layout) and global scales."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth
from parity_helpers import np_f32, np_u8, oracle_quant, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check_quant_bitexact(x, layout=nv.SF_TCGEN05, g_host=None):
    bits = host_bits(x)
    if g_host is None:
        g_gpu, amax_gpu = nv.global_scale(x)
        g_o, amax_o = oracle.global_scale(bits)
        torch.cuda.synchronize()
        assert np_f32(g_gpu)[0].tobytes() == np.float32(g_o).tobytes()
        assert np_f32(amax_gpu)[0] == amax_o
    else:
        g_o = np.float32(g_host)
        g_gpu = torch.tensor([g_o], dtype=torch.float32, device=x.device)
    codes, sf = nv.quantize(x, g_gpu, layout)
    torch.cuda.synchronize()
    oc, osf = oracle.quantize(bits, g_o)
    gc = np_u8(codes)
    mism = np.argwhere(gc != oc)
    assert mism.size == 0, f"{len(mism)} code bytes differ, first at {mism[:3].tolist()}"
    want_sf = oracle.sf_to_tcgen05(osf) if layout == nv.SF_TCGEN05 else osf.ravel()
    got_sf = np_u8(sf)
    assert got_sf.shape == want_sf.shape
    bad = np.flatnonzero(got_sf != want_sf)
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:5].tolist()}"


@pytest.mark.parametrize("shape", [(64, 256), (300, 160), (257, 96), (1, 32), (128, 5120),
                                   (129, 1024), (513, 2080)])
def test_quantize_bitexact_tcgen05(shape):
    x = synth.student_t_activations(shape[0], shape[1], seed=shape[0] * 7 + shape[1], device=DEV)
    check_quant_bitexact(x, nv.SF_TCGEN05)


@pytest.mark.parametrize("shape", [(64, 256), (300, 160), (33, 96)])
def test_quantize_bitexact_linear(shape):
    x = synth.student_t_activations(shape[0], shape[1], seed=5 + shape[0], device=DEV)
    check_quant_bitexact(x, nv.SF_LINEAR)


def test_tiny_config_operands_bitexact():
    xb, wb, _, _ = synth.tiny_inputs(device=DEV)
    check_quant_bitexact(xb)
    check_quant_bitexact(wb)


def test_strided_rows():
    big = synth.student_t_activations(200, 640, seed=3, device=DEV)
    x = big[:, 64:64 + 512]           # ld = 640 > cols = 512
    assert x.stride(0) == 640
    check_quant_bitexact(x)


def test_zero_tensor_and_zero_blocks():
    x = torch.zeros(130, 64, dtype=torch.bfloat16, device=DEV)
    check_quant_bitexact(x)             # amax 0 -> g = 1, all scales and codes 0
    y = synth.student_t_activations(130, 64, seed=9, device=DEV)
    y[:, 16:32] = 0
    y[7, :] = 0
    check_quant_bitexact(y)


def edge_rows():
    """Rows whose values hit E2M1 ties, signed zeros, saturation and E4M3
    subnormal / saturated scales under caller-chosen global scales."""
    rows = []
    base = [6, -6, 3, -3, 0.5, -0.5, 0.25, -0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 0, -0.1]
    rows.append(base)
    rows.append([6.375, -6.375] + [0.0] * 14)
    rows.append([2.0 ** -12, -2.0 ** -12] + [0.0] * 14)
    rows.append([0.0234375, 0.01171875, -0.01171875] + [0.0] * 13)
    rng = np.random.default_rng(0)
    for _ in range(12):
        rows.append(list(rng.choice([-1, 1], 16) * np.exp(rng.uniform(-12, 8, 16))))
    return np.array(rows, np.float32)


@pytest.mark.parametrize("g", [1.0, 0.5, 1e-3, 3.0e-7, 17.0, 1e-30])
def test_edge_values_under_given_global_scale(g):
    r = edge_rows()
    x = torch.from_numpy(np.tile(r, (1, 2))).to(torch.bfloat16).to(DEV)   # 32 columns
    check_quant_bitexact(x, nv.SF_TCGEN05, g_host=g)
    check_quant_bitexact(x, nv.SF_LINEAR, g_host=g)


# (block absmax, global scale as float32 bits) next to an E4M3 midpoint, where
# the order of the two float32 divisions of the block scale decides the code
SCALE_ORDER_CASES = [
    (1.0078125, 0x3EA1E1E1), (1.0625, 0x3EAAAAAA), (1.1640625, 0x3E3AFAFA),
    (1.328125, 0x3E1DAE61), (1.4375, 0x3E2AAAAB), (1.0546875, 0x3D555556),
]


def test_exact_ties_behind_an_inexact_reciprocal():
    # d = 1.875 (g = 1, block absmax 11.25): the quotients 1.25, 2.5 and 5 are
    # exact E2M1 ties, and 1/1.875 is not a float32 -- the kernel's encoder
    # must reach the even code exactly as a true division does
    x = np.zeros((2, 32), np.float32)
    x[0, :6] = [11.25, 2.34375, 4.6875, 9.375, -2.34375, -4.6875]
    x[1, 16:22] = [-11.25, 4.6875, 2.34375, -9.375, 9.375, 2.34375]
    xt = torch.from_numpy(x).to(torch.bfloat16).to(DEV)
    check_quant_bitexact(xt, nv.SF_TCGEN05, g_host=1.0)
    check_quant_bitexact(xt, nv.SF_LINEAR, g_host=1.0)


@pytest.mark.parametrize("ab,gbits", SCALE_ORDER_CASES)
def test_block_scale_division_order(ab, gbits):
    g = float(np.array([gbits], np.uint32).view(np.float32)[0])
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 7], x[0, 16] = ab, -ab / 2, -ab
    check_quant_bitexact(torch.from_numpy(x).to(torch.bfloat16).to(DEV), nv.SF_LINEAR, g_host=g)


def test_every_bf16_value_through_the_encoder():
    # all finite non-negative BF16 patterns and their negatives, 16 to a block,
    # under a few global scales: exercises every E2M1 rounding decision
    bits = np.arange(0, 0x7F80, dtype=np.uint16)
    bits = np.concatenate([bits, bits | 0x8000])
    n = (bits.size + 31) // 32 * 32
    bits = np.concatenate([bits, np.zeros(n - bits.size, np.uint16)]).reshape(-1, 32)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(DEV)
    for g in [1.0, 2.0 ** -20, 1e10]:
        check_quant_bitexact(x, nv.SF_TCGEN05, g_host=g)


def test_quantize_slices_into_fused_buffer():
    mods = [(96, 0.02), (64, 0.2), (64, 0.002), (200, 0.015)]
    K = 320
    ws = [synth.gaussian_weights(n, K, s, seed=40 + i, device=DEV) for i, (n, s) in enumerate(mods)]
    fw = nv.FusedWeight.from_modules(ws)
    torch.cuda.synchronize()
    oc, osf = [], []
    for w in ws:
        c, s, g = oracle_quant(host_bits(w))
        oc.append(c)
        osf.append(s)
    assert np.array_equal(np_u8(fw.codes), np.concatenate(oc))
    assert np.array_equal(np_u8(fw.sf), oracle.sf_to_tcgen05(np.concatenate(osf)))
    for g_t, w in zip(fw.g_list, ws):
        assert np_f32(g_t)[0] == oracle.global_scale(host_bits(w))[0]


def test_global_scale_workspace_reused_across_calls():
    for seed in range(5):
        x = synth.student_t_activations(77, 96, seed=seed, device=DEV) * (10.0 ** (seed - 2))
        g, amax = nv.global_scale(x.to(torch.bfloat16))
        g_o, a_o = oracle.global_scale(host_bits(x.to(torch.bfloat16)))
        torch.cuda.synchronize()
        assert np_f32(g)[0] == g_o and np_f32(amax)[0] == a_o


def test_empty_rows_are_a_no_op():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    g, amax = nv.global_scale(x)
    codes, sf = nv.quantize(x, g, nv.SF_LINEAR)
    torch.cuda.synchronize()
    assert np_f32(g)[0] == 1.0 and np_f32(amax)[0] == 0.0
    assert codes.numel() == 0
