"""CPU oracle for the NVFP4 W4A4 quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import this package.  The product
path (``nvfp4_w4a4_quantized_09_b200``) never imports it, and this package
imports nothing from the product: the two share no code.

The arithmetic lives in ``nvfp4_oracle.c`` (plain scalar C, binary32 steps for
the quantizer, FP64 for the GEMM); this module only marshals numpy arrays.
Method statement (pages on "Why Gated DeltaNet Survives 4-Bit Quantization:
NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM"):

* evolve.pub review, Scope & Claims -- NVFP4 W4A4 = E2M1 values with an E4M3
  scale per 16-element block, on both weights and activations.
* chatpaper.ai abstract -- per-module-calibrated checkpoints served by fused
  multi-module GEMM kernels need per-module global scales (the global-scale
  mismatch the paper repairs).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, brute force, invariants and torch's ``float8_e4m3fn`` cast; the one
reported-only quantity (quantized-vs-BF16 GEMM error beside the pages' ~11 %)
is marked "parity unpinned" there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None

E4M3_MAX = 448.0
E2M1_MAX = 6.0
BLOCK = 16


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no FMA contraction, IEEE semantics)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-fopenmp", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_e2m1_value.argtypes = [ctypes.c_int]
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.oracle_global_scale.argtypes = [P, I64, I64, I64, P]
        lib.oracle_global_scale.restype = ctypes.c_float
        lib.oracle_quantize.argtypes = [P, I64, I64, I64, ctypes.c_float, P, P]
        lib.oracle_quantize.restype = None
        lib.oracle_sf_offset_tcgen05.argtypes = [I64, I64, I64]
        lib.oracle_sf_offset_tcgen05.restype = I64
        lib.oracle_sf_to_tcgen05.argtypes = [P, I64, I64, P]
        lib.oracle_sf_to_tcgen05.restype = None
        lib.oracle_dequantize_noglobal.argtypes = [P, P, I64, I64, P]
        lib.oracle_dequantize_noglobal.restype = None
        lib.oracle_gemm_f64.argtypes = [P, P, P, I64, I64, P, I64, P]
        lib.oracle_gemm_f64.restype = None
        lib.oracle_bf16_round.argtypes = [P, I64, P]
        lib.oracle_bf16_round.restype = None
        lib.oracle_e2m1_encode_array.argtypes = [P, I64, P]
        lib.oracle_e4m3_encode_array.argtypes = [P, I64, P]
        lib.oracle_bf16_from_double_array.argtypes = [P, I64, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_silu_mul.argtypes = [P, I64, I64, I64, P]
        lib.oracle_silu_mul.restype = None
        lib.oracle_harmonize_scales.argtypes = [P, I64, I64, P, P, ctypes.c_int, P]
        lib.oracle_harmonize_scales.restype = ctypes.c_float
        lib.oracle_kv_scale.argtypes = [ctypes.c_float]
        lib.oracle_kv_scale.restype = ctypes.c_float
        lib.oracle_kv_quantize.argtypes = [P, I64, I64, I64, ctypes.c_float, P]
        lib.oracle_kv_quantize.restype = None
        lib.oracle_gdn_gates.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P]
        lib.oracle_gdn_gates.restype = None
        lib.oracle_silu_mul_f64.argtypes = [P, P, I64, I64, P]
        lib.oracle_silu_mul_f64.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# formats
# --------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (bit 3 the sign) -- oracle_e2m1_value."""
    return _L().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    """Value of an E4M3 byte (NaN for 0x7F/0xFF) -- oracle_e4m3_value."""
    return _L().oracle_e4m3_value(int(code))


def e2m1_encode(t) -> np.ndarray:
    """E2M1 RNE-satfinite codes (sign in bit 3) of a float32 array."""
    t = _c(t, np.float32)
    out = np.empty(t.shape, np.uint8)
    _L().oracle_e2m1_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def e4m3_encode(s) -> np.ndarray:
    """Unsigned E4M3 RNE codes saturated at 448 of a non-negative float32 array."""
    s = _c(s, np.float32)
    out = np.empty(s.shape, np.uint8)
    _L().oracle_e4m3_encode_array(_ptr(s), s.size, _ptr(out))
    return out


def bf16_from_double(x) -> np.ndarray:
    """One round-to-nearest-even step from FP64 to BF16 bit patterns (uint16)."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _L().oracle_bf16_from_double_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f64(b) -> np.ndarray:
    """Exact FP64 values of BF16 bit patterns (uint16)."""
    b = _c(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the path: global scale -> block scales + codes -> GEMM -> BF16
# --------------------------------------------------------------------------

def global_scale(x_bf16: np.ndarray):
    """(g, amax) of a BF16 matrix given as uint16 bit patterns [rows, cols]."""
    x = _c(x_bf16, np.uint16)
    rows, cols = x.shape
    amax = ctypes.c_float(0.0)
    g = _L().oracle_global_scale(_ptr(x), rows, cols, cols, ctypes.byref(amax))
    return np.float32(g), np.float32(amax.value)


def quantize(x_bf16: np.ndarray, g: float):
    """codes [rows, cols/2] uint8 and linear scales [rows, cols/16] uint8."""
    x = _c(x_bf16, np.uint16)
    rows, cols = x.shape
    assert cols % BLOCK == 0
    codes = np.empty((rows, cols // 2), np.uint8)
    sf = np.empty((rows, cols // BLOCK), np.uint8)
    _L().oracle_quantize(_ptr(x), rows, cols, cols, ctypes.c_float(float(g)),
                         _ptr(codes), _ptr(sf))
    return codes, sf


def sf_offset_tcgen05(r: int, c: int, sfcols_padded: int) -> int:
    """Byte offset of scale (row r, 16-block column c) in the tensor-core
    layout with sfcols_padded scale columns -- oracle_sf_offset_tcgen05."""
    return _L().oracle_sf_offset_tcgen05(r, c, sfcols_padded)


def sf_to_tcgen05(sf_linear: np.ndarray) -> np.ndarray:
    """Linear [rows, sfcols] scales -> flat padded tensor-core layout bytes."""
    sf = _c(sf_linear, np.uint8)
    rows, sfcols = sf.shape
    rows_p = (rows + 127) // 128 * 128
    cols_p = (sfcols + 3) // 4 * 4
    out = np.empty(rows_p * cols_p, np.uint8)
    _L().oracle_sf_to_tcgen05(_ptr(sf), rows, sfcols, _ptr(out))
    return out


def dequantize_noglobal(codes: np.ndarray, sf_linear: np.ndarray) -> np.ndarray:
    """FP64 [rows, cols] of E2M1(code) x E4M3(block scale), without the
    global scale (exact) -- oracle_dequantize_noglobal."""
    codes = _c(codes, np.uint8)
    sf = _c(sf_linear, np.uint8)
    rows = codes.shape[0]
    cols = codes.shape[1] * 2
    out = np.empty((rows, cols), np.float64)
    _L().oracle_dequantize_noglobal(_ptr(codes), _ptr(sf), rows, cols, _ptr(out))
    return out


def gemm_f64(A: np.ndarray, W: np.ndarray, alpha: np.ndarray, row_ids=None) -> np.ndarray:
    """alpha[n] * sum_k A[m,k] W[n,k] in FP64 for the selected rows m."""
    A = _c(A, np.float64)
    W = _c(W, np.float64)
    alpha = _c(alpha, np.float64)
    M, K = A.shape
    N = W.shape[0]
    assert W.shape[1] == K and alpha.shape == (N,)
    rid = np.arange(M, dtype=np.int64) if row_ids is None else _c(row_ids, np.int64)
    out = np.empty((rid.size, N), np.float64)
    _L().oracle_gemm_f64(_ptr(A), _ptr(W), _ptr(alpha), N, K, _ptr(rid), rid.size, _ptr(out))
    return out


def segment_alpha(g_a: float, segments) -> np.ndarray:
    """Per-column alpha[n] = gA * gW[seg(n)] in FP64 from [(n_offset, n_size, gW)]."""
    n_total = sum(int(s[1]) for s in segments)
    alpha = np.empty(n_total, np.float64)
    expect = 0
    for off, size, gw in segments:
        assert int(off) == expect, "segments must tile [0, N) in order"
        alpha[int(off):int(off) + int(size)] = float(np.float32(g_a)) * float(np.float32(gw))
        expect += int(size)
    return alpha


def linear(a_codes, a_sf, g_a, w_codes, w_sf, segments, row_ids=None):
    """Y64 and its BF16 rounding for the (fused) W4A4 GEMM.

    segments: [(n_offset, n_size, gW)] covering the weight rows in order; a
    single segment is the unfused layer.  Returns (Y64 [rows, N], Y_bf16 bits).
    """
    A = dequantize_noglobal(a_codes, a_sf)
    W = dequantize_noglobal(w_codes, w_sf)
    alpha = segment_alpha(g_a, segments)
    y64 = gemm_f64(A, W, alpha, row_ids)
    return y64, bf16_from_double(y64)


def silu_mul(gate_up_bf16: np.ndarray) -> np.ndarray:
    """h = bf16(SiLU(gate) * up) from a BF16 [rows, 2f] gate_up matrix (uint16 bits)."""
    gu = _c(gate_up_bf16, np.uint16)
    rows, two_f = gu.shape
    assert two_f % 2 == 0
    f = two_f // 2
    h = np.empty((rows, f), np.uint16)
    _L().oracle_silu_mul(_ptr(gu), rows, f, two_f, _ptr(h))
    return h


def harmonize_scales(sf_linear: np.ndarray, segments):
    """Checkpoint-side harmonisation of a fused weight's block scales.

    sf_linear: linear [rows, sfcols] scale bytes of the fused weight;
    segments: [(n_offset, n_size, g)] tiling the rows in order.  Returns
    (g_c, sf') with g_c = max g and every module's scales re-expressed
    against g_c, codes unchanged (oracle_harmonize_scales in the C file)."""
    sf = _c(sf_linear, np.uint8)
    rows, sfcols = sf.shape
    expect = 0
    for off, size, _ in segments:
        assert int(off) == expect, "segments must tile the rows in order"
        expect += int(size)
    seg_rows = np.array([int(s[1]) for s in segments], np.int64)
    seg_g = np.array([float(np.float32(s[2])) for s in segments], np.float32)
    out = np.empty_like(sf)
    gc = _L().oracle_harmonize_scales(_ptr(sf), rows, sfcols, _ptr(seg_rows), _ptr(seg_g),
                                      len(segments), _ptr(out))
    return np.float32(gc), out


def kv_scale(amax: float) -> np.float32:
    """Calibrated per-tensor FP8 KV-cache scale fl32(amax / 448) (1 if amax = 0)."""
    return np.float32(_L().oracle_kv_scale(ctypes.c_float(float(np.float32(amax)))))


def kv_quantize(x_bf16: np.ndarray, s: float) -> np.ndarray:
    """Signed E4M3 bytes of fl32(x / s), RNE, saturating at 448 (oracle_kv_quantize)."""
    x = _c(x_bf16, np.uint16)
    rows, cols = x.shape
    out = np.empty((rows, cols), np.uint8)
    _L().oracle_kv_quantize(_ptr(x), rows, cols, cols, ctypes.c_float(float(np.float32(s))), _ptr(out))
    return out


GATE_DECAY, GATE_SIGMOID = 1, 2


def gdn_gates(y64: np.ndarray, kind: int, a_log=None, dt_bias=None) -> np.ndarray:
    """BF16 bits of the gate functions on FP64 GEMM values y64 [rows, ncols]:
    kind 1 g = -exp(A_log) softplus(y + dt_bias) per column, kind 2 sigmoid(y)."""
    y = _c(y64, np.float64)
    rows, ncols = y.shape
    al = _c(np.zeros(ncols) if a_log is None else a_log, np.float32)
    db = _c(np.zeros(ncols) if dt_bias is None else dt_bias, np.float32)
    out = np.empty((rows, ncols), np.uint16)
    _L().oracle_gdn_gates(_ptr(y), rows, ncols, ncols, _ptr(al), _ptr(db), int(kind), _ptr(out))
    return out


def silu_mul_f64(gate64: np.ndarray, up64: np.ndarray) -> np.ndarray:
    """h = bf16(SiLU(gate) * up) from FP64 gate and up [rows, f] (BF16 bits)."""
    g = _c(gate64, np.float64)
    u = _c(up64, np.float64)
    assert g.shape == u.shape
    rows, f = g.shape
    h = np.empty((rows, f), np.uint16)
    _L().oracle_silu_mul_f64(_ptr(g), _ptr(u), rows, f, _ptr(h))
    return h


def num_threads() -> int:
    """Threads the oracle's parallel loops use."""
    return int(_L().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's parallel loops use from now on (timing only: each
    output is computed by one thread in k order, so results do not change)."""
    _L().oracle_set_num_threads(int(n))
