"""The C-ABI library without a GPU: it loads, exports every entry point that
include/nvfp4.h declares, and rejects bad arguments on the host before any
CUDA call (no compute runs here)."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_quantized_09_b200 import _lib, build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    _build.build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_path():
    names = declared_functions()
    for required in ["nvfp4_global_scale", "nvfp4_quantize", "nvfp4_gemm", "nvfp4_fused_gemm",
                     "nvfp4_sf_bytes", "nvfp4_quantize_slice"]:
        assert required in names


UTILITIES = {"nvfp4_sf_bytes", "nvfp4_last_device_status", "nvfp4_debug_wait_timeout",
             "nvfp4_status_string", "nvfp4_version"}
# entries that serve the library's callers rather than a step of the method:
# their comment says the pages have no counterpart instead of citing one
LIBRARY_ONLY = {"nvfp4_global_scale_noalloc"}


def test_every_computational_entry_documents_its_source_and_errors():
    # each declaration of the path is preceded by a comment that cites the
    # passage it follows and states its errors (utilities have no passage)
    src = open(HEADER).read()
    found = set()
    for m in re.finditer(r"/\*((?:(?!\*/).)*)\*/\s*\n(?:nvfp4_status|const char\*|int)\s+(nvfp4_[a-z0-9_]+)\(",
                         src, re.S):
        comment, name = m.group(1), m.group(2)
        found.add(name)
        if name in UTILITIES:
            continue
        if name in LIBRARY_ONLY:
            assert "Source" not in comment and "No passage of the pages" in comment, name
        else:
            assert "Source" in comment, f"{name}: no source passage"
        assert "Errors" in comment or "errors" in comment, f"{name}: no error behaviour"
    assert set(declared_functions()) - found <= {"nvfp4_kv_quantize_e4m3"}   # shares the KV block


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings_and_version(L):
    for s in range(7):
        assert len(L.nvfp4_status_string(s)) > 0
    assert L.nvfp4_version() >= 100


def test_sf_bytes(L):
    n = ctypes.c_size_t()
    assert L.nvfp4_sf_bytes(300, 160, _lib.SF_TCGEN05, ctypes.byref(n)) == 0
    assert n.value == 384 * 12
    assert L.nvfp4_sf_bytes(300, 160, _lib.SF_LINEAR, ctypes.byref(n)) == 0
    assert n.value == 300 * 10
    assert L.nvfp4_sf_bytes(32768, 5120, _lib.SF_TCGEN05, ctypes.byref(n)) == 0
    assert n.value == 32768 * 320
    assert L.nvfp4_sf_bytes(10, 24, _lib.SF_LINEAR, ctypes.byref(n)) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_sf_bytes(-1, 32, _lib.SF_LINEAR, ctypes.byref(n)) == _lib.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_sf_bytes(1, 32, 7, ctypes.byref(n)) == _lib.NVFP4_ERR_INVALID_ARG
    # sizes whose byte count would overflow are refused, not wrapped
    assert L.nvfp4_sf_bytes(1 << 31, 32, _lib.SF_LINEAR, ctypes.byref(n)) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_sf_bytes(1 << 40, 1 << 40, _lib.SF_TCGEN05, ctypes.byref(n)) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p(0x10008)       # 8-byte aligned only
NUL = ctypes.c_void_p(0)


def test_quantize_rejects_bad_arguments(L):
    q = L.nvfp4_quantize
    assert q(FAKE, 4, 48, 48, FAKE, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_ALIGNMENT   # cols % 32
    assert q(FAKE, 4, 64, 60, FAKE, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_ALIGNMENT   # ld % 8
    assert q(FAKE, 4, 64, 64, NUL, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG  # g null
    assert q(FAKE, 4, 64, 64, FAKE, FAKE, FAKE, 9, NUL) == _lib.NVFP4_ERR_INVALID_ARG  # layout
    assert q(FAKE, -1, 64, 64, FAKE, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 4, 64, 32, FAKE, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG  # ld < cols
    assert q(ODD, 4, 64, 64, FAKE, FAKE, FAKE, 1, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert q(FAKE, 4, 64, 64, FAKE, NUL, FAKE, 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 0, 64, 64, FAKE, NUL, NUL, 0, NUL) == _lib.NVFP4_OK                # empty


def test_quantize_slice_rejects_bad_ranges(L):
    q = L.nvfp4_quantize_slice
    assert q(FAKE, 4, 64, 64, FAKE, FAKE, FAKE, 1, 10, 12, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 4, 64, 64, FAKE, FAKE, FAKE, 1, -1, 12, NUL) == _lib.NVFP4_ERR_INVALID_ARG


def test_global_scale_rejects_bad_arguments(L):
    gs = L.nvfp4_global_scale
    assert gs(FAKE, 4, 64, 64, NUL, NUL, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # g_out
    assert gs(FAKE, 4, 64, 64, FAKE, NUL, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # workspace
    assert gs(FAKE, 4, 60, 64, FAKE, NUL, FAKE, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert gs(ODD, 4, 64, 64, FAKE, NUL, FAKE, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert gs(FAKE, 4, 64, 64, FAKE, NUL, ODD, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    # results inside the workspace the kernel clears at the end are refused
    WS = ctypes.c_void_p(0x40000)
    assert gs(FAKE, 4, 64, 64, ctypes.c_void_p(0x40000 + 200), NUL, WS, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert gs(FAKE, 4, 64, 64, FAKE, ctypes.c_void_p(0x40000 - 2), WS, NUL) == _lib.NVFP4_ERR_INVALID_ARG


def test_global_scale_noalloc_refuses_before_enqueuing(L):
    # the no-alloc form clears its scratch with a memset on the stream; every
    # refusal must come before that (no CUDA call is made for these)
    gs = L.nvfp4_global_scale_noalloc
    P = ctypes.c_void_p
    assert gs(FAKE, 4, 64, 64, NUL, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG          # g_out
    assert gs(NUL, 4, 64, 64, FAKE, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG          # x
    assert gs(FAKE, 4, 60, 64, FAKE, NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT           # cols % 8
    assert gs(FAKE, 4, 64, 60, FAKE, NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT           # ld % 8
    assert gs(FAKE, 4, 64, 56, FAKE, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG         # ld < cols
    assert gs(ODD, 4, 64, 64, P(0x30000), NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT      # x alignment
    assert gs(P(0x50000), 4, 64, 64, P(0x50000 + 100), NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG   # g in x
    assert gs(FAKE, 1 << 30, 64, 1 << 20, FAKE, NUL, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE


def test_gemm_rejects_bad_arguments(L):
    g = L.nvfp4_gemm
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert g(*ok, 128, 64, 128, 48, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE          # K % 32
    assert g(*ok, 128, 64, 128, 0, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE           # K = 0
    assert g(*ok, 100, 64, 128, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT                  # ldy < N
    assert g(*ok, 132, 64, 130, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT                  # ldy % 8
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, NUL, FAKE, 128, 64, 128, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert g(ODD, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 64, 128, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert g(*ok, 128, 0, 128, 64, NUL) == _lib.NVFP4_OK                              # M = 0


def seg_array(entries):
    arr = (_lib.Segment * len(entries))()
    for i, (o, n, p) in enumerate(entries):
        arr[i].n_offset, arr[i].n_size, arr[i].w_gscale = o, n, p
    return arr


def test_fused_gemm_validates_segment_table(L):
    f = L.nvfp4_fused_gemm
    args = (FAKE, FAKE, FAKE, FAKE, FAKE)
    good = seg_array([(0, 64, 0x10000), (64, 64, 0x10010)])
    assert f(*args, good, 0, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG      # nseg 0
    assert f(*args, good, 17, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # > max
    gap = seg_array([(0, 64, 0x10000), (72, 64, 0x10010)])
    assert f(*args, gap, 2, FAKE, 136, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG       # not contiguous
    empty = seg_array([(0, 64, 0x10000), (64, 0, 0x10010)])
    assert f(*args, empty, 2, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # n_size 0
    noscale = seg_array([(0, 64, 0x10000), (64, 64, 0)])
    assert f(*args, noscale, 2, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert f(*args, good, 2, FAKE, 120, 4, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT        # ldy < N
    assert f(*args, good, 2, FAKE, 128, 0, 64, NUL) == _lib.NVFP4_OK                   # M = 0
    # segment sizes whose sum would overflow int64 are refused one by one
    huge = seg_array([(0, 1 << 62, 0x10000), (1 << 62, 1 << 62, 0x10010)])
    assert f(*args, huge, 2, FAKE, 1 << 62, 4, 64, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE


def test_harmonize_rejects_bad_arguments(L):
    f = L.nvfp4_harmonize_scales
    good = seg_array([(0, 64, 0x20000), (64, 64, 0x20010)])   # scales apart from FAKE
    T, LIN = _lib.SF_TCGEN05, _lib.SF_LINEAR
    assert f(NUL, 64, good, 2, T, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # no scales
    assert f(FAKE, 64, good, 2, T, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG     # no g_common
    assert f(FAKE, 64, good, 0, T, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG    # nseg 0
    assert f(FAKE, 64, good, 17, T, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG   # > max
    assert f(FAKE, 64, good, 2, 7, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG    # layout
    gap = seg_array([(0, 64, 0x10000), (72, 64, 0x10010)])
    assert f(FAKE, 64, gap, 2, LIN, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG   # not contiguous
    noscale = seg_array([(0, 64, 0x10000), (64, 64, 0)])
    assert f(FAKE, 64, noscale, 2, LIN, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    huge = seg_array([(0, 1 << 62, 0x10000), (1 << 62, 1 << 62, 0x10010)])
    assert f(FAKE, 64, huge, 2, LIN, FAKE, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    # g_common may not alias a module scale the kernel is still reading
    assert f(FAKE, 64, good, 2, LIN, ctypes.c_void_p(0x20010), NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 24, good, 2, T, FAKE, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE   # K % 16
    assert f(FAKE, 0, good, 2, T, FAKE, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert f(ctypes.c_void_p(0x10008), 64, good, 2, T, FAKE, NUL) == _lib.NVFP4_ERR_ALIGNMENT


def test_kv_cache_entries_reject_bad_arguments(L):
    q = L.nvfp4_kv_quantize_e4m3
    assert q(FAKE, -1, 8, 8, FAKE, FAKE, 8, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 4, 8, 8, NUL, FAKE, 8, NUL) == _lib.NVFP4_ERR_INVALID_ARG      # no scale
    assert q(FAKE, 4, 12, 16, FAKE, FAKE, 16, NUL) == _lib.NVFP4_ERR_ALIGNMENT    # cols % 8
    assert q(FAKE, 4, 8, 12, FAKE, FAKE, 8, NUL) == _lib.NVFP4_ERR_ALIGNMENT      # ld % 8
    assert q(FAKE, 4, 8, 8, FAKE, FAKE, 12, NUL) == _lib.NVFP4_ERR_ALIGNMENT      # ldo % 8
    assert q(NUL, 4, 8, 8, FAKE, FAKE, 8, NUL) == _lib.NVFP4_ERR_INVALID_ARG      # no x
    assert q(FAKE, 4, 16, 8, FAKE, FAKE, 16, NUL) == _lib.NVFP4_ERR_INVALID_ARG   # ld < cols
    assert q(ODD, 4, 8, 8, FAKE, FAKE, 8, NUL) == _lib.NVFP4_ERR_ALIGNMENT        # x not 16-aligned
    assert q(FAKE, 4, 8, 8, FAKE, ctypes.c_void_p(0x10004), 8, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert q(FAKE, 0, 8, 8, FAKE, FAKE, 8, NUL) == _lib.NVFP4_OK                 # nothing to do
    assert L.nvfp4_kv_scale_from_amax(NUL, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_kv_scale_from_amax(FAKE, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG


def test_fused_gemm_act_validates_activations(L):
    f = L.nvfp4_fused_gemm_act
    args = (FAKE, FAKE, FAKE, FAKE, FAKE)
    segs = seg_array([(0, 64, 0x10000), (64, 64, 0x10010)])

    def acts(entries):
        arr = (_lib.SegmentAct * len(entries))()
        for i, (k, p0, p1) in enumerate(entries):
            arr[i].kind, arr[i].a_log, arr[i].dt_bias = k, p0, p1
        return arr
    bad_kind = acts([(0, 0, 0), (3, 0, 0)])
    assert f(*args, segs, bad_kind, 2, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    no_param = acts([(0, 0, 0), (_lib.ACT_DECAY_GATE, 0x10000, 0)])
    assert f(*args, segs, no_param, 2, FAKE, 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    ok = acts([(_lib.ACT_SIGMOID, 0, 0), (_lib.ACT_DECAY_GATE, 0x10000, 0x10010)])
    assert f(*args, segs, ok, 2, FAKE, 128, 0, 64, NUL) == _lib.NVFP4_OK          # M = 0
    none = ctypes.cast(None, ctypes.POINTER(_lib.SegmentAct))
    assert f(*args, segs, none, 2, FAKE, 128, 0, 64, NUL) == _lib.NVFP4_OK        # no table


def test_gemm_silu_mul_rejects_bad_arguments(L):
    f = L.nvfp4_gemm_silu_mul
    a = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)          # a_codes .. w_g, h
    assert f(*a, 256, 256, 256, 256, FAKE, FAKE, NUL, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE  # M <= 256
    assert f(*a, 256, 300, 200, 256, FAKE, FAKE, NUL, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE  # F % 128
    assert f(*a, 256, 300, 256, 100, FAKE, FAKE, NUL, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE  # K % 32
    assert f(*a, 128, 300, 256, 256, FAKE, FAKE, NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT          # ldh < F
    assert f(*a, 256, 300, 256, 256, NUL, FAKE, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG         # workspace
    assert f(*a, 256, 300, 256, 256, FAKE, NUL, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG         # h_g
    assert f(*a, 256, 300, 256, 256, ODD, FAKE, NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    WS = ctypes.c_void_p(0x40000)
    assert f(*a, 256, 300, 256, 256, WS, ctypes.c_void_p(0x40000 + 252), NUL, NUL) == \
        _lib.NVFP4_ERR_INVALID_ARG                                  # h_g inside the workspace


def test_silu_mul_rejects_bad_arguments(L):
    s = L.nvfp4_silu_mul
    assert s(FAKE, -1, 64, 128, FAKE, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert s(FAKE, 4, 60, 128, FAKE, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT      # f % 8
    assert s(FAKE, 4, 64, 120, FAKE, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG    # ld < 2f
    assert s(FAKE, 4, 64, 128, FAKE, 56, NUL) == _lib.NVFP4_ERR_INVALID_ARG    # ldh < f
    assert s(NUL, 4, 64, 128, FAKE, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert s(ODD, 4, 64, 128, FAKE, 64, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert s(FAKE, 0, 64, 128, FAKE, 64, NUL) == _lib.NVFP4_OK                 # nothing to do


def test_extents_that_would_overflow_are_refused(L):
    # sizes and strides whose byte products exceed any address space are
    # refused before any size arithmetic, instead of wrapping around
    big, wide = 1 << 30, 1 << 20
    assert L.nvfp4_global_scale(FAKE, big, 64, wide, FAKE, NUL, FAKE, NUL) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_quantize(FAKE, big, 64, wide, FAKE, FAKE, FAKE, 1, NUL) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    # 2^30 work items (1024-element chunks, padding rows included): beyond the
    # quantizer's walk bound, though the extents are fine
    P = ctypes.c_void_p
    assert L.nvfp4_quantize(FAKE, 1 << 26, 16384, 16384, P(1 << 44), P(1 << 42), P(1 << 43), 1, NUL) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_quantize_slice(FAKE, 4, 64, 64, FAKE, FAKE, FAKE, 1, 1 << 62, 1 << 62, NUL) == \
        _lib.NVFP4_ERR_INVALID_ARG                                              # offset + rows wraps
    assert L.nvfp4_kv_quantize_e4m3(FAKE, big, 64, wide, FAKE, FAKE, 64, NUL) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_silu_mul(FAKE, big, 64, wide, FAKE, 64, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_silu_mul(FAKE, 1, 1 << 62, 128, FAKE, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert L.nvfp4_gemm(*ok, wide, big, 128, 64, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    # 2^30 tiles of 128 x 128 or more: beyond the kernels' 32-bit tile indices
    # (an output of 2^47 bytes, under the extent bound, so this check decides)
    assert L.nvfp4_gemm(*ok, 1 << 23, 1 << 23, 1 << 23, 64, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_gemm_silu_mul(*ok, 1 << 62, 300, 1 << 62, 256, FAKE, FAKE, NUL, NUL) == \
        _lib.NVFP4_ERR_UNSUPPORTED_SHAPE


def test_debug_wait_rejects_bad_limits(L):
    assert L.nvfp4_debug_wait_timeout(0, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_debug_wait_timeout(2_000_000_000, NUL) == _lib.NVFP4_ERR_INVALID_ARG


def test_python_api_refuses_cpu_tensors():
    import torch
    import nvfp4_w4a4_quantized_09_b200 as nv
    with pytest.raises(ValueError):
        nv.quantize_tensor(torch.zeros(4, 64, dtype=torch.bfloat16))


def test_scalars_aliasing_an_output_are_refused(L):
    # a kernel reads these scalars while other CTAs write the output, so a
    # scalar inside the output's bytes is refused on the host (fake pointers,
    # never dereferenced)
    P = ctypes.c_void_p
    OUT, OUT2 = 0x50000, 0x60000
    # quantize: g inside the codes, or inside the scale bytes
    assert L.nvfp4_quantize(FAKE, 4, 64, 64, P(OUT + 16), P(OUT), P(OUT2), 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_quantize(FAKE, 4, 64, 64, P(OUT2 + 256), P(OUT), P(OUT2), 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # quantize: the codes, or the scale bytes, inside x (4 x 64 BF16 = 512 B)
    assert L.nvfp4_quantize(P(OUT), 4, 64, 64, P(0x20000), P(OUT + 256), P(OUT2), 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_quantize(P(OUT), 4, 64, 64, P(0x20000), P(OUT2), P(OUT + 496), 1, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # global scale: g_out inside x
    assert L.nvfp4_global_scale(P(OUT), 4, 64, 64, P(OUT + 256), NUL, FAKE, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # GEMM: the activation's scale inside y (4 x 128 BF16 = 1 KB)
    g = L.nvfp4_gemm
    assert g(FAKE, FAKE, P(OUT + 1000), FAKE, FAKE, FAKE, P(OUT), 128, 4, 128, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # fused GEMM: a module's scale inside y; a gate parameter array reaching into y
    f = L.nvfp4_fused_gemm
    segs = seg_array([(0, 64, 0x20000), (64, 64, OUT + 512)])
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, segs, 2, P(OUT), 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    fa = L.nvfp4_fused_gemm_act
    segs = seg_array([(0, 64, 0x20000), (64, 64, 0x20010)])
    acts = (_lib.SegmentAct * 2)()
    acts[1].kind, acts[1].a_log, acts[1].dt_bias = _lib.ACT_DECAY_GATE, OUT - 200, 0x30000   # 256 B: ends in y
    assert fa(FAKE, FAKE, FAKE, FAKE, FAKE, segs, acts, 2, P(OUT), 128, 4, 64, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # SiLU GEMM: an input scale inside h
    s = L.nvfp4_gemm_silu_mul
    assert s(FAKE, FAKE, P(OUT + 64), FAKE, FAKE, FAKE, P(OUT), 256, 300, 256, 256, P(0x40000),
             P(0x48000), NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # KV cache: the scale inside the output bytes
    assert L.nvfp4_kv_quantize_e4m3(FAKE, 4, 8, 8, P(OUT + 8), P(OUT), 8, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    # harmonisation: a module scale, or g_common, inside the scale bytes being rewritten
    h = L.nvfp4_harmonize_scales
    segs = seg_array([(0, 64, 0x20000), (64, 64, OUT + 100)])
    assert h(P(OUT), 64, segs, 2, _lib.SF_LINEAR, P(0x30000), NUL) == _lib.NVFP4_ERR_INVALID_ARG
    segs = seg_array([(0, 64, 0x20000), (64, 64, 0x20010)])
    assert h(P(OUT), 64, segs, 2, _lib.SF_LINEAR, P(OUT + 400), NUL) == _lib.NVFP4_ERR_INVALID_ARG


def test_fused_linear_host_rejects_bad_arguments_before_enqueuing(L):
    f = L.nvfp4_fused_linear_host
    P = ctypes.c_void_p
    segs = seg_array([(0, 64, 0x20000), (64, 64, 0x20010)])
    scratch = (P(0x100000), P(0x200000), P(0x300000), P(0x400000), P(0x410000), P(0x420000),
               P(0x500000))                                  # x_dev .. y_dev
    H = P(0x900000)                                          # host buffers (never touched)
    assert f(H, 4, 48, FAKE, FAKE, segs, 2, H, *scratch, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE  # K % 32
    odd = seg_array([(0, 64, 0x20000), (64, 60, 0x20010)])
    assert f(H, 4, 64, FAKE, FAKE, odd, 2, H, *scratch, NUL) == _lib.NVFP4_ERR_ALIGNMENT         # N % 8
    gap = seg_array([(0, 64, 0x20000), (72, 64, 0x20010)])
    assert f(H, 4, 64, FAKE, FAKE, gap, 2, H, *scratch, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert f(NUL, 4, 64, FAKE, FAKE, segs, 2, H, *scratch, NUL) == _lib.NVFP4_ERR_INVALID_ARG       # no x_host
    assert f(H, 4, 64, FAKE, FAKE, segs, 2, H, ODD, *scratch[1:], NUL) == _lib.NVFP4_ERR_ALIGNMENT
    same = (P(0x100000),) + scratch[1:6] + (P(0x100000),)   # y_dev on top of x_dev
    assert f(H, 4, 64, FAKE, FAKE, segs, 2, H, *same, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    g_in_codes = scratch[:3] + (P(0x200010),) + scratch[4:]  # a_g inside a_codes
    assert f(H, 4, 64, FAKE, FAKE, segs, 2, H, *g_in_codes, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    codes_in_x = scratch[:1] + (P(0x100100),) + scratch[2:]  # a_codes inside x_dev (512 B)
    assert f(H, 4, 64, FAKE, FAKE, segs, 2, H, *codes_in_x, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    sf_in_x = scratch[:2] + (P(0x1001F0),) + scratch[3:]     # a_sf reaching into x_dev
    assert f(H, 4, 64, FAKE, FAKE, segs, 2, H, *sf_in_x, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert f(H, 0, 64, FAKE, FAKE, segs, 2, H, *scratch, NUL) == _lib.NVFP4_OK                     # M = 0
    # the overlapped form makes the same checks before enqueuing anything
    o = L.nvfp4_fused_linear_host_overlap
    assert o(H, 4, 48, FAKE, FAKE, segs, 2, H, *scratch, NUL, NUL) == _lib.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert o(H, 4, 64, FAKE, FAKE, odd, 2, H, *scratch, NUL, NUL) == _lib.NVFP4_ERR_ALIGNMENT
    assert o(H, 4, 64, FAKE, FAKE, gap, 2, H, *scratch, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert o(NUL, 4, 64, FAKE, FAKE, segs, 2, H, *scratch, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert o(H, 4, 64, FAKE, FAKE, segs, 2, H, *same, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert o(H, 4, 64, FAKE, FAKE, segs, 2, H, *codes_in_x, NUL, NUL) == _lib.NVFP4_ERR_INVALID_ARG
    assert o(H, 0, 64, FAKE, FAKE, segs, 2, H, *scratch, NUL, NUL) == _lib.NVFP4_OK


def test_unused_gate_parameters_are_not_checked_for_aliasing(L):
    # a sigmoid segment's a_log is documented as unused: whatever it points at,
    # even inside y, does not refuse the call.  The decay segment has 300
    # columns (over the 256 the kernels stage), so the call still stops on the
    # host: NVFP4_ERR_CUDA here without a GPU, UNSUPPORTED_SHAPE on one --
    # never the aliasing refusal, and never a launch.
    P = ctypes.c_void_p
    Y = 0x50000
    segs = seg_array([(0, 64, 0x20000), (64, 300, 0x20010)])
    acts = (_lib.SegmentAct * 2)()
    acts[0].kind, acts[0].a_log, acts[0].dt_bias = _lib.ACT_SIGMOID, Y + 16, 0
    acts[1].kind, acts[1].a_log, acts[1].dt_bias = _lib.ACT_DECAY_GATE, 0x30000, 0x34000
    st = L.nvfp4_fused_gemm_act(FAKE, FAKE, FAKE, FAKE, FAKE, segs, acts, 2, P(Y), 368, 4, 64, NUL)
    assert st in (_lib.NVFP4_ERR_CUDA, _lib.NVFP4_ERR_UNSUPPORTED_SHAPE), st
