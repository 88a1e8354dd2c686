"""The allocation-free global scale, nvfp4_global_scale_noalloc.

Some callers cannot allocate device memory (a host framework whose pool
forbids outside cudaMalloc calls, a hook that runs where allocation is not
permitted), so they cannot pass the workspace nvfp4_global_scale needs; this
entry point keeps that workspace in a library-owned device array instead.
Called through the C ABI, twice in a row on different tensors (the second
call must not see the first call's leftovers), it must give exactly the
global scale and absmax of the workspace-taking entry point.  The file is
named to be collected last; it passes alone in a fresh process too, where its
first call also performs the per-device set-up.
"""
import ctypes

import pytest
import torch

from nvfp4_w4a4_quantized_09_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def with_workspace(x):
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    amax = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = torch.zeros(_lib.GLOBAL_SCALE_WORKSPACE_BYTES, dtype=torch.uint8, device=DEV)
    st = _lib.lib().nvfp4_global_scale(
        ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0),
        ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(amax.data_ptr()),
        ctypes.c_void_p(ws.data_ptr()), _stream())
    assert st == _lib.NVFP4_OK
    return g, amax


def without_allocation(x):
    g = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    st = _lib.lib().nvfp4_global_scale_noalloc(
        ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0),
        ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(amax.data_ptr()), _stream())
    assert st == _lib.NVFP4_OK
    return g, amax


def test_noalloc_matches_workspace_entry_point_twice():
    # a large tensor first, then a much smaller one: a stale maximum left in
    # the shared array would show up in the second result
    x1 = synth.student_t_activations(4096, 5120, seed=21, device=DEV)
    x2 = synth.student_t_activations(300, 256, seed=22, device=DEV) * 1e-3
    x2 = x2.to(torch.bfloat16)
    for x in (x1, x2):
        g_ref, a_ref = with_workspace(x)
        g, a = without_allocation(x)
        torch.cuda.synchronize()
        assert torch.equal(g.view(torch.int32), g_ref.view(torch.int32))
        assert torch.equal(a.view(torch.int32), a_ref.view(torch.int32))
    assert _lib.lib().nvfp4_last_device_status(_stream()) == _lib.NVFP4_OK


def test_noalloc_rejects_missing_output():
    x = torch.ones(4, 64, dtype=torch.bfloat16, device=DEV)
    st = _lib.lib().nvfp4_global_scale_noalloc(
        ctypes.c_void_p(x.data_ptr()), 4, 64, 64, ctypes.c_void_p(0), ctypes.c_void_p(0), _stream())
    assert st == _lib.NVFP4_ERR_INVALID_ARG
