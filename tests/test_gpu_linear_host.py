"""The whole layer through one C-ABI call with host buffers
(nvfp4_fused_linear_host): the host output equals, bit for bit, the device
path (global scale, quantize, fused GEMM) on the same activation, for a
fused weight and a single tensor, with a scratch reused across calls."""
import pytest
import torch

import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_host_buffers_give_the_device_path_bitwise():
    K = 512
    mods = [synth.gaussian_weights(n, K, s, seed=400 + i, device=DEV)
            for i, (n, s) in enumerate([(256, 0.02), (64, 0.2), (64, 0.002)])]
    fw = nv.FusedWeight.from_modules(mods)
    wq = nv.quantize_tensor(mods[0])
    for M in (5, 300):
        x = synth.student_t_activations(M, K, seed=401 + M, device=DEV)
        x_host = x.cpu().pin_memory()
        for w in (fw, wq):
            scratch = nv.HostLinearScratch(M, K, w.rows, DEV)
            for _ in range(2):                               # scratch reused
                y_host = nv.linear_host(x_host, w, scratch=scratch)
                torch.cuda.synchronize()
                y_dev = nv.linear(x, w)
                torch.cuda.synchronize()
                assert torch.equal(y_host.view(torch.int16), y_dev.cpu().view(torch.int16))
    assert nv.last_device_status() == 0


def test_overlapped_host_call_gives_the_device_path_bitwise():
    # nvfp4_fused_linear_host_overlap: copy out on a second stream in row
    # slices.  M = 5000 takes two GEMM slices (2048 + 2952 rows); consecutive
    # calls reuse one scratch with different activations and alternate two
    # host outputs, so each call's GEMM must wait for the previous call's copy
    # out of the shared device output.
    K = 512
    mods = [synth.gaussian_weights(n, K, s, seed=410 + i, device=DEV)
            for i, (n, s) in enumerate([(256, 0.02), (64, 0.2), (64, 0.002)])]
    fw = nv.FusedWeight.from_modules(mods)
    copy_stream = torch.cuda.Stream()
    for M in (5, 300, 5000):
        xs = [synth.student_t_activations(M, K, seed=411 + M + i, device=DEV) for i in range(3)]
        x_hosts = [x.cpu().pin_memory() for x in xs]
        y_hosts = [torch.empty(M, fw.rows, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
        scratch = nv.HostLinearScratch(M, K, fw.rows, DEV)
        for i in range(3):
            nv.linear_host(x_hosts[i], fw, y_hosts[i], scratch=scratch, copy_stream=copy_stream)
        torch.cuda.synchronize()
        for i in range(3):
            y_dev = nv.linear(xs[i], fw)
            torch.cuda.synchronize()
            assert torch.equal(y_hosts[i].view(torch.int16), y_dev.cpu().view(torch.int16)), (M, i)
    assert nv.last_device_status() == 0
