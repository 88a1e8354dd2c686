"""Few-token GEMMs issued back to back on one stream.  Each is launched as a
programmatic dependent of the kernel before it (its CTAs may start while that
kernel drains) and waits for it before reading global memory.  A chain whose
every GEMM consumes the previous GEMM's output, through the activation
quantizer, must give the same bits with no host synchronisation, eagerly and
replayed from a CUDA graph, as with a synchronisation after every step."""
import pytest
import torch

import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _chain(x, weights, sync):
    for w in weights:
        a = nv.quantize_tensor(x)
        x = nv.gemm(a, w)
        if sync:
            torch.cuda.synchronize()
    return x


@pytest.mark.parametrize("M,K", [(1, 5120), (24, 2048), (128, 5120)])
def test_dependent_chain_matches_stepwise(M, K):
    weights = [nv.quantize_tensor(synth.gaussian_weights(K, K, 0.02, seed=70 + i, device=DEV))
               for i in range(4)]
    x0 = synth.student_t_activations(M, K, seed=80 + M, device=DEV)
    torch.cuda.synchronize()
    ref = _chain(x0, weights, sync=True)
    got = _chain(x0, weights, sync=False)
    torch.cuda.synchronize()
    assert nv.last_device_status() == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_dependent_chain_in_a_graph():
    M, K = 8, 5120
    weights = [nv.quantize_tensor(synth.gaussian_weights(K, K, 0.02, seed=90 + i, device=DEV))
               for i in range(3)]
    x0 = synth.student_t_activations(M, K, seed=99, device=DEV)
    torch.cuda.synchronize()
    ref = _chain(x0, weights, sync=True)
    static_x = x0.clone()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        _chain(static_x, weights, sync=False)        # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = _chain(static_x, weights, sync=False)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert nv.last_device_status() == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
