"""Run one kernel of the path on a named workload a few times (for profilers).

    python -m nvfp4_w4a4_quantized_09_b200.profile_cases CASE [LAUNCHES]

CASE:
  gemm_gdn        fused GEMM, X [8192,5120] x W q/k/v/z/b/a [24704,5120]
  gemm_gateup     GEMM, X [8192,5120] x W [34816,5120]
  gemm_decode     fused GEMM, X [32,5120] x W [24640,5120]
  gemm_decode_m1  fused GEMM, X [1,5120] x W [24640,5120]
  quantize_act    quantizer on the activation [32768,5120]
  global_scale_act  global scale of the activation [32768,5120]

Inputs are built first (their kernels run before the profiled ones); each
case then launches its kernel LAUNCHES times (default 3) and synchronizes.
"""
from __future__ import annotations

import sys

import torch

import nvfp4_w4a4_quantized_09_b200 as nv
from nvfp4_w4a4_quantized_09_b200 import synth


def main(case: str, launches: int = 3) -> None:
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if case in ("gemm_gdn", "gemm_decode", "gemm_decode_m1"):
        M = {"gemm_gdn": 8192, "gemm_decode": 32, "gemm_decode_m1": 1}[case]
        mods = synth.GDN_MODULES if case == "gemm_gdn" else synth.GDN_MODULES_DECODE
        x = synth.student_t_activations(M, 5120, seed=3, device=dev)
        fw = nv.FusedWeight.from_modules([w for _, w in synth.gdn_weights(mods, device=dev)])
        a = nv.quantize_tensor(x)
        segs = fw.segments()
        y = torch.empty(M, fw.rows, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        for _ in range(launches):
            nv.fused_gemm(a, fw.codes, fw.sf, segs, y)
    elif case == "gemm_gateup":
        x = synth.student_t_activations(8192, 5120, seed=1, device=dev)
        w = synth.gaussian_weights(34816, 5120, 0.015, seed=20, device=dev)
        a, wq = nv.quantize_tensor(x), nv.quantize_tensor(w)
        y = torch.empty(8192, 34816, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        for _ in range(launches):
            nv.gemm(a, wq, y)
    elif case in ("quantize_act", "global_scale_act"):
        x = synth.student_t_activations(32768, 5120, seed=1, device=dev)
        g, amax = nv.global_scale(x)
        codes = torch.empty(32768, 2560, dtype=torch.uint8, device=dev)
        sf = torch.empty(nv.sf_bytes(32768, 5120), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        for _ in range(launches):
            if case == "quantize_act":
                nv.quantize(x, g, nv.SF_TCGEN05, codes, sf)
            else:
                nv.global_scale(x, g, amax)
    else:
        raise SystemExit(f"unknown case {case!r}")
    torch.cuda.synchronize()
    status = nv.last_device_status()
    if status != 0:
        raise SystemExit(f"device status {status}")


if __name__ == "__main__":
    main(sys.argv[1], int(sys.argv[2]) if len(sys.argv) > 2 else 3)
