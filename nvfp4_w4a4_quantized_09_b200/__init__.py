"""NVFP4 W4A4 quantized linear layer for B200 (sm_100a).

Thin torch-facing wrappers over the C ABI in ``include/nvfp4.h``: PyTorch only
provides device memory and streams; every step of the path (global scale,
16-block quantization, block-scaled FP4 GEMM, scaled BF16 epilogue, fused
multi-module GEMM with per-module global scales) runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: if ``libnvfp4.so`` is missing,
the first call raises.

Method: the pages on "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4
W4A4 for the Recurrent Half of a Hybrid 27B LLM" -- NVFP4 (4-bit E2M1 elements,
16 of them sharing one E4M3 scale) on weights and activations of every linear layer
(evolve.pub review, Scope & Claims), served by fused multi-module GEMMs whose
per-module global scales must be honoured (chatpaper.ai abstract).
"""
from __future__ import annotations

import ctypes
import functools
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from . import _lib
from ._lib import SF_LINEAR, SF_TCGEN05, MAX_SEGMENTS, Nvfp4Error

__all__ = [
    "SF_LINEAR", "SF_TCGEN05", "MAX_SEGMENTS", "Nvfp4Error", "QuantizedTensor",
    "ACT_NONE", "ACT_DECAY_GATE", "ACT_SIGMOID",
    "global_scale", "sf_bytes", "quantize", "quantize_into", "quantize_tensor",
    "gemm", "fused_gemm", "FusedWeight", "linear", "silu_mul", "mlp", "interleave_gate_up", "gemm_silu_mul", "harmonize", "kv_scale", "kv_quantize", "last_device_status",
    "save_quantized", "load_quantized", "linear_host", "HostLinearScratch",
    "debug_wait_timeout", "library_path",
]


def library_path() -> str:
    """Path of the CUDA library the binding loads (built in-tree)."""
    return _lib.LIB_PATH


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------
# argument checks: the C ABI checks sizes, alignment and strides it is given,
# but it cannot see how large a caller's buffer is.  Every buffer is checked
# here for dtype, shape (or size) and device before the library is called.
# ---------------------------------------------------------------------------
def _check_bf16_matrix(x: torch.Tensor, name: str):
    if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError(f"{name} must be a 2-D bfloat16 tensor")
    if x.stride(1) != 1:
        raise ValueError(f"{name} must have unit stride along its last dimension")


def _check_out_matrix(t: torch.Tensor, name: str, dtype: torch.dtype, rows: int, cols: int):
    """A row-major output [rows, cols] with unit column stride; its row stride
    may be wider than cols (the library checks its alignment)."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise ValueError(f"{name} must be a {dtype} tensor")
    if t.shape != (rows, cols):
        raise ValueError(f"{name} must have shape ({rows}, {cols}), got {tuple(t.shape)}")
    if cols > 0 and (t.stride(1) != 1 or (rows > 1 and t.stride(0) < cols)):
        raise ValueError(f"{name} must be row-major with unit stride along its last dimension")


def _check_packed(t: torch.Tensor, name: str, shape=None, min_bytes: Optional[int] = None):
    """A contiguous uint8 buffer: packed codes of the given shape, or flat
    scale bytes of at least min_bytes."""
    if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous uint8 tensor")
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_bytes is not None and t.numel() < min_bytes:
        raise ValueError(f"{name} holds {t.numel()} bytes, {min_bytes} needed")


def _check_f32(t: torch.Tensor, name: str, numel: int = 1):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 tensor")
    if t.numel() < numel:
        raise ValueError(f"{name} must hold at least {numel} element(s), got {t.numel()}")


def _check_quantized(q: "QuantizedTensor", name: str):
    if q.cols % 2:
        raise ValueError(f"{name}.cols must be even")
    _check_packed(q.codes, f"{name}.codes", shape=(q.rows, q.cols // 2))
    _check_packed(q.sf, f"{name}.sf", min_bytes=_sf_bytes_cached(q.rows, q.cols, q.layout))
    _check_f32(q.g, f"{name}.g")


def _check_devices(**tensors) -> torch.device:
    """All tensors on the current CUDA device (the library launches on the
    current device's stream); returns that device."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other operands on {dev}")
    if dev is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"operands are on {dev} but the current device is cuda:"
                         f"{torch.cuda.current_device()}; call torch.cuda.set_device first")
    return dev


_workspaces = {}


def _workspace(device: torch.device, stream=None) -> torch.Tensor:
    """Zero-initialised global-scale workspace, one per (device, stream): each
    call leaves it zeroed again, and calls on one stream run in order, so
    calls on different streams never share one."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (idx, s.cuda_stream)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(_lib.GLOBAL_SCALE_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def sf_bytes(rows: int, cols: int, layout: int = SF_TCGEN05) -> int:
    """Bytes of the block-scale buffer of a [rows, cols] tensor in `layout`
    (the tensor-core layout pads rows to 128 and scale columns to 4)."""
    n = ctypes.c_size_t(0)
    _lib.check("nvfp4_sf_bytes", _lib.lib().nvfp4_sf_bytes(rows, cols, layout, ctypes.byref(n)))
    return int(n.value)


@functools.lru_cache(maxsize=1024)
def _sf_bytes_cached(rows: int, cols: int, layout: int) -> int:
    return sf_bytes(rows, cols, layout)


def global_scale(x: torch.Tensor, g_out: Optional[torch.Tensor] = None,
                 amax_out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """(g, amax) as 1-element FP32 device tensors: g = amax / (6 * 448)."""
    _check_bf16_matrix(x, "x")
    if g_out is not None:
        _check_f32(g_out, "g_out")
    if amax_out is not None:
        _check_f32(amax_out, "amax_out")
    if workspace is not None:
        _check_packed(workspace, "workspace", min_bytes=_lib.GLOBAL_SCALE_WORKSPACE_BYTES)
    dev = _check_devices(x=x, g_out=g_out, amax_out=amax_out, workspace=workspace)
    g_out = torch.empty(1, dtype=torch.float32, device=dev) if g_out is None else g_out
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    ws = _workspace(dev, stream) if workspace is None else workspace
    rows, cols = x.shape
    _lib.check("nvfp4_global_scale", _lib.lib().nvfp4_global_scale(
        _ptr(x), rows, cols, x.stride(0), _ptr(g_out), _ptr(amax_out), _ptr(ws), _stream(stream)))
    return g_out, amax_out


@dataclass
class QuantizedTensor:
    """Packed NVFP4 tensor: codes [rows, cols/2] uint8, block scales (flat,
    in ``layout``), and its FP32 global scale(s) in device memory."""
    codes: torch.Tensor
    sf: torch.Tensor
    g: torch.Tensor
    rows: int
    cols: int
    layout: int = SF_TCGEN05


def quantize(x: torch.Tensor, g: torch.Tensor, layout: int = SF_TCGEN05,
             codes: Optional[torch.Tensor] = None, sf: Optional[torch.Tensor] = None,
             stream=None):
    """Codes and block scales of x under the global scale g (device tensor)."""
    _check_bf16_matrix(x, "x")
    _check_f32(g, "g")
    rows, cols = x.shape
    if codes is not None:
        _check_packed(codes, "codes", shape=(rows, cols // 2))
    if sf is not None:
        _check_packed(sf, "sf", min_bytes=_sf_bytes_cached(rows, cols, layout))
    dev = _check_devices(x=x, g=g, codes=codes, sf=sf)
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(sf_bytes(rows, cols, layout), dtype=torch.uint8, device=dev)
    _lib.check("nvfp4_quantize", _lib.lib().nvfp4_quantize(
        _ptr(x), rows, cols, x.stride(0), _ptr(g), _ptr(codes), _ptr(sf), layout, _stream(stream)))
    return codes, sf


def quantize_into(x: torch.Tensor, g: torch.Tensor, codes: torch.Tensor, sf: torch.Tensor,
                  row_offset: int, total_rows: int, layout: int = SF_TCGEN05, stream=None):
    """Quantize x as rows [row_offset, row_offset + rows) of a larger tensor."""
    _check_bf16_matrix(x, "x")
    _check_f32(g, "g")
    rows, cols = x.shape
    if row_offset < 0 or row_offset + rows > total_rows:
        raise ValueError(f"rows [{row_offset}, {row_offset + rows}) outside [0, {total_rows})")
    _check_packed(codes, "codes", shape=(total_rows, cols // 2))
    _check_packed(sf, "sf", min_bytes=_sf_bytes_cached(total_rows, cols, layout))
    _check_devices(x=x, g=g, codes=codes, sf=sf)
    _lib.check("nvfp4_quantize_slice", _lib.lib().nvfp4_quantize_slice(
        _ptr(x), rows, cols, x.stride(0), _ptr(g), _ptr(codes), _ptr(sf), layout,
        row_offset, total_rows, _stream(stream)))


def quantize_tensor(x: torch.Tensor, layout: int = SF_TCGEN05, stream=None) -> QuantizedTensor:
    """Global scale from the absmax, then 16-block quantization."""
    g, _ = global_scale(x, stream=stream)
    codes, sf = quantize(x, g, layout, stream=stream)
    return QuantizedTensor(codes, sf, g, x.shape[0], x.shape[1], layout)


def gemm(a: QuantizedTensor, w: QuantizedTensor, y: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """y = a @ w.T in BF16 from NVFP4 operands (both in the tensor-core layout)."""
    if a.layout != SF_TCGEN05 or w.layout != SF_TCGEN05:
        raise ValueError("the GEMM reads block scales in the tensor-core layout")
    if a.cols != w.cols:
        raise ValueError("inner dimensions differ")
    M, K, N = a.rows, a.cols, w.rows
    _check_quantized(a, "a")
    _check_quantized(w, "w")
    if y is not None:
        _check_out_matrix(y, "y", torch.bfloat16, M, N)
    dev = _check_devices(a_codes=a.codes, a_sf=a.sf, a_g=a.g, w_codes=w.codes, w_sf=w.sf, w_g=w.g,
                         y=y)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    _lib.check("nvfp4_gemm", _lib.lib().nvfp4_gemm(
        _ptr(a.codes), _ptr(a.sf), _ptr(a.g), _ptr(w.codes), _ptr(w.sf), _ptr(w.g),
        _ptr(y), y.stride(0), M, N, K, _stream(stream)))
    return y


class FusedWeight:
    """Several modules' weights concatenated along N, each quantized with its
    own global scale -- the layout a fused multi-module GEMM serves."""

    def __init__(self, codes, sf, g_list, sizes, cols):
        self.codes = codes
        self.sf = sf
        self.g_list = list(g_list)
        self.sizes = list(sizes)
        self.cols = cols
        self.rows = sum(self.sizes)

    @classmethod
    def from_modules(cls, weights: Sequence[torch.Tensor], stream=None) -> "FusedWeight":
        if not 1 <= len(weights) <= MAX_SEGMENTS:
            raise ValueError(f"1..{MAX_SEGMENTS} modules")
        for i, w in enumerate(weights):
            _check_bf16_matrix(w, f"weights[{i}]")
        cols = weights[0].shape[1]
        total = sum(w.shape[0] for w in weights)
        dev = weights[0].device
        codes = torch.empty(total, cols // 2, dtype=torch.uint8, device=dev)
        sf = torch.empty(sf_bytes(total, cols, SF_TCGEN05), dtype=torch.uint8, device=dev)
        gs, off = [], 0
        for w in weights:
            if w.shape[1] != cols:
                raise ValueError("modules must share K")
            g, _ = global_scale(w, stream=stream)
            quantize_into(w, g, codes, sf, off, total, SF_TCGEN05, stream=stream)
            gs.append(g)
            off += w.shape[0]
        return cls(codes, sf, gs, [w.shape[0] for w in weights], cols)

    def segments(self):
        out, off = [], 0
        for n, g in zip(self.sizes, self.g_list):
            out.append((off, n, g))
            off += n
        return out


def _segment_array(segments):
    arr = (_lib.Segment * max(len(segments), 1))()
    for i, (off, n, g) in enumerate(segments):
        arr[i].n_offset = int(off)
        arr[i].n_size = int(n)
        arr[i].w_gscale = g.data_ptr()
    return arr


def harmonize(w: "FusedWeight", layout: int = SF_TCGEN05, stream=None) -> QuantizedTensor:
    """Checkpoint-side repair of the global-scale mismatch: a copy of the
    fused weight's block scales re-expressed against g_c = max_i g_i (codes
    shared, not copied), served afterwards by the single-scale GEMM."""
    _check_packed(w.sf, "w.sf", min_bytes=_sf_bytes_cached(w.rows, w.cols, layout))
    segs = w.segments()
    _check_segments(segs, w.rows)
    dev = _check_devices(w_sf=w.sf, **{f"g[{i}]": g for i, (_, _, g) in enumerate(segs)})
    sf = w.sf.clone()
    g_c = torch.empty(1, dtype=torch.float32, device=dev)
    _lib.check("nvfp4_harmonize_scales", _lib.lib().nvfp4_harmonize_scales(
        _ptr(sf), w.cols, _segment_array(segs), len(segs), layout, _ptr(g_c), _stream(stream)))
    return QuantizedTensor(w.codes, sf, g_c, w.rows, w.cols, layout)


def _check_segments(segments, n_total: Optional[int] = None):
    """Segments [(n_offset, n_size, g)] tile [0, N) in order, each g a float32
    scalar tensor; returns N."""
    if not 1 <= len(segments) <= MAX_SEGMENTS:
        raise ValueError(f"1..{MAX_SEGMENTS} segments")
    off = 0
    for i, (o, n, g) in enumerate(segments):
        if int(o) != off or int(n) <= 0:
            raise ValueError(f"segment {i} = [{int(o)}, {int(o) + int(n)}) does not continue at {off}")
        _check_f32(g, f"segments[{i}] global scale")
        off += int(n)
    if n_total is not None and off != n_total:
        raise ValueError(f"segments cover {off} rows, the weight has {n_total}")
    return off


ACT_NONE, ACT_DECAY_GATE, ACT_SIGMOID = _lib.ACT_NONE, _lib.ACT_DECAY_GATE, _lib.ACT_SIGMOID


def fused_gemm(a: QuantizedTensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
               segments: List, y: Optional[torch.Tensor] = None, stream=None,
               acts: Optional[List] = None) -> torch.Tensor:
    """Fused multi-module GEMM; segments = [(n_offset, n_size, g_tensor)].

    acts (optional, one per segment): (kind, a_log, dt_bias) with kind one of
    ACT_NONE, ACT_DECAY_GATE (a_log, dt_bias: FP32 device tensors of n_size),
    ACT_SIGMOID -- the Gated DeltaNet gate functions applied in the epilogue."""
    if a.layout != SF_TCGEN05:
        raise ValueError("the GEMM reads block scales in the tensor-core layout")
    nseg = len(segments)
    if acts is not None and len(acts) != nseg:
        raise ValueError("one activation entry per segment")
    N = _check_segments(segments)
    M, K = a.rows, a.cols
    _check_quantized(a, "a")
    _check_packed(w_codes, "w_codes", shape=(N, K // 2))
    _check_packed(w_sf, "w_sf", min_bytes=_sf_bytes_cached(N, K, SF_TCGEN05))
    if y is not None:
        _check_out_matrix(y, "y", torch.bfloat16, M, N)
    params = {}
    if acts is not None:
        for i, ((_, n, _), (kind, a_log, dt_bias)) in enumerate(zip(segments, acts)):
            if int(kind) == ACT_DECAY_GATE:
                if a_log is None or dt_bias is None:
                    raise ValueError(f"segment {i}: the decay gate needs a_log and dt_bias")
                _check_f32(a_log, f"acts[{i}].a_log", int(n))
                _check_f32(dt_bias, f"acts[{i}].dt_bias", int(n))
                params[f"acts[{i}].a_log"], params[f"acts[{i}].dt_bias"] = a_log, dt_bias
    dev = _check_devices(a_codes=a.codes, a_sf=a.sf, a_g=a.g, w_codes=w_codes, w_sf=w_sf, y=y,
                         **{f"segments[{i}] g": g for i, (_, _, g) in enumerate(segments)}, **params)
    arr = _segment_array(segments)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    if acts is None:
        _lib.check("nvfp4_fused_gemm", _lib.lib().nvfp4_fused_gemm(
            _ptr(a.codes), _ptr(a.sf), _ptr(a.g), _ptr(w_codes), _ptr(w_sf), arr, nseg,
            _ptr(y), y.stride(0), M, K, _stream(stream)))
        return y
    act_arr = (_lib.SegmentAct * max(nseg, 1))()
    for i, (kind, a_log, dt_bias) in enumerate(acts):
        act_arr[i].kind = int(kind)
        act_arr[i].a_log = 0 if a_log is None else a_log.data_ptr()
        act_arr[i].dt_bias = 0 if dt_bias is None else dt_bias.data_ptr()
    _lib.check("nvfp4_fused_gemm_act", _lib.lib().nvfp4_fused_gemm_act(
        _ptr(a.codes), _ptr(a.sf), _ptr(a.g), _ptr(w_codes), _ptr(w_sf), arr, act_arr, nseg,
        _ptr(y), y.stride(0), M, K, _stream(stream)))
    return y


def linear(x: torch.Tensor, w, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """W4A4 linear layer: quantize the BF16 activation x at run time, then the
    (fused) NVFP4 GEMM against a pre-quantized weight (QuantizedTensor or
    FusedWeight)."""
    a = quantize_tensor(x, stream=stream)
    if isinstance(w, FusedWeight):
        return fused_gemm(a, w.codes, w.sf, w.segments(), y, stream)
    return gemm(a, w, y, stream)


class HostLinearScratch:
    """Device scratch of linear_host for one (M, K, N): the activation copy,
    its codes, scales, global scale and amax, the global-scale workspace and
    the output before its copy back.  Reuse it across calls of that shape on
    one stream (its workspace is left zeroed by every call)."""

    def __init__(self, M: int, K: int, N: int, device):
        self.shape = (int(M), int(K), int(N))
        self.x = torch.empty(M, K, dtype=torch.bfloat16, device=device)
        self.codes = torch.empty(M, K // 2, dtype=torch.uint8, device=device)
        self.sf = torch.empty(sf_bytes(M, K), dtype=torch.uint8, device=device)
        self.g = torch.empty(1, dtype=torch.float32, device=device)
        self.amax = torch.empty(1, dtype=torch.float32, device=device)
        self.workspace = torch.zeros(_lib.GLOBAL_SCALE_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=device)


def linear_host(x_host: torch.Tensor, w, y_host: Optional[torch.Tensor] = None,
                scratch: Optional[HostLinearScratch] = None, stream=None,
                copy_stream=None) -> torch.Tensor:
    """The W4A4 linear layer from a host BF16 activation [M, K] to a host BF16
    output [M, N] through one C-ABI call: copy in, global scale, quantization,
    fused GEMM against the pre-quantized weight (FusedWeight or
    QuantizedTensor), copy out.  Without `copy_stream` everything runs on
    `stream` (nvfp4_fused_linear_host): synchronize it before reading y_host.
    With `copy_stream` (nvfp4_fused_linear_host_overlap) the output is copied
    out on that stream in row slices while the GEMM proceeds, and consecutive
    calls overlap one call's copy out with the next one's copy in: y_host is
    ready once copy_stream has passed the call.  The copies are asynchronous
    when the host tensors are page-locked."""
    if not isinstance(x_host, torch.Tensor) or x_host.dtype != torch.bfloat16 or x_host.dim() != 2 \
            or x_host.is_cuda or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous 2-D bfloat16 host tensor")
    if isinstance(w, FusedWeight):
        segments = w.segments()
    elif isinstance(w, QuantizedTensor):
        if w.layout != SF_TCGEN05:
            raise ValueError("the GEMM reads block scales in the tensor-core layout")
        segments = [(0, w.rows, w.g)]
    else:
        raise TypeError("w must be a FusedWeight or a QuantizedTensor")
    M, K = x_host.shape
    if K != w.cols:
        raise ValueError(f"x_host has {K} columns, the weight {w.cols}")
    N = _check_segments(segments, w.rows)
    _check_packed(w.codes, "w.codes", shape=(N, K // 2))
    _check_packed(w.sf, "w.sf", min_bytes=_sf_bytes_cached(N, K, SF_TCGEN05))
    if y_host is None:
        y_host = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True)
    elif (not isinstance(y_host, torch.Tensor) or y_host.dtype != torch.bfloat16 or y_host.is_cuda
          or y_host.shape != (M, N) or not y_host.is_contiguous()):
        raise ValueError(f"y_host must be a contiguous bfloat16 host tensor of shape ({M}, {N})")
    if scratch is None:
        scratch = HostLinearScratch(M, K, N, w.codes.device)
    elif scratch.shape != (M, K, N):
        raise ValueError(f"scratch is for {scratch.shape}, the call needs {(M, K, N)}")
    _check_devices(w_codes=w.codes, w_sf=w.sf, x=scratch.x, codes=scratch.codes, sf=scratch.sf,
                   g=scratch.g, workspace=scratch.workspace, y=scratch.y,
                   **{f"segments[{i}] g": g for i, (_, _, g) in enumerate(segments)})
    args = (_ptr(x_host), M, K, _ptr(w.codes), _ptr(w.sf), _segment_array(segments), len(segments),
            _ptr(y_host), _ptr(scratch.x), _ptr(scratch.codes), _ptr(scratch.sf), _ptr(scratch.g),
            _ptr(scratch.amax), _ptr(scratch.workspace), _ptr(scratch.y), _stream(stream))
    if copy_stream is None:
        _lib.check("nvfp4_fused_linear_host", _lib.lib().nvfp4_fused_linear_host(*args))
    else:
        _lib.check("nvfp4_fused_linear_host_overlap",
                   _lib.lib().nvfp4_fused_linear_host_overlap(*args, _stream(copy_stream)))
    return y_host


def silu_mul(gate_up: torch.Tensor, h: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """h = SiLU(gate_up[:, :f]) * gate_up[:, f:] in BF16 (the MLP intermediate)."""
    _check_bf16_matrix(gate_up, "gate_up")
    rows, two_f = gate_up.shape
    if two_f % 2:
        raise ValueError("gate_up must have an even number of columns")
    f = two_f // 2
    if h is not None:
        _check_out_matrix(h, "h", torch.bfloat16, rows, f)
    dev = _check_devices(gate_up=gate_up, h=h)
    if h is None:
        h = torch.empty(rows, f, dtype=torch.bfloat16, device=dev)
    _lib.check("nvfp4_silu_mul", _lib.lib().nvfp4_silu_mul(
        _ptr(gate_up), rows, f, gate_up.stride(0), _ptr(h), h.stride(0), _stream(stream)))
    return h


def interleave_gate_up(w_gate_up: torch.Tensor, block: int = 128) -> torch.Tensor:
    """Rows of a [2F, K] gate_up weight reordered into the 128-row-block
    interleave nvfp4_gemm_silu_mul reads: gate block b, then up block b.
    A row permutation of the BF16 weight before quantization (offline)."""
    two_f = w_gate_up.shape[0]
    f = two_f // 2
    if two_f % 2 or f % block:
        raise ValueError("gate_up rows must be 2F with F a multiple of 128")
    g = w_gate_up[:f].reshape(f // block, block, -1)
    u = w_gate_up[f:].reshape(f // block, block, -1)
    return torch.stack([g, u], dim=1).reshape(two_f, -1).contiguous()


def gemm_silu_mul(a: QuantizedTensor, w_interleaved: QuantizedTensor,
                  h: Optional[torch.Tensor] = None, stream=None):
    """h = SiLU(gate) * up straight from the gate_up GEMM's accumulators
    (weight rows interleaved by interleave_gate_up), with the global scale of h
    for its requantization.  Returns (h, g_h, amax_h)."""
    if a.layout != SF_TCGEN05 or w_interleaved.layout != SF_TCGEN05:
        raise ValueError("the GEMM reads block scales in the tensor-core layout")
    if a.cols != w_interleaved.cols:
        raise ValueError("inner dimensions differ")
    if w_interleaved.rows % 2:
        raise ValueError("the gate_up weight must have 2F rows")
    M, K, F = a.rows, a.cols, w_interleaved.rows // 2
    _check_quantized(a, "a")
    _check_quantized(w_interleaved, "w_interleaved")
    if h is not None:
        _check_out_matrix(h, "h", torch.bfloat16, M, F)
    dev = _check_devices(a_codes=a.codes, a_sf=a.sf, a_g=a.g, w_codes=w_interleaved.codes,
                         w_sf=w_interleaved.sf, w_g=w_interleaved.g, h=h)
    if h is None:
        h = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    g_h = torch.empty(1, dtype=torch.float32, device=dev)
    amax_h = torch.empty(1, dtype=torch.float32, device=dev)
    _lib.check("nvfp4_gemm_silu_mul", _lib.lib().nvfp4_gemm_silu_mul(
        _ptr(a.codes), _ptr(a.sf), _ptr(a.g), _ptr(w_interleaved.codes), _ptr(w_interleaved.sf),
        _ptr(w_interleaved.g), _ptr(h), h.stride(0), M, F, K, _ptr(_workspace(dev, stream)),
        _ptr(g_h), _ptr(amax_h), _stream(stream)))
    return h, g_h, amax_h


def mlp(x: torch.Tensor, w_gate_up, w_down, stream=None, interleaved: bool = False) -> torch.Tensor:
    """W4A4 SiLU-gated MLP: gate_up GEMM, SiLU(gate)*up, requantization, down GEMM.

    With ``interleaved=True`` the gate_up weight is a QuantizedTensor whose
    rows interleave_gate_up arranged: SiLU(gate)*up and the global scale of h
    then come out of the gate_up GEMM's epilogue (three launches instead of
    five; the BF16 gate_up output never reaches memory)."""
    if not interleaved:
        gu = linear(x, w_gate_up, stream=stream)
        h = silu_mul(gu, stream=stream)
        return linear(h, w_down, stream=stream)
    if not isinstance(w_gate_up, QuantizedTensor):
        raise TypeError("the interleaved gate_up weight must be a QuantizedTensor")
    h, g_h, _ = gemm_silu_mul(quantize_tensor(x, stream=stream), w_gate_up, stream=stream)
    codes, sf = quantize(h, g_h, stream=stream)
    return gemm(QuantizedTensor(codes, sf, g_h, h.shape[0], h.shape[1]), w_down, stream=stream)


def kv_scale(calibration: torch.Tensor, stream=None) -> torch.Tensor:
    """Calibrated per-tensor FP8 KV-cache scale fl32(amax / 448) of a BF16
    calibration tensor (device FP32, 1 element)."""
    _, amax = global_scale(calibration, stream=stream)
    s = torch.empty(1, dtype=torch.float32, device=calibration.device)
    _lib.check("nvfp4_kv_scale_from_amax",
               _lib.lib().nvfp4_kv_scale_from_amax(_ptr(amax), _ptr(s), _stream(stream)))
    return s


def kv_quantize(x: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Signed E4M3 bytes of x / scale (RNE, saturating at 448) as uint8 [rows, cols]."""
    _check_bf16_matrix(x, "x")
    _check_f32(scale, "scale")
    rows, cols = x.shape
    if out is not None:
        _check_out_matrix(out, "out", torch.uint8, rows, cols)
    dev = _check_devices(x=x, scale=scale, out=out)
    if out is None:
        out = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
    _lib.check("nvfp4_kv_quantize_e4m3", _lib.lib().nvfp4_kv_quantize_e4m3(
        _ptr(x), rows, cols, x.stride(0), _ptr(scale), _ptr(out), out.stride(0), _stream(stream)))
    return out


# ---------------------------------------------------------------------------
# the quantized weight format on disk: quantize (and harmonise) once offline,
# serve many times.  One torch file holding plain CPU tensors and integers
# (loadable with weights_only=True): packed codes, scale bytes in their
# layout, one FP32 global scale per module and the module row counts.
# ---------------------------------------------------------------------------
_FORMAT = "nvfp4-w4a4"
_FORMAT_VERSION = 1


def save_quantized(path: str, w) -> None:
    """Write a QuantizedTensor or FusedWeight (device or host tensors) to path."""
    if isinstance(w, FusedWeight):
        kind, sizes, gs, layout = "fused", list(w.sizes), list(w.g_list), SF_TCGEN05
    elif isinstance(w, QuantizedTensor):
        kind, sizes, gs, layout = "single", [w.rows], [w.g], w.layout
    else:
        raise TypeError("save_quantized takes a QuantizedTensor or a FusedWeight")
    g = torch.cat([t.detach().reshape(-1)[:1].to("cpu", torch.float32) for t in gs])
    torch.save({"format": _FORMAT, "version": _FORMAT_VERSION, "kind": kind,
                "rows": int(sum(sizes)), "cols": int(w.cols), "layout": int(layout),
                "sizes": [int(n) for n in sizes],
                "codes": w.codes.detach().to("cpu").contiguous(),
                "sf": w.sf.detach().to("cpu").contiguous(), "g": g}, path)


def load_quantized(path: str, device="cuda"):
    """Read what save_quantized wrote, onto `device`; every field is checked
    against the others (shapes, scale bytes for the layout, one scale per
    module) before anything is returned."""
    d = torch.load(path, map_location="cpu", weights_only=True)
    if not isinstance(d, dict) or d.get("format") != _FORMAT or d.get("version") != _FORMAT_VERSION:
        raise ValueError(f"{path}: not an {_FORMAT} v{_FORMAT_VERSION} file")
    rows, cols, layout, sizes = d["rows"], d["cols"], d["layout"], d["sizes"]
    if layout not in (SF_LINEAR, SF_TCGEN05) or cols % 32 or sum(sizes) != rows or \
            any(n <= 0 for n in sizes) or d["kind"] not in ("single", "fused"):
        raise ValueError(f"{path}: inconsistent header")
    _check_packed(d["codes"], "codes", shape=(rows, cols // 2))
    _check_packed(d["sf"], "sf", min_bytes=_sf_bytes_cached(rows, cols, layout))
    if d["sf"].numel() != _sf_bytes_cached(rows, cols, layout):
        raise ValueError(f"{path}: {d['sf'].numel()} scale bytes for a [{rows}, {cols}] weight")
    _check_f32(d["g"], "g", len(sizes))
    if d["g"].numel() != len(sizes) or not bool(torch.isfinite(d["g"]).all()) or \
            not bool((d["g"] > 0).all()):
        raise ValueError(f"{path}: one positive finite global scale per module expected")
    codes, sf = d["codes"].to(device), d["sf"].to(device)
    g = [d["g"][i:i + 1].clone().to(device) for i in range(len(sizes))]
    if d["kind"] == "fused":
        if layout != SF_TCGEN05:
            raise ValueError(f"{path}: a fused weight is stored in the tensor-core layout")
        return FusedWeight(codes, sf, g, sizes, cols)
    if len(sizes) != 1:
        raise ValueError(f"{path}: a single tensor has one module")
    return QuantizedTensor(codes, sf, g[0], rows, cols, layout)


def last_device_status(stream=None) -> int:
    """Synchronize and return (and clear) the device status: 0 ok, 5 timeout."""
    return int(_lib.lib().nvfp4_last_device_status(_stream(stream)))


def debug_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch one warp whose first thread waits on a barrier that nothing
    arrives on.  The bounded wait gives up after limit_ns, so the device
    status then reads 5 (timeout) through last_device_status() and the
    context stays usable: the failure path of every kernel's waits,
    exercised without a fault."""
    _lib.check("nvfp4_debug_wait_timeout",
               _lib.lib().nvfp4_debug_wait_timeout(int(limit_ns), _stream(stream)))
