"""B200-native NVFP4 W4A4 linear layers: Python binding of ``libnvfp4.so``.

The functions named ``nvfp4_*`` mirror the C ABI of ``include/nvfp4.h`` one to
one (raw device pointers as ints, sizes, scales, a CUDA stream handle) and do
argument marshalling only.  The helpers without the prefix (``quantize``,
``gemm``, ``gemm_quant``, ``swizzle_sf``) take torch tensors, allocate the
outputs with torch (device memory is the only thing torch provides here) and
call the same entry points on the current torch stream; every tensor they
pass on, the caller's own output buffers included, is checked first (dtype,
contiguity, current device, enough elements for what the kernel touches).  Every step of the
computation runs in the library's CUDA kernels; there is no fallback: the
first call raises ImportError if the library was not built.

Build the library with ``python -m nvfp4_block_scaled_12_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

NVFP4_OK, NVFP4_EINVAL, NVFP4_EALIGN, NVFP4_EARCH, NVFP4_ECUDA, NVFP4_ETIMEOUT = range(6)
ACT_NONE, ACT_GELU_TANH = 0, 1
DST_BF16, DST_NVFP4 = 0, 1
MAX_RANGES = 8
NVFP4_DYNAMIC_WORKSPACE_BYTES = 8
NVFP4_NOALLOC_SCRATCH_BYTES = 256

_STATUS_NAMES = {0: "NVFP4_OK", 1: "NVFP4_EINVAL", 2: "NVFP4_EALIGN", 3: "NVFP4_EARCH", 4: "NVFP4_ECUDA",
                 5: "NVFP4_ETIMEOUT"}


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class ColRange(ctypes.Structure):
    """``nvfp4_colrange``: one column range of the fused epilogue."""
    _fields_ = [("begin", ctypes.c_int64), ("end", ctypes.c_int64), ("act", ctypes.c_int32),
                ("dst", ctypes.c_int32), ("dst_col", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m nvfp4_block_scaled_12_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, f32, vp, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32
    lib.nvfp4_sf_bytes.argtypes = [i64, i64]
    lib.nvfp4_sf_bytes.restype = ctypes.c_size_t
    lib.nvfp4_calibrate.argtypes = [vp, i64, vp, vp]
    lib.nvfp4_quantize.argtypes = [vp, i64, i64, f32, vp, vp, vp]
    lib.nvfp4_swizzle_sf.argtypes = [vp, i64, i64, vp, vp]
    lib.nvfp4_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, vp, vp, vp]
    lib.nvfp4_gemm_quant.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, vp, ctypes.POINTER(ColRange), i32,
                                     vp, i64, f32, vp, vp, i64, vp]
    lib.nvfp4_quantize_dynamic.argtypes = [vp, i64, i64, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.nvfp4_gemm_dynamic.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, vp, vp, vp, vp]
    lib.nvfp4_gemm_scaled.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, f32, vp, vp, vp]
    lib.nvfp4_gemm_amax.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, vp, f32, vp, vp, vp, vp]
    lib.nvfp4_quantize_from_amax.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
    lib.nvfp4_gemm_quant_scaled.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, f32, vp, ctypes.POINTER(ColRange),
                                            i32, vp, i64, f32, vp, vp, i64, vp]
    lib.nvfp4_testing_set_grid_wait.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
    lib.nvfp4_quantize_dynamic_noalloc.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    lib.nvfp4_mxfp8_sf_bytes.argtypes = [i64, i64]
    lib.nvfp4_mxfp8_sf_bytes.restype = ctypes.c_size_t
    lib.nvfp4_mxfp8_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.nvfp4_mxfp8_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, f32, vp, vp, vp]
    lib.nvfp4_fp8row_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.nvfp4_fp8row_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp]
    lib.nvfp4_dequantize.argtypes = [vp, vp, f32, i64, i64, vp, vp]
    lib.nvfp4_w4a16_gemm.argtypes = [vp, vp, vp, i64, i64, i64, f32, vp, vp, vp]
    lib.nvfp4_check_fault.argtypes = []
    lib.nvfp4_gemm_tile_shape.argtypes = [i64, i64, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.nvfp4_gemm_plan.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.nvfp4_quantize_tile_rows.argtypes = [i64, i64, i32]
    lib.nvfp4_quantize_tile_rows.restype = ctypes.c_int32
    for name in ("nvfp4_calibrate", "nvfp4_quantize", "nvfp4_swizzle_sf", "nvfp4_gemm", "nvfp4_gemm_quant",
                 "nvfp4_quantize_dynamic", "nvfp4_gemm_dynamic", "nvfp4_quantize_dynamic_noalloc",
                 "nvfp4_mxfp8_quantize", "nvfp4_mxfp8_gemm", "nvfp4_fp8row_quantize", "nvfp4_fp8row_gemm",
                 "nvfp4_dequantize", "nvfp4_check_fault", "nvfp4_gemm_tile_shape", "nvfp4_gemm_scaled",
                 "nvfp4_gemm_quant_scaled", "nvfp4_testing_set_grid_wait", "nvfp4_w4a16_gemm",
                 "nvfp4_gemm_plan", "nvfp4_gemm_amax", "nvfp4_quantize_from_amax"):
        getattr(lib, name).restype = ctypes.c_int
    lib.nvfp4_last_error.argtypes = []
    lib.nvfp4_last_error.restype = ctypes.c_char_p
    return lib


_lib_handle: Optional[ctypes.CDLL] = None


def library() -> ctypes.CDLL:
    """The loaded ``libnvfp4.so`` (loaded on first use)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


def _check(status: int) -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(status, nvfp4_last_error())


# --------------------------------------------------------------------------
# 1:1 mirrors of the C ABI (pointers and streams as ints; 0 = NULL)
# --------------------------------------------------------------------------

def nvfp4_sf_bytes(rows: int, k: int) -> int:
    return int(library().nvfp4_sf_bytes(rows, k))


def nvfp4_calibrate(x: int, n: int, out: int, stream: int) -> None:
    _check(library().nvfp4_calibrate(x, n, out, stream))


def nvfp4_quantize(x: int, M: int, K: int, g: float, codes: int, sf: int, stream: int) -> None:
    _check(library().nvfp4_quantize(x, M, K, g, codes, sf, stream))


def nvfp4_quantize_dynamic(x: int, M: int, K: int, codes: int, sf: int, scale_out: int, workspace: int,
                           workspace_bytes: int, stream: int) -> None:
    _check(library().nvfp4_quantize_dynamic(x, M, K, codes, sf, scale_out, workspace, workspace_bytes, stream))


def nvfp4_quantize_dynamic_noalloc(x: int, M: int, K: int, codes: int, sf: int, scale_out: int, stream: int) -> None:
    _check(library().nvfp4_quantize_dynamic_noalloc(x, M, K, codes, sf, scale_out, stream))


def nvfp4_quantize_from_amax(x: int, M: int, K: int, amax: int, codes: int, sf: int, scale_out: int,
                             stream: int) -> None:
    _check(library().nvfp4_quantize_from_amax(x, M, K, amax, codes, sf, scale_out, stream))


def nvfp4_swizzle_sf(sf_linear: int, rows: int, k: int, sf_swizzled: int, stream: int) -> None:
    _check(library().nvfp4_swizzle_sf(sf_linear, rows, k, sf_swizzled, stream))


def nvfp4_gemm(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, alpha: float, bias: int, y: int,
               stream: int) -> None:
    _check(library().nvfp4_gemm(a, sfa, b, sfb, M, N, K, alpha, bias or None, y, stream))


def nvfp4_gemm_scaled(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, g_a: float, g_b: float,
                      bias: int, y: int, stream: int) -> None:
    _check(library().nvfp4_gemm_scaled(a, sfa, b, sfb, M, N, K, g_a, g_b, bias or None, y, stream))


def nvfp4_gemm_amax(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, g_a: float, g_a_device: int,
                    g_b: float, bias: int, y: int, amax_out: int, stream: int) -> None:
    _check(library().nvfp4_gemm_amax(a, sfa, b, sfb, M, N, K, g_a, g_a_device or None, g_b, bias or None, y,
                                     amax_out, stream))


def nvfp4_gemm_dynamic(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, g_b: float, g_a: int,
                       bias: int, y: int, stream: int) -> None:
    _check(library().nvfp4_gemm_dynamic(a, sfa, b, sfb, M, N, K, g_b, g_a, bias or None, y, stream))


def nvfp4_gemm_quant(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, alpha: float, bias: int,
                     ranges: Sequence[ColRange], y_bf16: int, ldy: int, g_next: float, codes_next: int,
                     sf_next: int, k_next: int, stream: int) -> None:
    arr = (ColRange * len(ranges))(*ranges)
    _check(library().nvfp4_gemm_quant(a, sfa, b, sfb, M, N, K, alpha, bias or None, arr, len(ranges), y_bf16 or None,
                                 ldy, g_next, codes_next or None, sf_next or None, k_next, stream))


def nvfp4_gemm_quant_scaled(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, g_a: float, g_b: float,
                            bias: int, ranges: Sequence[ColRange], y_bf16: int, ldy: int, g_next: float,
                            codes_next: int, sf_next: int, k_next: int, stream: int) -> None:
    arr = (ColRange * len(ranges))(*ranges)
    _check(library().nvfp4_gemm_quant_scaled(a, sfa, b, sfb, M, N, K, g_a, g_b, bias or None, arr, len(ranges),
                                             y_bf16 or None, ldy, g_next, codes_next or None, sf_next or None, k_next,
                                             stream))


def nvfp4_testing_set_grid_wait(limit_ns: int, extra_arrivals: int) -> None:
    _check(library().nvfp4_testing_set_grid_wait(limit_ns, extra_arrivals))


def nvfp4_mxfp8_sf_bytes(rows: int, k: int) -> int:
    return int(library().nvfp4_mxfp8_sf_bytes(rows, k))


def nvfp4_mxfp8_quantize(x: int, M: int, K: int, codes: int, sf: int, stream: int) -> None:
    _check(library().nvfp4_mxfp8_quantize(x, M, K, codes, sf, stream))


def nvfp4_mxfp8_gemm(a: int, sfa: int, b: int, sfb: int, M: int, N: int, K: int, alpha: float, bias: int, y: int,
                     stream: int) -> None:
    _check(library().nvfp4_mxfp8_gemm(a, sfa, b, sfb, M, N, K, alpha, bias or None, y, stream))


def nvfp4_fp8row_quantize(x: int, M: int, K: int, codes: int, scale: int, stream: int) -> None:
    _check(library().nvfp4_fp8row_quantize(x, M, K, codes, scale, stream))


def nvfp4_fp8row_gemm(a: int, a_scale: int, b: int, b_scale: int, M: int, N: int, K: int, bias: int, y: int,
                      stream: int) -> None:
    _check(library().nvfp4_fp8row_gemm(a, a_scale, b, b_scale, M, N, K, bias or None, y, stream))


def nvfp4_dequantize(codes: int, sf: int, g: float, rows: int, K: int, out: int, stream: int) -> None:
    _check(library().nvfp4_dequantize(codes, sf, g, rows, K, out, stream))


def nvfp4_w4a16_gemm(x: int, w_codes: int, w_sf: int, M: int, N: int, K: int, g_w: float, bias: int, y: int,
                     stream: int) -> None:
    _check(library().nvfp4_w4a16_gemm(x, w_codes, w_sf, M, N, K, g_w, bias or None, y, stream))


def nvfp4_check_fault() -> None:
    _check(library().nvfp4_check_fault())


def nvfp4_gemm_tile_shape(M: int, N: int, num_sms: int) -> tuple:
    """(CTAs per tile, tile width, accumulator buffers) the GEMMs take for M x N."""
    out = (ctypes.c_int32 * 3)()
    _check(library().nvfp4_gemm_tile_shape(M, N, num_sms, out))
    return tuple(out)


def nvfp4_gemm_plan(M: int, N: int, K: int, num_sms: int, w4a16: int = 0) -> tuple:
    """(CTAs per tile, tile width, accumulator buffers, K split) the plain-epilogue
    GEMMs (w4a16 = 0: NVFP4; 1: W4A16) take for M x N x K."""
    out = (ctypes.c_int32 * 4)()
    _check(library().nvfp4_gemm_plan(M, N, K, num_sms, w4a16, out))
    return tuple(out)


def nvfp4_quantize_tile_rows(M: int, K: int, num_sms: int) -> int:
    return int(library().nvfp4_quantize_tile_rows(M, K, num_sms))


def nvfp4_last_error() -> str:
    return library().nvfp4_last_error().decode()


# --------------------------------------------------------------------------
# torch-tensor helpers (outputs allocated with torch on the input's device)
# --------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream(stream) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _need(t, dtype, shape, name, min_numel=None, dev=None):
    """``t`` must be a contiguous CUDA tensor of ``dtype`` on the current
    device, of ``shape`` (if given) and with at least ``min_numel`` elements
    (if given): the library reads and writes through its raw pointer."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {min_numel} needed")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    dev = torch.cuda.current_device() if dev is None else dev
    if t.device.index != dev:
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{dev}")


def _need_nvfp4(t, name, rows=None, k=None, dev=None):
    """An NVFP4Tensor whose buffers hold ``rows`` x ``k`` elements (its own
    rows and k when not given)."""
    rows = t.rows if rows is None else rows
    k = t.k if k is None else k
    torch = _torch()
    if (t.rows, t.k) != (rows, k):
        raise ValueError(f"{name} is [{t.rows}, {t.k}], [{rows}, {k}] needed")
    _need(t.codes, torch.uint8, None, f"{name}.codes", rows * k // 2, dev=dev)
    _need(t.sf, torch.uint8, None, f"{name}.sf", nvfp4_sf_bytes(rows, k), dev=dev)
    if t.g is None:  # the scale measured on the device: [amax, g]
        _need(t.scale, torch.float32, None, f"{name}.scale", 2, dev=dev)


@dataclass
class NVFP4Tensor:
    """A [rows, k] NVFP4 tensor on the GPU: packed codes, swizzled scales and
    the per-tensor decode scale g -- a host float, or for a scale measured on
    the device (quantize_dynamic) ``g = None`` and ``scale`` = the float32
    device tensor [amax, g]."""
    codes: "object"   # uint8 [rows, k/2]
    sf: "object"      # uint8 [nvfp4_sf_bytes(rows, k)]
    g: Optional[float]
    rows: int
    k: int
    scale: "object" = None


def calibrate(x, stream=None):
    """Per-tensor scale of bf16 ``x`` on the GPU.  Returns a float32 CUDA
    tensor [amax, g] with g = amax / 2688 (nothing is read back)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    _need(x, torch.bfloat16, None, "x", dev=dev)
    out = torch.empty(2, dtype=torch.float32, device=x.device)
    nvfp4_calibrate(_ptr(x), x.numel(), _ptr(out), _stream(stream))
    return out


def global_scale(x, stream=None) -> float:
    """g = amax(|x|) / 2688 computed on the GPU, read back as a Python float."""
    return float(calibrate(x, stream)[1].item())


def quantize(x, g: float, out: Optional[NVFP4Tensor] = None, stream=None) -> NVFP4Tensor:
    """Quantize bf16 ``x`` [M, K] to NVFP4 with per-tensor decode scale g."""
    torch = _torch()
    dev = torch.cuda.current_device()
    M, K = x.shape
    _need(x, torch.bfloat16, None, "x", dev=dev)
    if out is None:
        out = NVFP4Tensor(torch.empty(M, K // 2, dtype=torch.uint8, device=x.device),
                          torch.empty(nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=x.device), float(g), M, K)
    else:
        _need(out.codes, torch.uint8, None, "out.codes", M * K // 2, dev=dev)
        _need(out.sf, torch.uint8, None, "out.sf", nvfp4_sf_bytes(M, K), dev=dev)
        if (out.rows, out.k) != (M, K):
            raise ValueError(f"out is [{out.rows}, {out.k}], x is [{M}, {K}]")
    nvfp4_quantize(_ptr(x), M, K, float(g), _ptr(out.codes), _ptr(out.sf), _stream(stream))
    out.g = float(g)
    return out


def quantize_dynamic(x, out: Optional[NVFP4Tensor] = None, workspace=None, stream=None) -> NVFP4Tensor:
    """Quantize bf16 ``x`` [M, K] with the per-tensor scale measured on x in
    the same launch (g = amax/2688, clamped; nothing is read back).  The
    result's ``scale`` holds [amax, g] on the device."""
    torch = _torch()
    dev = torch.cuda.current_device()
    M, K = x.shape
    _need(x, torch.bfloat16, None, "x", dev=dev)
    if out is None:
        out = NVFP4Tensor(torch.empty(M, K // 2, dtype=torch.uint8, device=x.device),
                          torch.empty(nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=x.device), None, M, K)
    else:
        _need(out.codes, torch.uint8, None, "out.codes", M * K // 2, dev=dev)
        _need(out.sf, torch.uint8, None, "out.sf", nvfp4_sf_bytes(M, K), dev=dev)
        if (out.rows, out.k) != (M, K):
            raise ValueError(f"out is [{out.rows}, {out.k}], x is [{M}, {K}]")
    if out.scale is None:
        out.scale = torch.empty(2, dtype=torch.float32, device=x.device)
    _need(out.scale, torch.float32, None, "out.scale", 2, dev=dev)
    if workspace is None:
        workspace = torch.empty(NVFP4_DYNAMIC_WORKSPACE_BYTES, dtype=torch.uint8, device=x.device)
    _need(workspace, workspace.dtype, None, "workspace", dev=dev)
    nvfp4_quantize_dynamic(_ptr(x), M, K, _ptr(out.codes), _ptr(out.sf), _ptr(out.scale), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    out.g = None
    return out


def quantize_from_amax(x, amax, out: Optional[NVFP4Tensor] = None, stream=None) -> NVFP4Tensor:
    """Quantize bf16 ``x`` [M, K] in one pass with the dynamic rule's scale
    derived on the device from ``amax`` (a float32 device tensor whose first
    element is max|x|, e.g. the ``amax_out`` of the GEMM that produced x).  The
    result's ``scale`` holds [amax, g] on the device, as for quantize_dynamic."""
    torch = _torch()
    dev = torch.cuda.current_device()
    M, K = x.shape
    _need(x, torch.bfloat16, None, "x", dev=dev)
    _need(amax, torch.float32, None, "amax", dev=dev)
    if out is None:
        out = NVFP4Tensor(torch.empty(M, K // 2, dtype=torch.uint8, device=x.device),
                          torch.empty(nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=x.device), None, M, K)
    else:
        _need(out.codes, torch.uint8, None, "out.codes", M * K // 2, dev=dev)
        _need(out.sf, torch.uint8, None, "out.sf", nvfp4_sf_bytes(M, K), dev=dev)
        if (out.rows, out.k) != (M, K):
            raise ValueError(f"out is [{out.rows}, {out.k}], x is [{M}, {K}]")
    if out.scale is None:
        out.scale = torch.empty(2, dtype=torch.float32, device=x.device)
    _need(out.scale, torch.float32, None, "out.scale", 2, dev=dev)
    nvfp4_quantize_from_amax(_ptr(x), M, K, _ptr(amax), _ptr(out.codes), _ptr(out.sf), _ptr(out.scale),
                             _stream(stream))
    out.g = None
    return out


@dataclass
class MXFP8Tensor:
    """A [rows, k] MXFP8 tensor on the GPU: E4M3 codes (one byte per element)
    and swizzled E8M0 scales (one per 32 elements)."""
    codes: "object"   # uint8 [rows, k]
    sf: "object"      # uint8 [nvfp4_mxfp8_sf_bytes(rows, k)]
    rows: int
    k: int


def _need_mxfp8(t, name, rows=None, k=None, dev=None):
    rows = t.rows if rows is None else rows
    k = t.k if k is None else k
    torch = _torch()
    if (t.rows, t.k) != (rows, k):
        raise ValueError(f"{name} is [{t.rows}, {t.k}], [{rows}, {k}] needed")
    _need(t.codes, torch.uint8, None, f"{name}.codes", rows * k, dev=dev)
    _need(t.sf, torch.uint8, None, f"{name}.sf", nvfp4_mxfp8_sf_bytes(rows, k), dev=dev)


def quantize_mxfp8(x, out: Optional[MXFP8Tensor] = None, stream=None) -> MXFP8Tensor:
    """Quantize bf16 ``x`` [M, K] to MXFP8 (power-of-two block scales)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    M, K = x.shape
    _need(x, torch.bfloat16, None, "x", dev=dev)
    if out is None:
        out = MXFP8Tensor(torch.empty(M, K, dtype=torch.uint8, device=x.device),
                          torch.empty(nvfp4_mxfp8_sf_bytes(M, K), dtype=torch.uint8, device=x.device), M, K)
    else:
        _need_mxfp8(out, "out", M, K, dev=dev)
    nvfp4_mxfp8_quantize(_ptr(x), M, K, _ptr(out.codes), _ptr(out.sf), _stream(stream))
    return out


def gemm_mxfp8(a: MXFP8Tensor, b: MXFP8Tensor, bias=None, alpha: float = 1.0, y=None, stream=None):
    """y = bf16(alpha * a_hat @ b_hat^T + bias) for MXFP8 operands."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if a.k != b.k:
        raise ValueError("K mismatch")
    M, N, K = a.rows, b.rows, a.k
    _need_mxfp8(a, "a", dev=dev)
    _need_mxfp8(b, "b", dev=dev)
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias", dev=dev)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _need(y, torch.bfloat16, (M, N), "y", dev=dev)
    nvfp4_mxfp8_gemm(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(alpha), _ptr(bias),
                     _ptr(y), _stream(stream))
    return y


@dataclass
class FP8RowTensor:
    """A [rows, k] row-wise FP8 tensor on the GPU: E4M3 codes and one fp32
    scale per row."""
    codes: "object"   # uint8 [rows, k]
    scale: "object"   # float32 [rows]
    rows: int
    k: int


def _need_fp8row(t, name, rows=None, k=None, dev=None):
    rows = t.rows if rows is None else rows
    k = t.k if k is None else k
    torch = _torch()
    if (t.rows, t.k) != (rows, k):
        raise ValueError(f"{name} is [{t.rows}, {t.k}], [{rows}, {k}] needed")
    _need(t.codes, torch.uint8, None, f"{name}.codes", rows * k, dev=dev)
    _need(t.scale, torch.float32, None, f"{name}.scale", rows, dev=dev)


def quantize_fp8row(x, out: Optional[FP8RowTensor] = None, stream=None) -> FP8RowTensor:
    """Quantize bf16 ``x`` [M, K] to E4M3 with one absmax scale per row."""
    torch = _torch()
    dev = torch.cuda.current_device()
    M, K = x.shape
    _need(x, torch.bfloat16, None, "x", dev=dev)
    if out is None:
        out = FP8RowTensor(torch.empty(M, K, dtype=torch.uint8, device=x.device),
                           torch.empty(M, dtype=torch.float32, device=x.device), M, K)
    else:
        _need_fp8row(out, "out", M, K, dev=dev)
    nvfp4_fp8row_quantize(_ptr(x), M, K, _ptr(out.codes), _ptr(out.scale), _stream(stream))
    return out


def gemm_fp8row(a: FP8RowTensor, b: FP8RowTensor, bias=None, y=None, stream=None):
    """y = bf16(a_scale[m] * b_scale[n] * a_q @ b_q^T + bias)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if a.k != b.k:
        raise ValueError("K mismatch")
    M, N, K = a.rows, b.rows, a.k
    _need_fp8row(a, "a", dev=dev)
    _need_fp8row(b, "b", dev=dev)
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias", dev=dev)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _need(y, torch.bfloat16, (M, N), "y", dev=dev)
    nvfp4_fp8row_gemm(_ptr(a.codes), _ptr(a.scale), _ptr(b.codes), _ptr(b.scale), M, N, K, _ptr(bias), _ptr(y),
                      _stream(stream))
    return y


def dequantize(t: NVFP4Tensor, out=None, stream=None):
    """NVFP4 tensor -> bf16 [rows, k] (the W4A16 path's weight)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if t.g is None:
        raise ValueError("dequantize needs the per-tensor scale g on the host")
    _need_nvfp4(t, "t", dev=dev)
    if out is None:
        out = torch.empty(t.rows, t.k, dtype=torch.bfloat16, device=t.codes.device)
    _need(out, torch.bfloat16, (t.rows, t.k), "out", dev=dev)
    nvfp4_dequantize(_ptr(t.codes), _ptr(t.sf), float(t.g), t.rows, t.k, _ptr(out), _stream(stream))
    return out


def linear_w4a16(x, w: NVFP4Tensor, bias=None, y=None, stream=None):
    """W4A16 linear y = bf16(x @ w_bf16^T + bias): bf16 activations ``x``
    [M, K] against an NVFP4 weight that the GEMM dequantizes tile by tile in
    shared memory (the values ``dequantize`` would write), in one kernel."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if w.g is None:
        raise ValueError("the weight needs its per-tensor scale g on the host")
    M, K = x.shape
    N = w.rows
    if w.k != K:
        raise ValueError("K mismatch")
    _need(x, torch.bfloat16, None, "x", dev=dev)
    _need_nvfp4(w, "w", dev=dev)
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias", dev=dev)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, (M, N), "y", dev=dev)
    nvfp4_w4a16_gemm(_ptr(x), _ptr(w.codes), _ptr(w.sf), M, N, K, float(w.g), _ptr(bias), _ptr(y), _stream(stream))
    return y


def swizzle_sf(sf_linear, rows: int, k: int, stream=None):
    """ModelOpt row-major E4M3 scales [rows, k/16] -> swizzled buffer."""
    torch = _torch()
    dev = torch.cuda.current_device()
    _need(sf_linear, torch.uint8, (rows, k // 16), "sf_linear", dev=dev)
    out = torch.empty(nvfp4_sf_bytes(rows, k), dtype=torch.uint8, device=sf_linear.device)
    nvfp4_swizzle_sf(_ptr(sf_linear), rows, k, _ptr(out), _stream(stream))
    return out


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, bias=None, alpha: Optional[float] = None, y=None, stream=None,
         amax_out=None):
    """y = bf16(alpha * a_hat @ b_hat^T + bias).  Without ``alpha`` the
    library forms alpha = fl32(g_a * g_b) from the two per-tensor scales (the
    activation's read on the device when it was measured there).  With
    ``amax_out`` (a float32 device tensor) the epilogue also folds max|y|
    into amax_out[0] (an atomic max: zero it first to measure this y)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if a.k != b.k:
        raise ValueError("K mismatch")
    M, N, K = a.rows, b.rows, a.k
    if alpha is None and b.g is None:
        raise ValueError("the weight b needs its per-tensor scale g on the host, or pass alpha")
    _need_nvfp4(a, "a", dev=dev)
    _need_nvfp4(b, "b", dev=dev)
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias", dev=dev)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _need(y, torch.bfloat16, (M, N), "y", dev=dev)
    if amax_out is not None:
        _need(amax_out, torch.float32, None, "amax_out", dev=dev)
        # alpha whole (times 1), or the two scales, the activation's possibly on the device
        g_a, g_a_dev, g_b = ((float(alpha), 0, 1.0) if alpha is not None else
                             (0.0, _ptr(a.scale) + 4, float(b.g)) if a.g is None else (float(a.g), 0, float(b.g)))
        nvfp4_gemm_amax(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, g_a, g_a_dev, g_b,
                        _ptr(bias), _ptr(y), _ptr(amax_out), _stream(stream))
    elif alpha is not None:
        nvfp4_gemm(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(alpha), _ptr(bias),
                   _ptr(y), _stream(stream))
    elif a.g is None:
        # the activation's scale lives on the device: alpha = fl32(g_a * g_b) in the kernel
        nvfp4_gemm_dynamic(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(b.g),
                           _ptr(a.scale) + 4, _ptr(bias), _ptr(y), _stream(stream))
    else:
        nvfp4_gemm_scaled(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(a.g), float(b.g),
                          _ptr(bias), _ptr(y), _stream(stream))
    return y


def gemm_quant(a: NVFP4Tensor, b: NVFP4Tensor, ranges: Sequence[tuple], *, bias=None, alpha=None, y_bf16=None,
               g_next: float = 1.0, next_out: Optional[NVFP4Tensor] = None, stream=None) -> None:
    """Fused GEMM whose epilogue writes column ranges to a bf16 tensor and/or
    quantizes them into the next layer's NVFP4 input.  ``ranges`` holds
    ``(begin, end, act, dst, dst_col)`` tuples.  Without ``alpha`` the library
    forms alpha = fl32(g_a * g_b) from the two per-tensor scales."""
    torch = _torch()
    dev = torch.cuda.current_device()
    if a.k != b.k:
        raise ValueError("K mismatch")
    M, N, K = a.rows, b.rows, a.k
    _need_nvfp4(a, "a", dev=dev)
    _need_nvfp4(b, "b", dev=dev)
    if alpha is None and (a.g is None or b.g is None):
        raise ValueError("gemm_quant needs alpha, or both per-tensor scales on the host")
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias", dev=dev)
    if y_bf16 is not None:
        _need(y_bf16, torch.bfloat16, None, "y_bf16", dev=dev)
        if y_bf16.dim() != 2 or y_bf16.shape[0] < M:
            raise ValueError(f"y_bf16 must be 2-D with at least {M} rows, got {tuple(y_bf16.shape)}")
    if next_out is not None:
        _need(next_out.codes, torch.uint8, None, "next_out.codes", M * next_out.k // 2, dev=dev)
        _need(next_out.sf, torch.uint8, None, "next_out.sf", nvfp4_sf_bytes(M, next_out.k), dev=dev)
        if next_out.rows != M:
            raise ValueError(f"next_out has {next_out.rows} rows, the GEMM writes {M}")
    rs = [ColRange(int(r[0]), int(r[1]), int(r[2]), int(r[3]), int(r[4])) for r in ranges]
    ldy = int(y_bf16.shape[1]) if y_bf16 is not None else 0
    codes_next = next_out.codes if next_out is not None else None
    sf_next = next_out.sf if next_out is not None else None
    k_next = next_out.k if next_out is not None else 0
    if alpha is not None:
        nvfp4_gemm_quant(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(alpha), _ptr(bias),
                         rs, _ptr(y_bf16), ldy, float(g_next), _ptr(codes_next), _ptr(sf_next), k_next,
                         _stream(stream))
    else:
        nvfp4_gemm_quant_scaled(_ptr(a.codes), _ptr(a.sf), _ptr(b.codes), _ptr(b.sf), M, N, K, float(a.g),
                                float(b.g), _ptr(bias), rs, _ptr(y_bf16), ldy, float(g_next), _ptr(codes_next),
                                _ptr(sf_next), k_next, _stream(stream))
    if next_out is not None:
        next_out.g = float(g_next)
