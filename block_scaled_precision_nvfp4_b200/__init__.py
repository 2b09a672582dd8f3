"""B200 (sm_100a) block-scaled NVFP4 matmul: Python binding of the C ABI in include/nvfp4.h.

The names mirror the C entry points.  This module only marshals arguments:
torch tensors (CUDA memory, allocated by PyTorch) become raw pointers and the
current torch stream becomes the ``stream`` argument; every step of the
computation runs in the library's own kernels.  There is no CPU fallback: on a
machine whose library cannot load, or whose device has no path, each call
raises.

Formats (metrale_circuit ``hardware::exec`` module doc, bullets 1-2):
packed E2M1 codes ``uint8[rows, K/2]`` (even k in the low nibble), E4M3 group
scales ``uint8[rows, K/16]`` (one per 16 consecutive k), FP32 per-tensor scales,
BF16 output ``[M, N]`` = alpha * (A.sA)(W.sW)^T.
"""
from __future__ import annotations

import ctypes
import enum
import os
import threading

from . import _build

__all__ = [
    "Fmt", "Kind", "Exec", "Status", "NvFp4Error", "load_library", "library_path",
    "nvfp4_kind_of", "nvfp4_exec_of", "nvfp4_exec_of_arch", "nvfp4_pair_name",
    "nvfp4_exec_name", "nvfp4_set_fp4_kernel_disabled", "nvfp4_version",
    "nvfp4_check_device_error", "gemm_nvfp4_w4a4", "gemm_nvfp4_via_fp8", "gemm_nvfp4_w4a8", "gemm_w4a16",
    "gemm_nvfp4_w4a4_grouped", "gemm_nvfp4_w4a4_grouped_host", "nvfp4_scale_layout_bytes",
    "nvfp4_pack_scales", "nvfp4_prepare_scales", "nvfp4_workspace_size", "Op",
    "gemm_nvfp4_w4a4_packed", "nvfp4_w4a4_packed_workspace_bytes", "w4a4_packed_workspace",
    "nvfp4_grouped_scale_layout_bytes", "nvfp4_pack_scales_grouped",
    "gemm_nvfp4_w4a4_grouped_packed", "nvfp4_quantize_bf16", "nvfp4_quantize_bf16_routed",
    "nvfp4_fp4_fallback",
    "nvfp4_node_exec", "moe_route", "moe_permute_rows", "moe_combine", "GroupedSchedule",
    "C_FUNCTIONS",
]


class Fmt(enum.IntEnum):
    BF16 = 0
    FP8_E4M3 = 1
    NVFP4 = 2


class Kind(enum.IntEnum):
    BF16_MMA = 0
    FP8_MMA = 1
    FP4_BLOCK_SCALED = 2
    INVALID = -1


class Exec(enum.IntEnum):
    FP4_MMA = 0
    FP8_EXACT = 1
    BF16_WIDEN = 2
    NO_FP4_KERNEL = 3
    NO_PATH = 4


class Op(enum.IntEnum):
    """Operations of nvfp4_workspace_size."""
    W4A4 = 0
    VIA_FP8 = 1
    W4A16 = 2
    W4A4_GROUPED = 3
    W4A8 = 4
    W4A4_PACKED = 5
    QUANTIZE = 6
    MOE_ROUTE = 7


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    MISALIGNED = 2
    NOPATH = 3
    NO_FP4_KERNEL = 4
    CUDA = 5
    DEVICE_TIMEOUT = 6


class NvFp4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = Status(status)
        super().__init__(f"{self.status.name}: {message}")


# C signatures: name -> (restype, argtypes)
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_S = ctypes.c_char_p
C_FUNCTIONS = {
    "nvfp4_version": (_S, []),
    "nvfp4_last_error": (_S, []),
    "nvfp4_kind_of": (_I, [_I]),
    "nvfp4_exec_of_arch": (_I, [_I, _I, _I, _I]),
    "nvfp4_exec_of": (_I, [_I, _I, _I]),
    "nvfp4_fp4_fallback": (_I, [_I]),
    "nvfp4_node_exec": (_I, [_I, _I, _P, _P, _I, _P]),
    "nvfp4_set_fp4_kernel_disabled": (None, [_I]),
    "nvfp4_pair_name": (_S, [_I, _I]),
    "nvfp4_exec_name": (_S, [_I]),
    "nvfp4_check_device_error": (_I, [_P]),
    "gemm_nvfp4_w4a4": (_I, [_P, _P, _F, _P, _P, _F, _P, _I, _I, _I, _P]),
    "gemm_nvfp4_via_fp8": (_I, [_P, _P, _F, _P, _P, _F, _P, _I, _I, _I, _P]),
    "gemm_nvfp4_w4a8": (_I, [_P, _F, _P, _P, _F, _P, _I, _I, _I, _P]),
    "nvfp4_scale_layout_bytes": (_Z, [_I, _I]),
    "nvfp4_pack_scales": (_I, [_P, _I, _I, _P, _P]),
    "gemm_nvfp4_w4a4_packed": (_I, [_P, _P, _F, _P, _P, _F, _P, _I, _I, _I, _P]),
    "nvfp4_w4a4_packed_workspace_bytes": (_Z, [_I, _I, _I, _I]),
    "nvfp4_w4a4_packed_workspace_bytes_for": (_Z, [_I, _I, _I, _I, _I]),
    "gemm_nvfp4_w4a4_packed_ws": (_I, [_P, _P, _F, _P, _P, _F, _P, _I, _I, _I, _I, _P, _Z, _P]),
    "gemm_w4a16": (_I, [_P, _P, _P, _F, _P, _I, _I, _I, _P]),
    "gemm_nvfp4_w4a4_grouped": (_I, [_P, _P, _F, _P, _P, _P, _P, _I, _I, _P, _I, _I, _P, _Z, _P]),
    "gemm_nvfp4_w4a4_grouped_host": (_I, [_P, _P, _F, _P, _P, _P, _P, _I, _P, _I, _I, _P]),
    "nvfp4_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "nvfp4_prepare_scales": (_I, [_P, _P, _I, _I, _P]),
    "nvfp4_grouped_scale_layout_bytes": (_Z, [_P, _I, _I]),
    "nvfp4_pack_scales_grouped": (_I, [_P, _P, _I, _I, _P, _P]),
    "gemm_nvfp4_w4a4_grouped_packed": (_I, [_P, _P, _F, _P, _P, _P, _P, _I, _P, _I, _I, _P]),
    "nvfp4_quantize_workspace_bytes": (_Z, []),
    "nvfp4_moe_route_workspace_bytes": (_Z, [_I, _I]),
    "nvfp4_moe_route": (_I, [_P, _I, _I, _P, _P, _P, _P, _Z, _P]),
    "nvfp4_moe_permute_rows": (_I, [_P, _Z, _I, _I, _I, _P, _P, _P]),
    "nvfp4_moe_combine": (_I, [_P, _I, _P, _P, _I, _I, _I, _P, _P]),
    "nvfp4_grouped_sched_bytes": (_Z, []),
    "nvfp4_grouped_scale_layout_bytes_bound": (_Z, [_I, _I, _I]),
    "nvfp4_grouped_schedule": (_I, [_P, _I, _I, _I, _I, _P, _F, _P, _P, _P]),
    "nvfp4_pack_scales_grouped_sched": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "gemm_nvfp4_w4a4_grouped_packed_sched": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _P]),
    "gemm_nvfp4_w4a4_grouped_packed_sched_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, _P, _P,
                                                          _I, _I, _I, _P]),
    "nvfp4_quantize_bf16": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "nvfp4_quantize_bf16_noalloc": (_I, [_P, _I, _I, _P, _P, _P, _P, _P]),
    "nvfp4_quantize_bf16_routed": (_I, [_P, _I, _I, _P, _I, _P, _P, _P, _P, _Z, _P]),
}

_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB


def load_library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libnvfp4_b200.so (building it with nvcc if absent).  Raises if it cannot load."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_build.LIB):
                if not build_if_missing:
                    raise OSError(f"{_build.LIB} is missing; run block_scaled_precision_nvfp4_b200."
                                  "_build.build()")
                _build.build()
            lib = ctypes.CDLL(_build.LIB)
            for name, (res, args) in C_FUNCTIONS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _err(status: int):
    if status != 0:
        msg = load_library().nvfp4_last_error().decode(errors="replace")
        raise NvFp4Error(status, msg)


# --- planning -------------------------------------------------------------------

def nvfp4_version() -> str:
    return load_library().nvfp4_version().decode()


def nvfp4_kind_of(activation: Fmt) -> Kind:
    return Kind(load_library().nvfp4_kind_of(int(activation)))


def nvfp4_exec_of_arch(sm_arch: int, weight: Fmt, activation: Fmt,
                       fp4_kernel_disabled: bool = False) -> Exec:
    return Exec(load_library().nvfp4_exec_of_arch(int(sm_arch), int(weight), int(activation),
                                                  int(bool(fp4_kernel_disabled))))


def nvfp4_fp4_fallback(sm_arch: int) -> Exec:
    """How an NVFP4 activation runs on class sm_arch without an FP4 block-scale kernel."""
    return Exec(load_library().nvfp4_fp4_fallback(int(sm_arch)))


def nvfp4_node_exec(sm_arch: int, nodes, fp4_kernel_disabled: bool = False) -> list:
    """node_exec over a list of (weight Fmt, activation Fmt) nodes on class sm_arch."""
    import ctypes
    nodes = list(nodes)
    n = len(nodes)
    w = (ctypes.c_int32 * max(n, 1))(*[int(a) for a, _ in nodes])
    a = (ctypes.c_int32 * max(n, 1))(*[int(b) for _, b in nodes])
    out = (ctypes.c_int32 * max(n, 1))()
    _err(load_library().nvfp4_node_exec(int(sm_arch), int(bool(fp4_kernel_disabled)),
                                        ctypes.cast(w, ctypes.c_void_p), ctypes.cast(a, ctypes.c_void_p),
                                        n, ctypes.cast(out, ctypes.c_void_p)))
    return [Exec(out[i]) for i in range(n)]


def nvfp4_exec_of(device: int, weight: Fmt, activation: Fmt) -> Exec:
    return Exec(load_library().nvfp4_exec_of(int(device), int(weight), int(activation)))


def nvfp4_set_fp4_kernel_disabled(disabled: bool) -> None:
    load_library().nvfp4_set_fp4_kernel_disabled(int(bool(disabled)))


def nvfp4_pair_name(weight: Fmt, activation: Fmt) -> str:
    return load_library().nvfp4_pair_name(int(weight), int(activation)).decode()


def nvfp4_exec_name(e: Exec) -> str:
    return load_library().nvfp4_exec_name(int(e)).decode()


# --- tensor marshalling -----------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dev_tensor(t, dtype, shape, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (there is no CPU path)")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def nvfp4_check_device_error(stream=None) -> None:
    _err(load_library().nvfp4_check_device_error(_stream_ptr(stream)))


# --- matmuls ----------------------------------------------------------------------

def _w4a4_common(fn_name, A, sA, gA, W, sW, gW, out, stream):
    torch = _torch()
    M, half_k = A.shape
    N = W.shape[0]
    K = 2 * half_k
    pa = _dev_tensor(A, torch.uint8, (M, K // 2), "A")
    psa = _dev_tensor(sA, torch.uint8, (M, K // 16), "sA")
    pw = _dev_tensor(W, torch.uint8, (N, K // 2), "W")
    psw = _dev_tensor(sW, torch.uint8, (N, K // 16), "sW")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(getattr(load_library(), fn_name)(pa, psa, float(gA), pw, psw, float(gW), py, M, N, K,
                                          _stream_ptr(stream)))
    return out


def gemm_nvfp4_w4a4(A, sA, gA, W, sW, gW, out=None, stream=None):
    """Y[M,N] (bf16) = gA*gW * (A.sA)(W.sW)^T on the block-scaled FP4 MMA."""
    return _w4a4_common("gemm_nvfp4_w4a4", A, sA, gA, W, sW, gW, out, stream)


def nvfp4_scale_layout_bytes(rows: int, K: int) -> int:
    return int(load_library().nvfp4_scale_layout_bytes(int(rows), int(K)))


def nvfp4_pack_scales(s, K=None, out=None, stream=None):
    """Plain E4M3 scales uint8 [rows, K/16] -> the MMA's packed scale layout (uint8, 1-D)."""
    torch = _torch()
    rows, groups = s.shape
    K = 16 * groups if K is None else int(K)
    ps = _dev_tensor(s, torch.uint8, (rows, K // 16), "s")
    n = nvfp4_scale_layout_bytes(rows, K)
    if out is None:
        out = torch.empty(max(n, 16), dtype=torch.uint8, device=s.device)
    if out.dtype != torch.uint8 or not out.is_cuda or out.numel() < n or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous CUDA uint8 tensor of >= {n} bytes")
    _err(load_library().nvfp4_pack_scales(ps, rows, K, out.data_ptr(), _stream_ptr(stream)))
    return out


def nvfp4_quantize_bf16(x, plain=True, packed=True, workspace=None, stream=None, out=None):
    """Two-level NVFP4 quantisation of a BF16 [rows, K] CUDA tensor on the GPU.

    Returns (codes uint8 [rows, K/2], scales uint8 [rows, K/16] or None,
    packed scales uint8 1-D or None, g: a 1-element float32 CUDA tensor).
    `out`, if given, is such a tuple of preallocated tensors to write into."""
    torch = _torch()
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise TypeError("x must be a 2-D torch.Tensor")
    rows, K = x.shape
    px = _dev_tensor(x, torch.bfloat16, (rows, K), "x")
    dev = x.device
    if out is not None:
        codes, scales, sp, g = out
    else:
        codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((rows, K // 16), dtype=torch.uint8, device=dev) if plain else None
        sp = (torch.empty(max(nvfp4_scale_layout_bytes(rows, K), 16), dtype=torch.uint8, device=dev)
              if packed else None)
        g = torch.empty(4, dtype=torch.float32, device=dev)
    _dev_tensor(codes, torch.uint8, (rows, K // 2), "codes")
    if scales is not None:
        _dev_tensor(scales, torch.uint8, (rows, K // 16), "scales")
    if sp is not None:
        need = nvfp4_scale_layout_bytes(rows, K)
        if sp.dtype != torch.uint8 or not sp.is_cuda or not sp.is_contiguous() or sp.numel() < need:
            raise ValueError(f"packed scales must be a contiguous CUDA uint8 tensor of >= {need} bytes")
    if g.dtype != torch.float32 or not g.is_cuda or g.numel() < 1:
        raise ValueError("g must be a CUDA float32 tensor")
    lib = load_library()
    nws = int(lib.nvfp4_quantize_workspace_bytes())
    if workspace is None:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
            or not workspace.is_contiguous() or workspace.numel() * workspace.element_size() < nws):
        raise ValueError(f"workspace must be a contiguous CUDA tensor of >= {nws} bytes")
    _err(lib.nvfp4_quantize_bf16(px, rows, K, codes.data_ptr(),
                                 scales.data_ptr() if scales is not None else None,
                                 sp.data_ptr() if sp is not None else None, g.data_ptr(),
                                 workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream_ptr(stream)))
    return codes, scales, sp, g[:1]


def nvfp4_quantize_bf16_routed(x, dest, k=1, workspace=None, stream=None, out=None):
    """nvfp4_quantize_bf16 writing token row r's codes and plain scales to rows
    dest[r*k + j] (j < k): the quantised rows in an MoE dispatch's order.

    `dest` is the int32 [rows*k] CUDA tensor nvfp4_moe_route returns.  Returns (codes
    uint8 [rows*k, K/2], scales uint8 [rows*k, K/16], g: 1-element float32 CUDA tensor);
    `out`, if given, is such a tuple of preallocated tensors."""
    torch = _torch()
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise TypeError("x must be a 2-D torch.Tensor")
    rows, K = x.shape
    k = int(k)
    px = _dev_tensor(x, torch.bfloat16, (rows, K), "x")
    pd = _dev_tensor(dest, torch.int32, (rows * k,), "dest")
    dev = x.device
    if out is not None:
        codes, scales, g = out
    else:
        codes = torch.empty((rows * k, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((rows * k, K // 16), dtype=torch.uint8, device=dev)
        g = torch.empty(4, dtype=torch.float32, device=dev)
    _dev_tensor(codes, torch.uint8, (rows * k, K // 2), "codes")
    _dev_tensor(scales, torch.uint8, (rows * k, K // 16), "scales")
    if g.dtype != torch.float32 or not g.is_cuda or g.numel() < 1:
        raise ValueError("g must be a CUDA float32 tensor")
    lib = load_library()
    nws = int(lib.nvfp4_quantize_workspace_bytes())
    if workspace is None:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
            or not workspace.is_contiguous() or workspace.numel() * workspace.element_size() < nws):
        raise ValueError(f"workspace must be a contiguous CUDA tensor of >= {nws} bytes")
    _err(lib.nvfp4_quantize_bf16_routed(px, rows, K, pd, k, codes.data_ptr(), scales.data_ptr(),
                                        g.data_ptr(), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream)))
    return codes, scales, g[:1]


def nvfp4_w4a4_packed_workspace_bytes(M, N, K, max_pairs=0):
    """Device bytes the balanced (stream-K) pair product needs on the current device; 0: none."""
    return int(load_library().nvfp4_w4a4_packed_workspace_bytes(int(M), int(N), int(K),
                                                                int(max_pairs)))


def w4a4_packed_workspace(M, N, K, max_pairs=0, device=None):
    """A zeroed workspace for gemm_nvfp4_w4a4_packed(..., workspace=...), or None when
    the shape needs none.  It stays valid across calls of this shape (or any shape
    needing no more bytes); calls that overlap on the GPU need one each."""
    torch = _torch()
    n = nvfp4_w4a4_packed_workspace_bytes(M, N, K, max_pairs)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda") if n else None


def gemm_nvfp4_w4a4_packed(A, sA_packed, gA, W, sW_packed, gW, out=None, stream=None,
                           workspace=None, max_pairs=0):
    """gemm_nvfp4_w4a4 with scales packed by nvfp4_pack_scales (pairs of SMs, K % 256 == 0).
    With a workspace (w4a4_packed_workspace), the last waves of tiles are balanced over
    the pairs (stream-K); max_pairs > 0 caps the number of SM pairs."""
    torch = _torch()
    M, half_k = A.shape
    N = W.shape[0]
    K = 2 * half_k
    pa = _dev_tensor(A, torch.uint8, (M, K // 2), "A")
    pw = _dev_tensor(W, torch.uint8, (N, K // 2), "W")
    for name, t, rows in (("sA_packed", sA_packed, M), ("sW_packed", sW_packed, N)):
        need = nvfp4_scale_layout_bytes(rows, K)
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_cuda
                or not t.is_contiguous() or t.numel() < need):
            raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of >= {need} bytes")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    if workspace is None and not max_pairs:
        _err(load_library().gemm_nvfp4_w4a4_packed(pa, sA_packed.data_ptr(), float(gA), pw,
                                                   sW_packed.data_ptr(), float(gW), py, M, N, K,
                                                   _stream_ptr(stream)))
        return out
    if workspace is not None and (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
                                  or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    pws = workspace.data_ptr() if workspace is not None else None
    nws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _err(load_library().gemm_nvfp4_w4a4_packed_ws(pa, sA_packed.data_ptr(), float(gA), pw,
                                                  sW_packed.data_ptr(), float(gW), py, M, N, K,
                                                  int(max_pairs), pws, nws, _stream_ptr(stream)))
    return out


def gemm_nvfp4_via_fp8(A, sA, gA, W, sW, gW, out=None, stream=None):
    """The same product through the exact E2M1->E4M3 conversion on the FP8 MMA."""
    return _w4a4_common("gemm_nvfp4_via_fp8", A, sA, gA, W, sW, gW, out, stream)


def gemm_nvfp4_w4a8(A_fp8, gA, W, sW, gW, out=None, stream=None):
    """Y[M,N] (bf16) = gA*gW * A_fp8 . (W.sW)^T: E4M3 activation bytes [M,K] under NVFP4
    weights, on the exact E4M3 path (K % 256 == 0)."""
    torch = _torch()
    M, K = A_fp8.shape
    N = W.shape[0]
    a = A_fp8.view(torch.uint8) if A_fp8.dtype != torch.uint8 else A_fp8
    pa = _dev_tensor(a, torch.uint8, (M, K), "A_fp8")
    pw = _dev_tensor(W, torch.uint8, (N, K // 2), "W")
    psw = _dev_tensor(sW, torch.uint8, (N, K // 16), "sW")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A_fp8.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(load_library().gemm_nvfp4_w4a8(pa, float(gA), pw, psw, float(gW), py, M, N, K,
                                        _stream_ptr(stream)))
    return out


def gemm_w4a16(A, W, sW, gW, out=None, stream=None):
    """Y[M,N] (bf16) = gW * A_bf16 . (W.sW)^T, weights widened to BF16 in registers."""
    torch = _torch()
    M, K = A.shape
    N = W.shape[0]
    pa = _dev_tensor(A, torch.bfloat16, (M, K), "A")
    pw = _dev_tensor(W, torch.uint8, (N, K // 2), "W")
    psw = _dev_tensor(sW, torch.uint8, (N, K // 16), "sW")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(load_library().gemm_w4a16(pa, pw, psw, float(gW), py, M, N, K, _stream_ptr(stream)))
    return out


def gemm_nvfp4_w4a4_grouped(A, sA, gA, W, sW, gW, offsets, out=None, workspace=None,
                            stream=None):
    """Grouped W4A4: W [E,N,K/2], sW [E,N,K/16], gW (E floats).  With offsets a CUDA
    int32 tensor [E+1], the C entry gemm_nvfp4_w4a4_grouped (device offsets, the
    plan made on the device; `workspace` a CUDA uint8 tensor of at least
    nvfp4_workspace_size(Op.W4A4_GROUPED, M, N, K, E) bytes, allocated here if None);
    with host offsets (E+1 ints), gemm_nvfp4_w4a4_grouped_host."""
    torch = _torch()
    if not (isinstance(offsets, torch.Tensor) and offsets.is_cuda):
        return gemm_nvfp4_w4a4_grouped_host(A, sA, gA, W, sW, gW, offsets, out, stream)
    M, half_k = A.shape
    K = 2 * half_k
    E, N = W.shape[0], W.shape[1]
    pa = _dev_tensor(A, torch.uint8, (M, K // 2), "A")
    psa = _dev_tensor(sA, torch.uint8, (M, K // 16), "sA")
    pw = _dev_tensor(W, torch.uint8, (E, N, K // 2), "W")
    psw = _dev_tensor(sW, torch.uint8, (E, N, K // 16), "sW")
    po = _dev_tensor(offsets, torch.int32, (E + 1,), "offsets")
    gws = (ctypes.c_float * E)(*[float(x) for x in gW])
    need = int(load_library().nvfp4_workspace_size(int(Op.W4A4_GROUPED), M, N, K, E))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=A.device)
    if workspace.dtype != torch.uint8 or not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(load_library().gemm_nvfp4_w4a4_grouped(pa, psa, float(gA), pw, psw,
                                                ctypes.cast(gws, ctypes.c_void_p), po, E, M, py,
                                                N, K, workspace.data_ptr(), workspace.numel(),
                                                _stream_ptr(stream)))
    return out


def gemm_nvfp4_w4a4_grouped_host(A, sA, gA, W, sW, gW, offsets, out=None, stream=None):
    """Grouped W4A4 planned on the host: W [E,N,K/2], sW [E,N,K/16], gW (E floats),
    offsets (E+1 ints, host)."""
    torch = _torch()
    M, half_k = A.shape
    K = 2 * half_k
    E, N = W.shape[0], W.shape[1]
    pa = _dev_tensor(A, torch.uint8, (M, K // 2), "A")
    psa = _dev_tensor(sA, torch.uint8, (M, K // 16), "sA")
    pw = _dev_tensor(W, torch.uint8, (E, N, K // 2), "W")
    psw = _dev_tensor(sW, torch.uint8, (E, N, K // 16), "sW")
    off = (ctypes.c_int32 * (E + 1))(*[int(x) for x in offsets])
    gws = (ctypes.c_float * E)(*[float(x) for x in gW])
    if len(offsets) != E + 1 or int(offsets[-1]) != M:
        raise ValueError("offsets must hold E+1 row offsets ending at A.shape[0]")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(load_library().gemm_nvfp4_w4a4_grouped_host(pa, psa, float(gA), pw, psw,
                                                     ctypes.cast(gws, ctypes.c_void_p),
                                                     ctypes.cast(off, ctypes.c_void_p), E, py, N,
                                                     K, _stream_ptr(stream)))
    return out


def nvfp4_workspace_size(op, M, N, K, E=1) -> int:
    """Device bytes of caller workspace operation `op` (an Op) needs."""
    return int(load_library().nvfp4_workspace_size(int(op), int(M), int(N), int(K), int(E)))


def nvfp4_prepare_scales(s, K=None, out=None, stream=None):
    """Plain scales uint8 [rows, K/16] -> the MMA scale layout (uint8 1-D), through the C
    entry nvfp4_prepare_scales."""
    torch = _torch()
    rows, groups = s.shape
    K = 16 * groups if K is None else int(K)
    ps = _dev_tensor(s, torch.uint8, (rows, K // 16), "s")
    n = nvfp4_scale_layout_bytes(rows, K)
    if out is None:
        out = torch.empty(max(n, 16), dtype=torch.uint8, device=s.device)
    if out.dtype != torch.uint8 or not out.is_cuda or out.numel() < n or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous CUDA uint8 tensor of >= {n} bytes")
    _err(load_library().nvfp4_prepare_scales(ps, out.data_ptr(), rows, K, _stream_ptr(stream)))
    return out


def _offsets_arg(offsets, E=None):
    vals = [int(x) for x in offsets]
    if E is not None and len(vals) != E + 1:
        raise ValueError(f"offsets must hold E+1 = {E + 1} row offsets")
    return (ctypes.c_int32 * len(vals))(*vals), len(vals) - 1


def nvfp4_grouped_scale_layout_bytes(offsets, K: int) -> int:
    off, E = _offsets_arg(offsets)
    return int(load_library().nvfp4_grouped_scale_layout_bytes(ctypes.cast(off, ctypes.c_void_p),
                                                                E, int(K)))


def nvfp4_pack_scales_grouped(s, offsets, K=None, out=None, stream=None):
    """Plain scales uint8 [offsets[-1], K/16] -> the grouped packed layout (each
    group of rows starting on a 128-row block), uint8 1-D."""
    torch = _torch()
    rows, groups = s.shape
    K = 16 * groups if K is None else int(K)
    off, E = _offsets_arg(offsets)
    if int(offsets[-1]) != rows:
        raise ValueError("offsets must end at s.shape[0]")
    ps = _dev_tensor(s, torch.uint8, (rows, K // 16), "s")
    n = nvfp4_grouped_scale_layout_bytes(offsets, K)
    if out is None:
        out = torch.empty(max(n, 16), dtype=torch.uint8, device=s.device)
    if out.dtype != torch.uint8 or not out.is_cuda or out.numel() < n or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous CUDA uint8 tensor of >= {n} bytes")
    _err(load_library().nvfp4_pack_scales_grouped(ps, ctypes.cast(off, ctypes.c_void_p), E, K,
                                                  out.data_ptr(), _stream_ptr(stream)))
    return out


def gemm_nvfp4_w4a4_grouped_packed(A, sA_packed, gA, W, sW_packed, gW, offsets, out=None,
                                   stream=None):
    """Grouped W4A4 with packed scales: sA_packed from nvfp4_pack_scales_grouped(sA,
    offsets), sW_packed from nvfp4_pack_scales_grouped(sW.view(E*N, -1), [0, N, .., E*N])."""
    torch = _torch()
    M, half_k = A.shape
    K = 2 * half_k
    E, N = W.shape[0], W.shape[1]
    if len(offsets) != E + 1 or int(offsets[-1]) != M:
        raise ValueError("offsets must hold E+1 row offsets ending at A.shape[0]")
    pa = _dev_tensor(A, torch.uint8, (M, K // 2), "A")
    pw = _dev_tensor(W, torch.uint8, (E, N, K // 2), "W")
    needs = (("sA_packed", sA_packed, nvfp4_grouped_scale_layout_bytes(offsets, K)),
             ("sW_packed", sW_packed,
              nvfp4_grouped_scale_layout_bytes([e * N for e in range(E + 1)], K)))
    for name, t, need in needs:
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_cuda
                or not t.is_contiguous() or t.numel() < need):
            raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of >= {need} bytes")
    off, _ = _offsets_arg(offsets, E)
    gws = (ctypes.c_float * E)(*[float(x) for x in gW])
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    py = _dev_tensor(out, torch.bfloat16, (M, N), "out")
    _err(load_library().gemm_nvfp4_w4a4_grouped_packed(
        pa, sA_packed.data_ptr(), float(gA), pw, sW_packed.data_ptr(),
        ctypes.cast(gws, ctypes.c_void_p), ctypes.cast(off, ctypes.c_void_p), E, py, N, K,
        _stream_ptr(stream)))
    return out


# --- MoE dispatch and combine around the grouped product ---------------------------

def moe_route(expert_ids, E, workspace=None, stream=None):
    """Top-k routing -> (offsets [E+1], dest [P], src [P]), device int32.

    expert_ids: CUDA int32 [T, k] (or [P]); pair p = t*k + j.  Rows of expert e in
    the grouped order are offsets[e] .. offsets[e+1]-1, pairs in their order p."""
    torch = _torch()
    ids = expert_ids.reshape(-1)
    P = ids.numel()
    pid = _dev_tensor(ids, torch.int32, (P,), "expert_ids")
    lib = load_library()
    need = int(lib.nvfp4_moe_route_workspace_bytes(P, int(E)))
    if need == 0:
        raise ValueError(f"E must be in [1, 256] (got {E})")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=ids.device)
    offsets = torch.empty(int(E) + 1, dtype=torch.int32, device=ids.device)
    dest = torch.empty(max(P, 1), dtype=torch.int32, device=ids.device)
    src = torch.empty(max(P, 1), dtype=torch.int32, device=ids.device)
    _err(lib.nvfp4_moe_route(pid, P, int(E), offsets.data_ptr(), dest.data_ptr(), src.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream)))
    return offsets, dest[:P], src[:P]


def moe_permute_rows(x, src, k, out=None, stream=None):
    """Rows of x (CUDA uint8 [rows, row_bytes], token order) -> expert-grouped order:
    out[r] = x[src[r] // k], one row per pair."""
    torch = _torch()
    rows, row_bytes = x.shape
    P = src.numel()
    px = _dev_tensor(x, torch.uint8, (rows, row_bytes), "x")
    ps = _dev_tensor(src, torch.int32, (P,), "src")
    if out is None:
        out = torch.empty((P, row_bytes), dtype=torch.uint8, device=x.device)
    po = _dev_tensor(out, torch.uint8, (P, row_bytes), "out")
    _err(load_library().nvfp4_moe_permute_rows(px, row_bytes, rows, P, int(k), ps, po,
                                               _stream_ptr(stream)))
    return out


def moe_combine(Yg, dest, weights, T, k, out=None, stream=None):
    """Y[t] = BF16(sum_j weights[t, j] * Yg[dest[t*k + j]]), FP32 in j order.
    Yg: CUDA bf16 [P, N] in the expert-grouped order; weights: float32 [T, k] or None."""
    torch = _torch()
    P, N = Yg.shape
    py = _dev_tensor(Yg, torch.bfloat16, (P, N), "Yg")
    pd = _dev_tensor(dest.reshape(-1), torch.int32, (T * k,), "dest")
    pw = None
    if weights is not None:
        pw = _dev_tensor(weights.reshape(-1), torch.float32, (T * k,), "weights")
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=Yg.device)
    po = _dev_tensor(out, torch.bfloat16, (T, N), "out")
    _err(load_library().nvfp4_moe_combine(py, P, pd, pw, int(T), int(k), N, po, _stream_ptr(stream)))
    return out


# --- grouped product planned on the device ------------------------------------------

class GroupedSchedule:
    """The grouped product's tile schedule planned on the device from device offsets.

    sched = GroupedSchedule(offsets_dev, E, M, N, K, gW, gA=None or a 1-element CUDA
    float32 tensor or a float).  Then pack(sA_plain) -> packed activation scales and
    gemm(A, sA_packed, W, sW_packed) -> Y, with no host round trip."""

    def __init__(self, offsets, E, M, N, K, gW, gA=1.0, stream=None):
        torch = _torch()
        self.E, self.M, self.N, self.K = int(E), int(M), int(N), int(K)
        self.buf = torch.empty(int(load_library().nvfp4_grouped_sched_bytes()),
                               dtype=torch.uint8, device=offsets.device)
        self.plan(offsets, gW, gA, stream)

    def plan(self, offsets, gW, gA=1.0, stream=None):
        """(Re)plans into this schedule's buffer from new device offsets (same E, M,
        N, K); later pack/gemm calls on the stream use the new plan."""
        import ctypes
        torch = _torch()
        lib = load_library()
        po = _dev_tensor(offsets, torch.int32, (self.E + 1,), "offsets")
        gws = (ctypes.c_float * self.E)(*[float(x) for x in gW])
        ga_dev, ga = None, 1.0
        if isinstance(gA, torch.Tensor):
            ga_dev = _dev_tensor(gA.reshape(-1)[:1], torch.float32, (1,), "gA")
        else:
            ga = float(gA)
        _err(lib.nvfp4_grouped_schedule(po, self.E, self.M, self.N, self.K, ga_dev, ga,
                                        ctypes.cast(gws, ctypes.c_void_p), self.buf.data_ptr(),
                                        _stream_ptr(stream)))

    def pack(self, s_plain, out=None, stream=None):
        torch = _torch()
        ps = _dev_tensor(s_plain, torch.uint8, (self.M, self.K // 16), "s_plain")
        n = int(load_library().nvfp4_grouped_scale_layout_bytes_bound(self.M, self.E, self.K))
        if out is None:
            out = torch.empty(max(n, 16), dtype=torch.uint8, device=s_plain.device)
        if out.dtype != torch.uint8 or not out.is_cuda or out.numel() < n or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous CUDA uint8 tensor of >= {n} bytes")
        _err(load_library().nvfp4_pack_scales_grouped_sched(ps, self.M, self.E, self.K,
                                                            self.buf.data_ptr(), out.data_ptr(),
                                                            _stream_ptr(stream)))
        return out

    def gemm(self, A, sA_packed, W, sW_packed, out=None, stream=None):
        torch = _torch()
        pa = _dev_tensor(A, torch.uint8, (self.M, self.K // 2), "A")
        pw = _dev_tensor(W, torch.uint8, (self.E, self.N, self.K // 2), "W")
        if out is None:
            out = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=A.device)
        py = _dev_tensor(out, torch.bfloat16, (self.M, self.N), "out")
        _err(load_library().gemm_nvfp4_w4a4_grouped_packed_sched(
            pa, sA_packed.data_ptr(), pw, sW_packed.data_ptr(), self.buf.data_ptr(), self.E,
            self.M, py, self.N, self.K, _stream_ptr(stream)))
        return out

    def gemm_combine(self, A, sA_packed, W, sW_packed, src, T, weights=None, out=None,
                     stream=None):
        """gemm with the top-1 combine in its epilogue: grouped row r goes to out row
        src[r], times weights[src[r]] (device float [T]; None: 1).  out [T, N] bf16."""
        torch = _torch()
        pa = _dev_tensor(A, torch.uint8, (self.M, self.K // 2), "A")
        pw = _dev_tensor(W, torch.uint8, (self.E, self.N, self.K // 2), "W")
        psrc = _dev_tensor(src, torch.int32, (self.M,), "src")
        pwt = (_dev_tensor(weights.reshape(-1), torch.float32, (int(T),), "weights")
               if weights is not None else None)
        if out is None:
            out = torch.empty((int(T), self.N), dtype=torch.bfloat16, device=A.device)
        py = _dev_tensor(out, torch.bfloat16, (int(T), self.N), "out")
        _err(load_library().gemm_nvfp4_w4a4_grouped_packed_sched_combine(
            pa, sA_packed.data_ptr(), pw, sW_packed.data_ptr(), self.buf.data_ptr(), self.E,
            self.M, psrc, pwt, py, int(T), self.N, self.K, _stream_ptr(stream)))
        return out
