"""Thin Python binding of the C ABI in include/awq.h (ctypes; argument marshalling only).

Every computation happens in the CUDA library: this module checks dtypes and
shapes, takes data pointers and the current CUDA stream from torch tensors, and
calls the entry point of the same name.  It raises if the library is missing:
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from .build import LIB

AWQ_OK = 0
AWQ_OP_QUANTIZE_PACK, AWQ_OP_SCALE_SEARCH, AWQ_OP_GEMV, AWQ_OP_GEMM = 0, 1, 2, 3
STATUS_NAMES = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_UNSUPPORTED", 3: "AWQ_ERR_WORKSPACE",
                4: "AWQ_ERR_CUDA", 5: "AWQ_ERR_TIMEOUT", 6: "AWQ_ERR_RANGE"}
(AWQ_ERR_INVALID_ARG, AWQ_ERR_UNSUPPORTED, AWQ_ERR_WORKSPACE, AWQ_ERR_CUDA, AWQ_ERR_TIMEOUT,
 AWQ_ERR_RANGE) = 1, 2, 3, 4, 5, 6

# Every symbol the header declares, with its ctypes signature.
_u16p = ctypes.c_void_p
_u32p = ctypes.c_void_p


class QuantConfig(ctypes.Structure):
    """awq_quant_config: the pages' quant_config {w_bit, q_group_size, zero_point}."""
    _fields_ = [("w_bit", ctypes.c_int32), ("q_group_size", ctypes.c_int32), ("zero_point", ctypes.c_int32)]


SIGNATURES = {
    "awq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "awq_abi_version": (ctypes.c_int32, []),
    "awq_quantize_pack": (ctypes.c_int, [_u16p, _u16p, ctypes.c_int32, ctypes.c_int32, QuantConfig,
                                         _u32p, _u16p, _u32p, ctypes.c_void_p]),
    "awq_scale_search": (ctypes.c_int, [_u16p, ctypes.c_int32, _u16p, ctypes.c_int32, ctypes.c_int32,
                                        QuantConfig, ctypes.c_int32, _u16p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "awq_scale_search_duo": (ctypes.c_int, [_u16p, ctypes.c_int32, _u16p, ctypes.c_int32, ctypes.c_int32,
                                            QuantConfig, ctypes.c_int32, _u16p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "awq_scale_search_noalloc": (ctypes.c_int, [_u16p, ctypes.c_int32, _u16p, ctypes.c_int32, ctypes.c_int32,
                                                QuantConfig, ctypes.c_int32, _u16p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p]),
    "awq_fold_inverse_scale": (ctypes.c_int, [_u16p, _u16p, ctypes.c_int32, ctypes.c_int32, _u16p,
                                              ctypes.c_void_p]),
    "awq_linear_gemv": (ctypes.c_int, [_u16p, ctypes.c_int32, _u32p, _u16p, _u32p, ctypes.c_int32,
                                       ctypes.c_int32, QuantConfig, _u16p, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "awq_linear_gemm": (ctypes.c_int, [_u16p, ctypes.c_int32, _u32p, _u16p, _u32p, ctypes.c_int32,
                                       ctypes.c_int32, QuantConfig, _u16p, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "awq_apply_clip": (ctypes.c_int, [_u16p, ctypes.c_int32, _u16p, _u16p, ctypes.c_int32, ctypes.c_int32,
                                      QuantConfig, ctypes.c_int32, ctypes.c_int32, _u32p, _u16p, _u32p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                      ctypes.c_void_p]),
    "awq_apply_clip_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                         QuantConfig, ctypes.c_int32]),
    "awq_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              QuantConfig]),
    "awq_device_error": (ctypes.c_int, [ctypes.c_void_p]),
    "awq_check_bounded_wait": (ctypes.c_int, [ctypes.c_void_p]),
}

_lib = None


def load_library(path: str = LIB) -> ctypes.CDLL:
    """Load libawq_b200.so and attach the signatures (raises if it is not built)."""
    global _lib
    if _lib is not None and path == LIB:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run `python -m bit_weight_only_linear_b200.build`)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB:
        _lib = lib
    return lib


class AWQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = load_library().awq_status_string(status).decode()
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}: {msg}")


def _check(fn: str, status: int) -> None:
    if status != AWQ_OK:
        raise AWQError(fn, status)


def config(group_size: int = 128, zero_point: bool = True, w_bit: int = 4) -> QuantConfig:
    return QuantConfig(int(w_bit), int(group_size), 1 if zero_point else 0)


def _dev(t: Optional[torch.Tensor], name: str, dtypes) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr()


_F16 = (torch.float16,)
_W32 = (torch.int32, torch.uint32)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def packed_shapes(N: int, K: int, group_size: int, zero_point: bool):
    ng = K // group_size
    return (N, K // 8), (N, ng), ((N, (ng + 7) // 8) if zero_point else None)


def quantize_pack(W: torch.Tensor, s: Optional[torch.Tensor] = None, group_size: int = 128,
                  zero_point: bool = True, out=None, stream=None):
    """awq_quantize_pack: W [N][K] fp16, s [K] fp16 or None -> (qweight int32 [N][K/8],
    scales fp16 [N][K/G], qzeros int32 [N][ceil(K/G/8)] or None)."""
    N, K = W.shape
    qs, ss, zs = packed_shapes(N, K, group_size, zero_point)
    if out is None:
        qweight = torch.empty(qs, dtype=torch.int32, device=W.device)
        scales = torch.empty(ss, dtype=torch.float16, device=W.device)
        qzeros = torch.empty(zs, dtype=torch.int32, device=W.device) if zero_point else None
    else:
        qweight, scales, qzeros = out
    st = load_library().awq_quantize_pack(
        _dev(W, "W", _F16), _dev(s, "s", _F16), N, K, config(group_size, zero_point),
        _dev(qweight, "qweight", _W32), _dev(scales, "scales", _F16), _dev(qzeros, "qzeros", _W32),
        _stream(stream))
    _check("awq_quantize_pack", st)
    return qweight, scales, qzeros


def fold_inverse_scale(X: torch.Tensor, s: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """awq_fold_inverse_scale: X' = fp16(X / s) per input channel."""
    M, K = X.shape
    out = torch.empty_like(X) if out is None else out
    st = load_library().awq_fold_inverse_scale(_dev(X, "X", _F16), _dev(s, "s", _F16), M, K,
                                               _dev(out, "out", _F16), _stream(stream))
    _check("awq_fold_inverse_scale", st)
    return out


def _linear(fn_name: str, X, qweight, scales, qzeros, group_size, zero_point, out, workspace, stream):
    M, K = X.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K:
        raise ValueError("qweight must be [N][K/8]")
    out = torch.empty((M, N), dtype=torch.float16, device=X.device) if out is None else out
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    fn = getattr(load_library(), fn_name)
    st = fn(_dev(X, "X", _F16), M, _dev(qweight, "qweight", _W32), _dev(scales, "scales", _F16),
            _dev(qzeros, "qzeros", _W32), N, K, config(group_size, zero_point), _dev(out, "Y", _F16),
            ws_ptr, ws_bytes, _stream(stream))
    _check(fn_name, st)
    return out


def linear_gemv(X, qweight, scales, qzeros, group_size=128, zero_point=True, out=None, workspace=None,
                stream=None) -> torch.Tensor:
    """awq_linear_gemv: Y [M][N] = X [M][K] . deq(W)^T, decode form (M <= 8)."""
    return _linear("awq_linear_gemv", X, qweight, scales, qzeros, group_size, zero_point, out, workspace, stream)


_GEMM_WS = {}


def gemm_workspace(M: int, N: int, K: int, group_size: int = 128, zero_point: bool = True, device=None):
    """A device workspace large enough for awq_linear_gemm at these sizes (the split-K
    partial sums), cached per device and grown on demand; None when none is needed."""
    need = workspace_bytes(AWQ_OP_GEMM, M, N, K, group_size, zero_point)
    if need == 0:
        return None
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    ws = _GEMM_WS.get(dev)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        _GEMM_WS[dev] = ws
    return ws


def linear_gemm(X, qweight, scales, qzeros, group_size=128, zero_point=True, out=None, workspace=None,
                stream=None) -> torch.Tensor:
    """awq_linear_gemm: Y [M][N] = X [M][K] . deq(W)^T, tcgen05 tensor-core form (any M).  A
    batch too small to fill the GPU splits K over a workspace (the cached one of
    gemm_workspace() unless one is given)."""
    if workspace is None:
        workspace = gemm_workspace(X.shape[0], qweight.shape[0], X.shape[1], group_size, zero_point, X.device)
    return _linear("awq_linear_gemm", X, qweight, scales, qzeros, group_size, zero_point, out, workspace, stream)


def workspace_bytes(op: int, M: int, N: int, K: int, group_size: int = 128, zero_point: bool = True) -> int:
    return int(load_library().awq_workspace_bytes(op, M, N, K, config(group_size, zero_point)))


def scale_search(X: torch.Tensor, W: torch.Tensor, group_size: int = 128, zero_point: bool = True,
                 n_grid: int = 20, workspace: Optional[torch.Tensor] = None, stream=None, out=None,
                 duo_scaling: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """awq_scale_search (awq_scale_search_duo with duo_scaling): returns (s* fp16 [K], losses
    fp64 [n_grid], best index int32 [1]), all on device (into `out` = (s, losses, best) when
    given)."""
    M, K = X.shape
    N = W.shape[0]
    if workspace is None:
        need = workspace_bytes(AWQ_OP_SCALE_SEARCH, M, N, K, group_size, zero_point)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    if out is None:
        s_out = torch.empty(K, dtype=torch.float16, device=X.device)
        losses = torch.empty(n_grid, dtype=torch.float64, device=X.device)
        best = torch.empty(1, dtype=torch.int32, device=X.device)
    else:
        s_out, losses, best = out
    name = "awq_scale_search_duo" if duo_scaling else "awq_scale_search"
    st = getattr(load_library(), name)(
        _dev(X, "X", _F16), M, _dev(W, "W", _F16), N, K, config(group_size, zero_point), n_grid,
        _dev(s_out, "s_out", _F16), losses.data_ptr(), best.data_ptr(), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(name, st)
    return s_out, losses, best


def scale_search_noalloc(X: torch.Tensor, W: torch.Tensor, group_size: int = 128, zero_point: bool = True,
                         n_grid: int = 20, stream=None, out=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """awq_scale_search_noalloc: the scale search on the library's fixed scratch (for
    callers that cannot allocate device memory).  Returns (s*, losses, best index) on
    device, into `out` when given (otherwise torch allocates them here, for convenience)."""
    M, K = X.shape
    N = W.shape[0]
    if out is None:
        s_out = torch.empty(K, dtype=torch.float16, device=X.device)
        losses = torch.empty(n_grid, dtype=torch.float64, device=X.device)
        best = torch.empty(1, dtype=torch.int32, device=X.device)
    else:
        s_out, losses, best = out
    st = load_library().awq_scale_search_noalloc(
        _dev(X, "X", _F16), M, _dev(W, "W", _F16), N, K, config(group_size, zero_point), n_grid,
        _dev(s_out, "s_out", _F16), losses.data_ptr(), best.data_ptr(), _stream(stream))
    _check("awq_scale_search_noalloc", st)
    return s_out, losses, best


def check_bounded_wait(stream=None) -> None:
    """awq_check_bounded_wait: enqueue a kernel whose wait can never complete (it gives up
    after the library's 2 s limit and flags a timeout, read by device_error())."""
    _check("awq_check_bounded_wait", load_library().awq_check_bounded_wait(_stream(stream)))


def device_error(stream=None) -> None:
    """Synchronise and raise AWQError if a bounded device wait ran out."""
    _check("awq_device_error", load_library().awq_device_error(_stream(stream)))


def apply_clip(X: torch.Tensor, W: torch.Tensor, s: Optional[torch.Tensor], group_size: int = 128,
               zero_point: bool = True, n_grid: int = 20, n_clip: int = 10, out=None,
               workspace: Optional[torch.Tensor] = None, stream=None, errors: bool = False):
    """awq_apply_clip: per-group clip ratio chosen by the group's output error, then the
    packed clipped weights.  Returns (qweight, scales, qzeros or None, clip index uint8
    [N][K/G]), plus the errors fp64 [N][K/G][n_clip] when `errors`."""
    M, K = X.shape
    N = W.shape[0]
    lib = load_library()
    if workspace is None:
        need = int(lib.awq_apply_clip_workspace_bytes(M, N, K, config(group_size, zero_point), n_clip))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    qs, ss, zs = packed_shapes(N, K, group_size, zero_point)
    if out is None:
        qweight = torch.empty(qs, dtype=torch.int32, device=W.device)
        scales = torch.empty(ss, dtype=torch.float16, device=W.device)
        qzeros = torch.empty(zs, dtype=torch.int32, device=W.device) if zero_point else None
        idx = torch.empty((N, K // group_size), dtype=torch.uint8, device=W.device)
    else:
        qweight, scales, qzeros, idx = out
    err = torch.empty((N, K // group_size, n_clip), dtype=torch.float64, device=W.device) if errors else None
    st = lib.awq_apply_clip(
        _dev(X, "X", _F16), M, _dev(W, "W", _F16), _dev(s, "s", _F16), N, K, config(group_size, zero_point),
        n_grid, n_clip, _dev(qweight, "qweight", _W32), _dev(scales, "scales", _F16), _dev(qzeros, "qzeros", _W32),
        0 if idx is None else idx.data_ptr(), 0 if err is None else err.data_ptr(), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("awq_apply_clip", st)
    if errors:
        return qweight, scales, qzeros, idx, err
    return qweight, scales, qzeros, idx
