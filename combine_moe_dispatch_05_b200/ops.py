"""Thin Python binding of the C ABI in include/moe_dispatch.h.

Every function here only checks tensor types and shapes, allocates outputs
when the caller did not pass them, and forwards raw device pointers, sizes and
the current CUDA stream to the library.  All arithmetic runs in the CUDA kernels
of libmoe_dispatch.so; there is no fallback: if the library is missing or a
tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_dispatch.so")

OK, ERR_INVALID_ARG, ERR_EXPERT_RANGE, ERR_DUPLICATE_EXPERT = 0, 1, 2, 3
ERR_CAPACITY, ERR_TIMEOUT, ERR_CUDA, ERR_UNSUPPORTED, ERR_BOUNDS = 4, 5, 6, 7, 8
DTYPE_BF16, DTYPE_E4M3 = 0, 1
TILE = 128

# name -> (restype, argtypes); the exported C entry points, in header order
_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_int]),
    "moe_version": (_int, []),
    "moe_padded_capacity": (_i64, [_i64, _int, _int]),
    "moe_layout_workspace_bytes": (_sz, [_i64, _int, _int]),
    "moe_dispatch_layout": (_int, [_vp, _i64, _int, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _i64, _vp, _vp, _sz, _vp]),
    "moe_dispatch_layout_static": (_int, [_vp, _i64, _int, _int, _int, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _i64, _vp, _vp]),
    "moe_dispatch_permute": (_int, [_vp, _int, _i64, _int, _i64, _vp, _i64, _vp, _int, _vp, _vp,
                                    _int, _vp, _vp, _i64, _vp, _vp, _vp, _vp]),
    "moe_dispatch": (_int, [_vp, _i64, _int, _int, _int, _vp, _int, _int, _i64, _vp, _i64, _vp,
                            _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp, _vp, _vp,
                            _vp]),
    "moe_dispatch_permute_consume": (_int, [_vp, _int, _i64, _int, _i64, _vp, _i64, _vp, _int,
                                            _vp, _vp, _int, _vp, _vp, _vp, _i64, _vp, _vp, _i64,
                                            _vp, _vp]),
    "moe_dispatch_permute_quant": (_int, [_vp, _i64, _int, _i64, _vp, _int, _vp, _vp, _int, _vp,
                                          _vp, _i64, _vp, _vp, _vp, _vp]),
    "moe_combine": (_int, [_vp, _vp, _vp, _vp, _i64, _int, _int, _i64, _vp, _vp, _vp]),
    "moe_combine_bwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _i64, _vp,
                               _vp, _vp, _vp]),
    "moe_dispatch_bwd": (_int, [_vp, _vp, _i64, _int, _int, _i64, _vp, _vp, _vp]),
    "moe_quantize_e4m3": (_int, [_vp, _i64, _int, _i64, _vp, _vp, _vp, _vp]),
    "moe_plan_balance": (_int, [_vp, _int, _int, _vp, ctypes.c_double, _int, _vp, _vp, _vp,
                                _vp]),
    "moe_wait_tiles_checksum": (_int, [_vp, _vp, _int, _vp, _i64, _vp, _int, _i64, _vp, _i64,
                                       _vp, _vp]),
}

_lib = None


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def lib() -> ctypes.CDLL:
    """Loads libmoe_dispatch.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                              f"(run `python -m combine_moe_dispatch_05_b200.build`)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != OK:
        raise MoEError(rc, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, name: str, dtype=None, contiguous=True):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# --------------------------------------------------------------- status --
def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def read_status(status: torch.Tensor) -> int:
    """Synchronises with the status tensor's producer and returns its value."""
    return int(status.item())


def raise_on_status(status: torch.Tensor, where: str = "device"):
    v = read_status(status)
    if v != OK:
        raise MoEError(v, where)


# ---------------------------------------------------------------- sizes --
def padded_capacity(T: int, K: int, E: int) -> int:
    v = lib().moe_padded_capacity(T, K, E)
    if v < 0:
        raise ValueError("bad sizes")
    return int(v)


def layout_workspace_bytes(T: int, K: int, E: int) -> int:
    v = lib().moe_layout_workspace_bytes(T, K, E)
    if v == ctypes.c_size_t(-1).value:
        raise ValueError("bad sizes")
    return int(v)


# --------------------------------------------------------------- layout --
@dataclasses.dataclass
class Layout:
    T: int
    K: int
    E: int
    R: int
    P_cap: int
    expert_counts: torch.Tensor
    expert_offsets: torch.Tensor
    rank_counts: torch.Tensor
    rank_offsets: torch.Tensor
    dst_row: torch.Tensor
    row_src: Optional[torch.Tensor]
    tile_ready: Optional[torch.Tensor]
    workspace: Optional[torch.Tensor]   # None for layouts filled by moe_dispatch_layout_static
    work: torch.Tensor                  # permute's scheduling words: int32 [2], zero between calls


def alloc_layout(T: int, K: int, E: int, R: int, device, P_cap: Optional[int] = None,
                 with_row_src=True, with_counters=True, with_workspace=True) -> Layout:
    P_cap = padded_capacity(T, K, E) if P_cap is None else P_cap
    i32 = dict(dtype=torch.int32, device=device)
    ws = torch.empty(max(1, layout_workspace_bytes(T, K, E)), dtype=torch.uint8,
                     device=device) if with_workspace else None
    return Layout(
        T, K, E, R, P_cap,
        torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R, **i32),
        torch.empty(R + 1, **i32), torch.empty(max(T * K, 1), **i32),
        torch.empty(max(P_cap, 1), **i32) if with_row_src else None,
        torch.empty(max((P_cap + TILE - 1) // TILE, 1), dtype=torch.int32, device=device)
        if with_counters else None,
        ws, torch.zeros(2, **i32))


def moe_dispatch_layout(topk_idx: torch.Tensor, E: int, R: int, layout: Optional[Layout] = None,
                        status: Optional[torch.Tensor] = None, P_cap: Optional[int] = None,
                        stream=None) -> Layout:
    _cuda(topk_idx, "topk_idx", torch.int32)
    T, K = topk_idx.shape
    L = layout or alloc_layout(T, K, E, R, topk_idx.device, P_cap)
    if L.workspace is None:
        raise ValueError("this layout has no workspace (use moe_dispatch_layout_static)")
    rc = lib().moe_dispatch_layout(
        _ptr(topk_idx), T, K, E, R, _ptr(L.expert_counts), _ptr(L.expert_offsets),
        _ptr(L.rank_counts), _ptr(L.rank_offsets), _ptr(L.dst_row), _ptr(L.row_src),
        _ptr(L.tile_ready), L.P_cap, _ptr(status), _ptr(L.workspace), L.workspace.numel(),
        _stream(stream))
    _check(rc, "moe_dispatch_layout")
    return L


def moe_dispatch_layout_static(topk_idx: torch.Tensor, E: int, R: int,
                               layout: Optional[Layout] = None,
                               status: Optional[torch.Tensor] = None,
                               P_cap: Optional[int] = None, stream=None) -> Layout:
    """moe_dispatch_layout without a workspace, for callers that cannot
    allocate device memory at call time: the library's own static scratch is
    used.  Outputs are still the caller's: pass ``layout`` (for instance from
    ``alloc_layout(..., with_workspace=False)`` at start-up) so that this call
    allocates nothing; without it the output tensors, and only those, are
    allocated here."""
    _cuda(topk_idx, "topk_idx", torch.int32)
    T, K = topk_idx.shape
    L = layout or alloc_layout(T, K, E, R, topk_idx.device, P_cap, with_workspace=False)
    rc = lib().moe_dispatch_layout_static(
        _ptr(topk_idx), T, K, E, R, _ptr(L.expert_counts), _ptr(L.expert_offsets),
        _ptr(L.rank_counts), _ptr(L.rank_offsets), _ptr(L.dst_row), _ptr(L.row_src),
        _ptr(L.tile_ready), L.P_cap, _ptr(status), _stream(stream))
    _check(rc, "moe_dispatch_layout_static")
    return L


# -------------------------------------------------------------- permute --
def moe_dispatch_permute(x: torch.Tensor, L: Layout, xp: Optional[torch.Tensor] = None,
                         x_scales: Optional[torch.Tensor] = None,
                         xp_scales: Optional[torch.Tensor] = None, use_counters: bool = True,
                         status: Optional[torch.Tensor] = None, stream=None):
    """bf16 rows (x.dtype == bfloat16) or E4M3 codes (x.dtype == uint8 or
    float8_e4m3fn, with x_scales fp32 [T, H/128]).  Returns xp (and xp_scales)."""
    _cuda(x, "x", contiguous=False)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, H = x.shape
    if T != L.T:
        raise ValueError(f"x has {T} rows but the layout was built for {L.T} tokens")
    if x.dtype == torch.bfloat16:
        dt, el = DTYPE_BF16, torch.bfloat16
    elif x.dtype in (torch.uint8, torch.float8_e4m3fn):
        dt, el = DTYPE_E4M3, x.dtype
    else:
        raise TypeError("x must be bfloat16 or E4M3 (uint8 / float8_e4m3fn)")
    if xp is None:
        xp = torch.empty((L.P_cap, H), dtype=el, device=x.device)
    _shape(_cuda(xp, "xp"), "xp", (L.P_cap, H))
    xs_stride = 0
    if dt == DTYPE_E4M3:
        _cuda(x_scales, "x_scales", torch.float32, contiguous=False)
        _shape(x_scales, "x_scales", (T, H // 128))
        xs_stride = x_scales.stride(0)
        if xp_scales is None:
            xp_scales = torch.empty((L.P_cap, H // 128), dtype=torch.float32, device=x.device)
        _shape(_cuda(xp_scales, "xp_scales", torch.float32), "xp_scales", (L.P_cap, H // 128))
    rc = lib().moe_dispatch_permute(
        _ptr(x), dt, T, H, x.stride(0), _ptr(x_scales), xs_stride, _ptr(L.dst_row), L.K,
        _ptr(L.expert_counts), _ptr(L.expert_offsets), L.E, _ptr(xp), _ptr(xp_scales), L.P_cap,
        _ptr(L.tile_ready) if use_counters else None, _ptr(L.work), _ptr(status),
        _stream(stream))
    _check(rc, "moe_dispatch_permute")
    return (xp, xp_scales) if dt == DTYPE_E4M3 else xp


def moe_dispatch(topk_idx: torch.Tensor, x: torch.Tensor, E: int, R: int,
                 layout: Optional[Layout] = None, xp: Optional[torch.Tensor] = None,
                 x_scales: Optional[torch.Tensor] = None,
                 xp_scales: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                 P_cap: Optional[int] = None, stream=None):
    """moe_dispatch_layout followed by moe_dispatch_permute in one call (the
    permute's first row loads overlap the layout).  Returns (layout, xp) or,
    for E4M3 codes, (layout, xp, xp_scales)."""
    _cuda(topk_idx, "topk_idx", torch.int32)
    _cuda(x, "x", contiguous=False)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, K = topk_idx.shape
    if x.shape[0] != T:
        raise ValueError(f"x has {x.shape[0]} rows but topk_idx has {T}")
    H = x.shape[1]
    if x.dtype == torch.bfloat16:
        dt, el = DTYPE_BF16, torch.bfloat16
    elif x.dtype in (torch.uint8, torch.float8_e4m3fn):
        dt, el = DTYPE_E4M3, x.dtype
    else:
        raise TypeError("x must be bfloat16 or E4M3 (uint8 / float8_e4m3fn)")
    L = layout or alloc_layout(T, K, E, R, topk_idx.device, P_cap)
    if L.workspace is None:
        raise ValueError("this layout has no workspace")
    if xp is None:
        xp = torch.empty((L.P_cap, H), dtype=el, device=x.device)
    _shape(_cuda(xp, "xp"), "xp", (L.P_cap, H))
    xs_stride = 0
    if dt == DTYPE_E4M3:
        _cuda(x_scales, "x_scales", torch.float32, contiguous=False)
        _shape(x_scales, "x_scales", (T, H // 128))
        xs_stride = x_scales.stride(0)
        if xp_scales is None:
            xp_scales = torch.empty((L.P_cap, H // 128), dtype=torch.float32, device=x.device)
        _shape(_cuda(xp_scales, "xp_scales", torch.float32), "xp_scales", (L.P_cap, H // 128))
    rc = lib().moe_dispatch(
        _ptr(topk_idx), T, K, E, R, _ptr(x), dt, H, x.stride(0), _ptr(x_scales), xs_stride,
        _ptr(L.expert_counts), _ptr(L.expert_offsets), _ptr(L.rank_counts), _ptr(L.rank_offsets),
        _ptr(L.dst_row), _ptr(L.row_src), _ptr(L.tile_ready), L.P_cap, _ptr(L.workspace),
        L.workspace.numel(), _ptr(xp), _ptr(xp_scales), _ptr(L.work), _ptr(status),
        _stream(stream))
    _check(rc, "moe_dispatch")
    return (L, xp, xp_scales) if dt == DTYPE_E4M3 else (L, xp)


def moe_dispatch_permute_consume(x: torch.Tensor, L: Layout, xp: Optional[torch.Tensor] = None,
                                 x_scales: Optional[torch.Tensor] = None,
                                 xp_scales: Optional[torch.Tensor] = None,
                                 checksums: Optional[torch.Tensor] = None,
                                 timeout_ns: int = 10**9, status: Optional[torch.Tensor] = None,
                                 stream=None):
    """Permute with a concurrent tile consumer in one cooperative launch.
    Returns (xp[, xp_scales], checksums)."""
    _cuda(x, "x", contiguous=False)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, H = x.shape
    if T != L.T:
        raise ValueError(f"x has {T} rows but the layout was built for {L.T} tokens")
    if x.dtype == torch.bfloat16:
        dt = DTYPE_BF16
    elif x.dtype in (torch.uint8, torch.float8_e4m3fn):
        dt = DTYPE_E4M3
    else:
        raise TypeError("x must be bfloat16 or E4M3 (uint8 / float8_e4m3fn)")
    if xp is None:
        xp = torch.empty((L.P_cap, H), dtype=x.dtype, device=x.device)
    _shape(_cuda(xp, "xp"), "xp", (L.P_cap, H))
    xs_stride = 0
    if dt == DTYPE_E4M3:
        _cuda(x_scales, "x_scales", torch.float32, contiguous=False)
        _shape(x_scales, "x_scales", (T, H // 128))
        xs_stride = x_scales.stride(0)
        if xp_scales is None:
            xp_scales = torch.empty((L.P_cap, H // 128), dtype=torch.float32, device=x.device)
        _shape(_cuda(xp_scales, "xp_scales", torch.float32), "xp_scales", (L.P_cap, H // 128))
    if checksums is None:
        checksums = torch.zeros(max((L.P_cap + TILE - 1) // TILE, 1), dtype=torch.int32,
                                device=x.device)
    rc = lib().moe_dispatch_permute_consume(
        _ptr(x), dt, T, H, x.stride(0), _ptr(x_scales), xs_stride, _ptr(L.dst_row), L.K,
        _ptr(L.expert_counts), _ptr(L.expert_offsets), L.E, _ptr(L.row_src), _ptr(xp),
        _ptr(xp_scales), L.P_cap, _ptr(L.tile_ready), _ptr(checksums), timeout_ns, _ptr(status),
        _stream(stream))
    _check(rc, "moe_dispatch_permute_consume")
    return (xp, xp_scales, checksums) if dt == DTYPE_E4M3 else (xp, checksums)


def moe_dispatch_permute_quant(x: torch.Tensor, L: Layout, xp: Optional[torch.Tensor] = None,
                               xp_scales: Optional[torch.Tensor] = None,
                               use_counters: bool = True, status: Optional[torch.Tensor] = None,
                               stream=None):
    """bf16 rows -> E4M3 codes + per-128-channel scales, written straight into
    the expert-major buffer.  Returns (xp uint8 [P_cap, H], xp_scales)."""
    _cuda(x, "x", torch.bfloat16, contiguous=False)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, H = x.shape
    if T != L.T:
        raise ValueError(f"x has {T} rows but the layout was built for {L.T} tokens")
    if xp is None:
        xp = torch.empty((L.P_cap, H), dtype=torch.uint8, device=x.device)
    if xp_scales is None:
        xp_scales = torch.empty((L.P_cap, H // 128), dtype=torch.float32, device=x.device)
    _shape(_cuda(xp, "xp"), "xp", (L.P_cap, H))
    _shape(_cuda(xp_scales, "xp_scales", torch.float32), "xp_scales", (L.P_cap, H // 128))
    rc = lib().moe_dispatch_permute_quant(
        _ptr(x), T, H, x.stride(0), _ptr(L.dst_row), L.K, _ptr(L.expert_counts),
        _ptr(L.expert_offsets), L.E, _ptr(xp), _ptr(xp_scales), L.P_cap,
        _ptr(L.tile_ready) if use_counters else None, _ptr(L.work), _ptr(status),
        _stream(stream))
    _check(rc, "moe_dispatch_permute_quant")
    return xp, xp_scales


# -------------------------------------------------------------- combine --
def moe_combine(y: torch.Tensor, dst_row: torch.Tensor, scales: torch.Tensor,
                shared_x: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                P_cap: Optional[int] = None, status: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    _cuda(y, "y", torch.bfloat16)
    _cuda(dst_row, "dst_row", torch.int32)
    _cuda(scales, "scales", torch.float32)
    T, K = scales.shape
    H = y.shape[1]
    if dst_row.numel() < T * K:
        raise ValueError(f"dst_row has {dst_row.numel()} entries, needs T*K = {T * K}")
    if P_cap is not None and P_cap > y.shape[0]:
        raise ValueError(f"P_cap={P_cap} exceeds the {y.shape[0]} rows of y")
    if shared_x is not None:
        _shape(_cuda(shared_x, "shared_x", torch.bfloat16), "shared_x", (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    _shape(_cuda(out, "out", torch.bfloat16), "out", (T, H))
    rc = lib().moe_combine(_ptr(y), _ptr(dst_row), _ptr(scales), _ptr(shared_x), T, K, H,
                           y.shape[0] if P_cap is None else P_cap, _ptr(out), _ptr(status),
                           _stream(stream))
    _check(rc, "moe_combine")
    return out


def moe_combine_bwd(grad_out: torch.Tensor, y: torch.Tensor, scales: torch.Tensor, L: Layout,
                    grad_y: Optional[torch.Tensor] = None,
                    grad_scales: Optional[torch.Tensor] = None,
                    status: Optional[torch.Tensor] = None, stream=None):
    _cuda(grad_out, "grad_out", torch.bfloat16)
    _cuda(y, "y", torch.bfloat16)
    _cuda(scales, "scales", torch.float32)
    T, K = scales.shape
    H = grad_out.shape[1]
    _shape(grad_out, "grad_out", (T, H))
    if (T, K) != (L.T, L.K):
        raise ValueError(f"scales is {T}x{K} but the layout was built for {L.T}x{L.K}")
    if y.shape[0] < L.P_cap or y.shape[1] != H:
        raise ValueError(f"y must have at least P_cap={L.P_cap} rows of {H}, got "
                         f"{tuple(y.shape)}")
    if grad_y is None:
        grad_y = torch.empty((L.P_cap, H), dtype=torch.bfloat16, device=y.device)
    if grad_scales is None:
        grad_scales = torch.empty((T, K), dtype=torch.float32, device=y.device)
    _shape(_cuda(grad_y, "grad_y", torch.bfloat16), "grad_y", (L.P_cap, H))
    _shape(_cuda(grad_scales, "grad_scales", torch.float32), "grad_scales", (T, K))
    rc = lib().moe_combine_bwd(_ptr(grad_out), _ptr(y), _ptr(scales), _ptr(L.dst_row),
                               _ptr(L.expert_counts), _ptr(L.expert_offsets), L.E, T, K, H,
                               L.P_cap, _ptr(grad_y), _ptr(grad_scales), _ptr(status),
                               _stream(stream))
    _check(rc, "moe_combine_bwd")
    return grad_y, grad_scales


def moe_dispatch_bwd(grad_xp: torch.Tensor, dst_row: torch.Tensor, T: int, K: int,
                     grad_x: Optional[torch.Tensor] = None, P_cap: Optional[int] = None,
                     status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _cuda(grad_xp, "grad_xp", torch.bfloat16)
    _cuda(dst_row, "dst_row", torch.int32)
    H = grad_xp.shape[1]
    if dst_row.numel() < T * K:
        raise ValueError(f"dst_row has {dst_row.numel()} entries, needs T*K = {T * K}")
    if P_cap is not None and P_cap > grad_xp.shape[0]:
        raise ValueError(f"P_cap={P_cap} exceeds the {grad_xp.shape[0]} rows of grad_xp")
    if grad_x is None:
        grad_x = torch.empty((T, H), dtype=torch.bfloat16, device=grad_xp.device)
    _shape(_cuda(grad_x, "grad_x", torch.bfloat16), "grad_x", (T, H))
    rc = lib().moe_dispatch_bwd(_ptr(grad_xp), _ptr(dst_row), T, K, H,
                                grad_xp.shape[0] if P_cap is None else P_cap, _ptr(grad_x),
                                _ptr(status), _stream(stream))
    _check(rc, "moe_dispatch_bwd")
    return grad_x


# ------------------------------------------------------------------ fp8 --
def moe_quantize_e4m3(x: torch.Tensor, q: Optional[torch.Tensor] = None,
                      q_scales: Optional[torch.Tensor] = None,
                      status: Optional[torch.Tensor] = None, stream=None):
    _cuda(x, "x", torch.bfloat16, contiguous=False)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, H = x.shape
    if q is None:
        q = torch.empty((T, H), dtype=torch.uint8, device=x.device)
    if q_scales is None:
        q_scales = torch.empty((T, H // 128), dtype=torch.float32, device=x.device)
    _shape(_cuda(q, "q"), "q", (T, H))
    _shape(_cuda(q_scales, "q_scales", torch.float32), "q_scales", (T, H // 128))
    rc = lib().moe_quantize_e4m3(_ptr(x), T, H, x.stride(0), _ptr(q), _ptr(q_scales),
                                 _ptr(status), _stream(stream))
    _check(rc, "moe_quantize_e4m3")
    return q, q_scales


# ------------------------------------------------------------- counters --
def moe_wait_tiles_checksum(L: Layout, xp: torch.Tensor, xp_scales: Optional[torch.Tensor] = None,
                            checksums: Optional[torch.Tensor] = None, timeout_ns: int = 10**9,
                            status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _cuda(xp, "xp")
    if checksums is None:
        checksums = torch.zeros(max((L.P_cap + TILE - 1) // TILE, 1), dtype=torch.int32,
                                device=xp.device)
    row_bytes = xp.shape[1] * xp.element_size()
    sc = 0 if xp_scales is None else xp_scales.shape[1]
    rc = lib().moe_wait_tiles_checksum(_ptr(L.tile_ready), _ptr(L.expert_offsets), L.E, _ptr(xp),
                                       row_bytes, _ptr(xp_scales), sc, L.P_cap, _ptr(checksums),
                                       timeout_ns, _ptr(status), _stream(stream))
    _check(rc, "moe_wait_tiles_checksum")
    return checksums


# -------------------------------------------------------------- planner --
class _Move(ctypes.Structure):
    _fields_ = [("expert", ctypes.c_int32), ("src_rank", ctypes.c_int32),
                ("dst_rank", ctypes.c_int32), ("tokens", ctypes.c_int32)]


class _Cost(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in ("a", "b", "b2", "c", "beta", "mig")]


def moe_plan_balance(expert_counts, R: int, a=0.0, b=1.0, b2=0.0, c=0.0, beta=0.01, mig=0.0,
                     min_gain=0.0, max_moves=256):
    """Host planner (no GPU).  expert_counts: host sequence of E ints.
    Returns (moves [(expert, src, dst, tokens)], makespan_before, makespan_after)."""
    counts = (ctypes.c_int32 * len(expert_counts))(*[int(v) for v in expert_counts])
    cost = _Cost(a, b, b2, c, beta, mig)
    moves = (_Move * max(max_moves, 1))()
    n = ctypes.c_int(0)
    mb, ma = ctypes.c_double(0.0), ctypes.c_double(0.0)
    rc = lib().moe_plan_balance(ctypes.cast(counts, _vp), len(expert_counts), R,
                                ctypes.cast(ctypes.pointer(cost), _vp), float(min_gain),
                                max_moves, ctypes.cast(moves, _vp), ctypes.byref(n),
                                ctypes.byref(mb), ctypes.byref(ma))
    _check(rc, "moe_plan_balance")
    out = [(m.expert, m.src_rank, m.dst_rank, m.tokens) for m in moves[:n.value]]
    return out, mb.value, ma.value
