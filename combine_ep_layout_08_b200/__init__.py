"""B200-native MoE expert-parallel permutation engine (dispatch layout,
dispatch, combine) -- Python binding.

This module only marshals arguments: every step runs in the CUDA kernels of
``libep.so`` behind the C ABI of ``include/ep.h``; PyTorch supplies device
memory and the current stream.  The function names are the C names.  There
is no CPU fallback: if the library is missing, every call raises.

Typical use::

    h = ep_handle_create(max_tokens=8192, num_topk=8, num_experts=256, num_ranks=8)
    ep_layout(h, topk_idx)                         # int64 [T, k] on the GPU
    recv_x, recv_scales = ep_dispatch(h, x, fmt="fp8")
    y = expert(recv_x, recv_scales)                # user code, receive layout
    out = ep_combine(h, y, topk_weights)           # bf16 [T, H]
    ep_handle_check(h)                             # raises on a device-side error

Also: ``ep_layout_dispatch`` (layout and dispatch in one launch for decode-
sized batches), fp16 rows (``fmt="fp16"`` / fp16 tensors), token ranges
(``ep_dispatch_range`` / ``ep_combine_range``), one receive buffer per
expert-parallel rank (``ep_allgather_topk``, ``ep_dispatch_ranks``,
``ep_combine_ranks``), GEMM-ready helpers (``fmt="fp8_mn"``,
``ep_dispatch_weights``, ``ep_zero_pad_rows``) and the backward
(``ep_dispatch_backward``, ``ep_combine_backward``).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "EPError", "EPHandle", "ep_workspace_bytes", "ep_recv_rows_upper_bound", "ep_handle_create",
    "ep_layout", "ep_layout_dispatch", "ep_handle_view", "ep_handle_read_counts", "ep_dispatch", "ep_combine",
    "ep_dispatch_range", "ep_combine_range", "ep_dispatch_backward", "ep_combine_backward",
    "ep_dispatch_weights", "ep_zero_pad_rows", "ep_dispatch_ranks", "ep_combine_ranks",
    "ep_dispatch_ranks_backward", "ep_combine_ranks_backward", "ep_allgather_topk",
    "ep_ipc_export", "ep_ipc_open", "ep_ipc_close", "ep_ipc_share", "IPCShare",
    "ep_handle_check", "ep_strerror", "library_path", "load_library",
    "EP_OK", "EP_ERR_INVALID_ARG", "EP_ERR_ALIGNMENT", "EP_ERR_WORKSPACE_TOO_SMALL",
    "EP_ERR_CAPACITY", "EP_ERR_BAD_INDEX", "EP_ERR_CUDA", "EP_ERR_STATE", "EP_ERR_NO_MEMORY",
    "EP_ERR_TIMEOUT",
]

EP_OK = 0
EP_ERR_INVALID_ARG = 1
EP_ERR_ALIGNMENT = 2
EP_ERR_WORKSPACE_TOO_SMALL = 3
EP_ERR_CAPACITY = 4
EP_ERR_BAD_INDEX = 5
EP_ERR_CUDA = 6
EP_ERR_STATE = 7
EP_ERR_NO_MEMORY = 8
EP_ERR_TIMEOUT = 9

EP_FMT_BF16 = 0
EP_FMT_FP8_E4M3_1X128 = 1
EP_FMT_FP8_E4M3_1X128_MN = 2
EP_FMT_FP16 = 3
_FMTS = {"bf16": EP_FMT_BF16, "fp8": EP_FMT_FP8_E4M3_1X128, "fp8_mn": EP_FMT_FP8_E4M3_1X128_MN,
         "fp16": EP_FMT_FP16}
EP_DTYPE_BF16 = 0
EP_DTYPE_FP16 = 1
_DTYPES = {torch.bfloat16: EP_DTYPE_BF16, torch.float16: EP_DTYPE_FP16}
_COPY_FMT = {torch.bfloat16: EP_FMT_BF16, torch.float16: EP_FMT_FP16}


def _fmt_code(fmt: Optional[str], dtype: torch.dtype) -> int:
    """Format code; None or "copy" means the rows in the input's own 16-bit type."""
    if fmt is None or fmt == "copy":
        return _COPY_FMT[dtype]
    return _FMTS[fmt]


def _is_copy(f: int) -> bool:
    return f in (EP_FMT_BF16, EP_FMT_FP16)

VIEWS = {
    "num_tokens_per_expert": (0, torch.int32),
    "num_tokens_per_rank": (1, torch.int32),
    "num_rows_per_rank": (2, torch.int32),
    "expert_off": (3, torch.int32),
    "rank_off": (4, torch.int32),
    "is_token_in_rank": (5, torch.uint8),
    "dst_row": (6, torch.int32),
    "recv_src": (7, torch.int32),
    "total_recv_rows": (8, torch.int32),
    "error_words": (9, torch.int32),
}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libep.so")
_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libep.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:  # loaded: no lock on the per-call path
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                "libep.so is missing at %s; build it with "
                "`python -m combine_ep_layout_08_b200._build` (nvcc, sm_100a). "
                "There is no CPU fallback." % _LIB_PATH)
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sigs = {
            "ep_workspace_bytes": ([I, I, I, I, I], SZ),
            "ep_recv_rows_upper_bound": ([I, I, I, I], I64),
            "ep_handle_create": ([P, SZ, I, I, I, I, I, ctypes.POINTER(P)], I),
            "ep_handle_destroy": ([P], None),
            "ep_layout": ([P, P, I, P], I),
            "ep_layout_dispatch": ([P, P, I, P, I, I, P, P, I64, P], I),
            "ep_handle_view": ([P, I, ctypes.POINTER(I64)], P),
            "ep_handle_read_counts": ([P, P, P, P, P, P], I),
            "ep_dispatch": ([P, P, I, I, P, P, I64, P], I),
            "ep_combine": ([P, P, I64, P, I, P, P], I),
            "ep_dispatch_ex": ([P, P, I, I, I, P, P, I64, P], I),
            "ep_dispatch_ranks": ([P, I, I, P, I, I, P, P, P, P], I),
            "ep_dispatch_backward_ex": ([P, P, I64, I, I, P, P], I),
            "ep_dispatch_ranks_backward": ([P, I, I, P, P, I, I, P, P], I),
            "ep_combine_ranks_backward": ([P, I, I, P, P, P, P, I, I, P, P, P, P], I),
            "ep_combine_backward_ex": ([P, P, P, I64, P, I, I, P, I64, P, P], I),
            "ep_combine_ranks": ([P, I, I, P, P, P, I, I, P, P], I),
            "ep_combine_ex": ([P, P, I64, P, I, I, P, P], I),
            "ep_dispatch_range": ([P, I, I, P, I, I, P, P, I64, P], I),
            "ep_dispatch_backward": ([P, P, I64, I, P, P], I),
            "ep_dispatch_weights": ([P, P, P, I64, P], I),
            "ep_zero_pad_rows": ([P, P, I64, I64, P], I),
            "ep_combine_backward": ([P, P, P, I64, P, I, P, I64, P, P], I),
            "ep_combine_range": ([P, I, I, P, I64, P, I, P, P], I),
            "ep_handle_check": ([P, P], I),
            "ep_ipc_export": ([P, P, ctypes.POINTER(ctypes.c_uint64)], I),
            "ep_ipc_open": ([P, ctypes.c_uint64, ctypes.POINTER(P), ctypes.POINTER(P)], I),
            "ep_ipc_close": ([P], I),
            "ep_strerror": ([I], ctypes.c_char_p),
            "ep_last_error_message": ([], ctypes.c_char_p),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


class EPError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load_library()
        msg = lib.ep_strerror(status).decode()
        if status == EP_ERR_CUDA:
            msg += " -- " + lib.ep_last_error_message().decode()
        super().__init__("%s: %s" % (where, msg))
        self.status = status


def _check(status: int, where: str):
    if status != EP_OK:
        raise EPError(status, where)


def ep_strerror(status: int) -> str:
    return load_library().ep_strerror(status).decode()


# PyTorch's raw current-stream getter (no Stream object per call), where this
# build of PyTorch has it; the public API otherwise.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device):
    if _raw_stream is not None:
        return _raw_stream(device.index)
    return torch.cuda.current_stream(device).cuda_stream


class _NoSwitch:
    """The handle's device is already current: nothing to switch."""

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_NO_SWITCH = _NoSwitch()


def _on(h: "EPHandle"):
    """Make the handle's device current for the duration of a library call."""
    if torch.cuda.current_device() == h.device.index:
        return _NO_SWITCH
    return torch.cuda.device(h.device)


def _ptr(t: Optional[torch.Tensor]):
    return t.data_ptr() if t is not None and t.numel() > 0 else None


def ep_workspace_bytes(max_tokens: int, num_topk: int, num_experts: int, num_ranks: int,
                       block_m: int = 128) -> int:
    return int(load_library().ep_workspace_bytes(max_tokens, num_topk, num_experts, num_ranks,
                                                 block_m))


def ep_recv_rows_upper_bound(T: int, num_topk: int, num_experts: int, block_m: int = 128) -> int:
    return int(load_library().ep_recv_rows_upper_bound(T, num_topk, num_experts, block_m))


class EPHandle:
    """Owns the device workspace (a torch uint8 tensor) and the C handle."""

    def __init__(self, max_tokens: int, num_topk: int, num_experts: int, num_ranks: int,
                 block_m: int = 128, device=None):
        lib = load_library()
        device = torch.device("cuda") if device is None else torch.device(device)
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.device = device
        self.max_tokens, self.k, self.E, self.R, self.block_m = (
            max_tokens, num_topk, num_experts, num_ranks, block_m)
        nbytes = ep_workspace_bytes(max_tokens, num_topk, num_experts, num_ranks, block_m)
        if nbytes == 0:
            raise EPError(EP_ERR_INVALID_ARG, "ep_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(lib.ep_handle_create(_ptr(self.workspace), nbytes, max_tokens, num_topk,
                                    num_experts, num_ranks, block_m, ctypes.byref(h)),
               "ep_handle_create")
        self._h = h
        self.T = None

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load_library().ep_handle_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ep_handle_create(max_tokens: int, num_topk: int, num_experts: int, num_ranks: int,
                     block_m: int = 128, device=None) -> EPHandle:
    return EPHandle(max_tokens, num_topk, num_experts, num_ranks, block_m, device)


def ep_layout(h: EPHandle, topk_idx: torch.Tensor) -> None:
    """get_dispatch_layout of int64 [T, k] top-k indices (-1 = unused slot)."""
    if topk_idx.dtype != torch.int64 or topk_idx.dim() != 2 or topk_idx.shape[1] != h.k:
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout: topk_idx must be int64 [T, %d]" % h.k)
    if not topk_idx.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout: topk_idx must be contiguous")
    _same_device(h, "ep_layout", topk_idx)
    T = topk_idx.shape[0]
    with _on(h):
        _check(load_library().ep_layout(h.handle, _ptr(topk_idx), T, _stream(h.device)),
               "ep_layout")
    h.T = T


def ep_handle_view(h: EPHandle, what: str) -> torch.Tensor:
    """A tensor view of one layout array inside the workspace (no copy)."""
    code, dtype = VIEWS[what]
    n = ctypes.c_int64()
    p = load_library().ep_handle_view(h.handle, code, ctypes.byref(n))
    if not p:
        raise EPError(EP_ERR_INVALID_ARG, "ep_handle_view(%s)" % what)
    off = p - h.workspace.data_ptr()
    nbytes = n.value * torch.empty((), dtype=dtype).element_size()
    v = h.workspace[off: off + nbytes].view(dtype)
    T = h.T or 0
    if what == "is_token_in_rank":
        v = v.view(T, h.R)
    elif what == "dst_row":
        v = v.view(T, h.k)
    return v


def ep_handle_read_counts(h: EPHandle) -> dict:
    """Counts of the last layout, copied to the host (synchronises the stream)."""
    import numpy as np

    a = np.zeros(h.E, np.int32)
    b = np.zeros(h.R, np.int32)
    c = np.zeros(h.R, np.int32)
    d = np.zeros(1, np.int32)
    with _on(h):
        _check(load_library().ep_handle_read_counts(
            h.handle, a.ctypes.data_as(ctypes.c_void_p), b.ctypes.data_as(ctypes.c_void_p),
            c.ctypes.data_as(ctypes.c_void_p), d.ctypes.data_as(ctypes.c_void_p),
            _stream(h.device)), "ep_handle_read_counts")
    return dict(num_tokens_per_expert=a, num_tokens_per_rank=b, num_rows_per_rank=c,
                total_recv_rows=int(d[0]))


def _same_device(h: EPHandle, where: str, *tensors) -> None:
    """Every tensor given (None skipped) lives on the handle's device."""
    for t in tensors:
        if t is not None and t.device != h.device:
            raise EPError(EP_ERR_INVALID_ARG, "%s: tensors must be on %s" % (where, h.device))


def _rank_list(h: EPHandle, where: str, tensors) -> None:
    """Per-rank buffers: 2-D, on a device of the handle's kind (CUDA; other
    GPUs' buffers, seen as peers, are allowed)."""
    for t in tensors:
        if t.device.type != h.device.type or t.dim() != 2:
            raise EPError(EP_ERR_INVALID_ARG, "%s: per-rank buffers must be 2-D %s tensors"
                          % (where, h.device.type))


def _check_recv(where: str, H: int, f: int, recv_x, recv_scales):
    """Receive buffers of format f: recv_x [cap, H] of the format's type; FP8
    scales f32 [>= cap, H/128] (row-major) or [H/128, cap] (MN-major)."""
    want = _recv_dtype(f)
    if (recv_x.dtype != want or recv_x.dim() != 2 or recv_x.shape[1] != H
            or not recv_x.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "%s: recv_x must be contiguous %s [*, %d]"
                      % (where, want, H))
    cap = recv_x.shape[0]
    if _is_copy(f):
        return
    if recv_scales is None or recv_scales.dtype != torch.float32 or recv_scales.dim() != 2 \
            or not recv_scales.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "%s: FP8 needs contiguous f32 recv_scales" % where)
    if f == EP_FMT_FP8_E4M3_1X128 and (recv_scales.shape[0] < cap
                                       or recv_scales.shape[1] != H // 128):
        raise EPError(EP_ERR_INVALID_ARG, "%s: recv_scales must be f32 [cap, H/128]" % where)
    if f == EP_FMT_FP8_E4M3_1X128_MN and tuple(recv_scales.shape) != (H // 128, cap):
        raise EPError(EP_ERR_INVALID_ARG, "%s: recv_scales must be f32 [H/128, cap]" % where)


def _recv_buffers(h: EPHandle, T: int, H: int, f: int, device, recv_x, recv_scales,
                  capacity_rows, where: str):
    """Allocate missing receive buffers (default capacity: the no-sync bound)
    and check them."""
    if recv_x is None:
        cap = capacity_rows if capacity_rows is not None else \
            ep_recv_rows_upper_bound(T, h.k, h.E, h.block_m)
        if f == EP_FMT_FP8_E4M3_1X128_MN:
            cap = (cap + 3) // 4 * 4
        recv_x = torch.empty((cap, H), dtype=_recv_dtype(f), device=device)
    cap = recv_x.shape[0]
    if f == EP_FMT_FP8_E4M3_1X128 and recv_scales is None:
        recv_scales = torch.empty((cap, H // 128), dtype=torch.float32, device=device)
    if f == EP_FMT_FP8_E4M3_1X128_MN and recv_scales is None:
        recv_scales = torch.empty((H // 128, cap), dtype=torch.float32, device=device)
    _check_recv(where, H, f, recv_x, recv_scales)
    _same_device(h, where, recv_x, recv_scales)
    return recv_x, (recv_scales if not _is_copy(f) else None)


def _recv_dtype(f: int) -> torch.dtype:
    return {EP_FMT_BF16: torch.bfloat16, EP_FMT_FP16: torch.float16}.get(f, torch.float8_e4m3fn)


def ep_dispatch(h: EPHandle, x: torch.Tensor, fmt: Optional[str] = None,
                recv_x: Optional[torch.Tensor] = None, recv_scales: Optional[torch.Tensor] = None,
                capacity_rows: Optional[int] = None):
    """Scatter x [T, H] (bf16 or fp16) into the receive layout.  Returns
    (recv_x, recv_scales); recv_scales is None for the row copies.  Buffers not
    given are allocated with capacity_rows rows (default: the no-sync upper
    bound).  fmt: None / "copy" (rows in x's type), "bf16", "fp16", "fp8"
    (row-major scales [cap, H/128]) or "fp8_mn" (MN-major scales [H/128, cap])."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch")
    if (x.dtype not in _DTYPES or x.dim() != 2 or x.shape[0] != h.T
            or not x.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch: x must be contiguous bf16/fp16 [T, H]")
    T, H = x.shape
    f = _fmt_code(fmt, x.dtype)
    if _is_copy(f) and f != _COPY_FMT[x.dtype]:
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch: a row copy keeps x's type")
    _same_device(h, "ep_dispatch", x)
    recv_x, recv_scales = _recv_buffers(h, T, H, f, x.device, recv_x, recv_scales, capacity_rows,
                                        "ep_dispatch")
    lib = load_library()
    with _on(h):
        if x.dtype == torch.bfloat16:
            _check(lib.ep_dispatch(h.handle, _ptr(x), H, f, _ptr(recv_x), _ptr(recv_scales),
                                   recv_x.shape[0], _stream(h.device)), "ep_dispatch")
        else:
            _check(lib.ep_dispatch_ex(h.handle, _ptr(x), _DTYPES[x.dtype], H, f, _ptr(recv_x),
                                      _ptr(recv_scales), recv_x.shape[0], _stream(h.device)),
                   "ep_dispatch_ex")
    return recv_x, recv_scales


def ep_layout_dispatch(h: EPHandle, topk_idx: torch.Tensor, x: torch.Tensor,
                       fmt: Optional[str] = None,
                       recv_x: Optional[torch.Tensor] = None,
                       recv_scales: Optional[torch.Tensor] = None,
                       capacity_rows: Optional[int] = None):
    """ep_layout then ep_dispatch, in one launch for decode-sized batches (x bf16,
    or fp16 copied as rows)."""
    if topk_idx.dtype != torch.int64 or topk_idx.dim() != 2 or topk_idx.shape[1] != h.k:
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout_dispatch: topk_idx must be int64 [T, %d]" % h.k)
    if not topk_idx.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout_dispatch: topk_idx must be contiguous")
    T = topk_idx.shape[0]
    if x.dtype not in _DTYPES or x.dim() != 2 or x.shape[0] != T or not x.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout_dispatch: x must be contiguous [T, H]")
    H = x.shape[1]
    f = _fmt_code(fmt, x.dtype)
    if x.dtype == torch.float16 and f != EP_FMT_FP16:
        raise EPError(EP_ERR_INVALID_ARG, "ep_layout_dispatch: fp16 x takes the fp16 copy only; "
                      "for FP8 of fp16 rows call ep_layout then ep_dispatch")
    _same_device(h, "ep_layout_dispatch", topk_idx, x)
    recv_x, recv_scales = _recv_buffers(h, T, H, f, x.device, recv_x, recv_scales, capacity_rows,
                                        "ep_layout_dispatch")
    with _on(h):
        _check(load_library().ep_layout_dispatch(
            h.handle, _ptr(topk_idx), T, _ptr(x), H, f, _ptr(recv_x), _ptr(recv_scales),
            recv_x.shape[0], _stream(h.device)), "ep_layout_dispatch")
    h.T = T
    return recv_x, recv_scales


def ep_combine(h: EPHandle, y: torch.Tensor, topk_weights: torch.Tensor,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Weighted gather-reduce of y [rows, H] (receive layout; bf16 or fp16) into
    out [T, H] of the same type."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_combine")
    if y.dtype not in _DTYPES or y.dim() != 2 or not y.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine: y must be contiguous bf16/fp16 [rows, H]")
    if (topk_weights.dtype != torch.float32 or tuple(topk_weights.shape) != (h.T, h.k)
            or not topk_weights.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine: topk_weights must be f32 [T, k]")
    H = y.shape[1]
    if out is None:
        out = torch.empty((h.T, H), dtype=y.dtype, device=y.device)
    if out.dtype != y.dtype or tuple(out.shape) != (h.T, H) or not out.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine: out must be contiguous [T, H], y's type")
    _same_device(h, "ep_combine", y, topk_weights, out)
    lib = load_library()
    with _on(h):
        if y.dtype == torch.bfloat16:
            _check(lib.ep_combine(h.handle, _ptr(y), y.shape[0], _ptr(topk_weights), H,
                                  _ptr(out), _stream(h.device)), "ep_combine")
        else:
            _check(lib.ep_combine_ex(h.handle, _ptr(y), y.shape[0], _ptr(topk_weights), H,
                                     _DTYPES[y.dtype], _ptr(out), _stream(h.device)),
                   "ep_combine_ex")
    return out


def ep_dispatch_range(h: EPHandle, t_begin: int, x_rows: torch.Tensor, fmt: str,
                      recv_x: torch.Tensor, recv_scales: Optional[torch.Tensor] = None) -> None:
    """Dispatch tokens [t_begin, t_begin + len(x_rows)) of the last layout into
    the given receive buffers (x_rows: contiguous bf16 [n, H], the rows of
    those tokens)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch_range")
    if x_rows.dtype not in _DTYPES or x_rows.dim() != 2 or not x_rows.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_range: x_rows must be contiguous [n, H]")
    f = _fmt_code(fmt, x_rows.dtype)
    if _is_copy(f) and f != _COPY_FMT[x_rows.dtype] or not _is_copy(f) and \
            x_rows.dtype != torch.bfloat16:
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_range: x_rows type and format disagree")
    n, H = x_rows.shape
    _check_recv("ep_dispatch_range", H, f, recv_x, recv_scales)
    _same_device(h, "ep_dispatch_range", x_rows, recv_x,
                 recv_scales if not _is_copy(f) else None)
    with _on(h):
        _check(load_library().ep_dispatch_range(
            h.handle, t_begin, n, _ptr(x_rows), H, f, _ptr(recv_x),
            _ptr(recv_scales) if not _is_copy(f) else ctypes.c_void_p(0), recv_x.shape[0],
            _stream(h.device)),
            "ep_dispatch_range")


def ep_combine_range(h: EPHandle, t_begin: int, y: torch.Tensor, topk_weights_rows: torch.Tensor,
                     out_rows: torch.Tensor) -> None:
    """Combine tokens [t_begin, t_begin + len(out_rows)) of the last layout
    (topk_weights_rows: f32 [n, k]; out_rows: bf16 [n, H], contiguous)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_combine_range")
    if out_rows.dim() != 2 or y.dim() != 2:
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_range: y and out_rows must be 2-D")
    n, H = out_rows.shape
    if (y.dtype != torch.bfloat16 or y.shape[1] != H or not y.is_contiguous()
            or out_rows.dtype != torch.bfloat16 or not out_rows.is_contiguous()
            or topk_weights_rows.dtype != torch.float32
            or tuple(topk_weights_rows.shape) != (n, h.k) or not topk_weights_rows.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_range: bad tensor")
    _same_device(h, "ep_combine_range", y, topk_weights_rows, out_rows)
    with _on(h):
        _check(load_library().ep_combine_range(
            h.handle, t_begin, n, _ptr(y), y.shape[0], _ptr(topk_weights_rows), H, _ptr(out_rows),
            _stream(h.device)), "ep_combine_range")


def _table(values, ctype):
    return (ctype * len(values))(*values)


def ep_dispatch_ranks(h: EPHandle, t_begin: int, x_rows: torch.Tensor, fmt: Optional[str],
                      recv_x: list, recv_scales: Optional[list] = None) -> None:
    """Expert-parallel dispatch of tokens [t_begin, t_begin + len(x_rows)) of
    the last (global) layout into one receive buffer per rank: rank p gets
    rows [rank_off[p], rank_off[p+1]) of the layout, renumbered from 0, in
    recv_x[p] (and its FP8 scales in recv_scales[p]).  On several GPUs the
    entries are peer views of the ranks' buffers."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch_ranks")
    if x_rows.dtype not in _DTYPES or x_rows.dim() != 2 or not x_rows.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_ranks: x_rows must be contiguous [n, H]")
    f = _fmt_code(fmt, x_rows.dtype)
    if (_is_copy(f) and f != _COPY_FMT[x_rows.dtype]) or \
            (not _is_copy(f) and (f != EP_FMT_FP8_E4M3_1X128 or x_rows.dtype != torch.bfloat16)):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_ranks: row copy or bf16 -> fp8 (row-major)")
    n, H = x_rows.shape
    if len(recv_x) != h.R or (not _is_copy(f) and (recv_scales is None or len(recv_scales) != h.R)):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_ranks: one buffer per rank")
    _same_device(h, "ep_dispatch_ranks", x_rows)
    _rank_list(h, "ep_dispatch_ranks", recv_x if _is_copy(f) else list(recv_x) + list(recv_scales))
    for p, r in enumerate(recv_x):
        _check_recv("ep_dispatch_ranks", H, f, r, None if _is_copy(f) else recv_scales[p])
    ptrs = _table([_ptr(r) for r in recv_x], ctypes.c_void_p)
    rows = _table([r.shape[0] for r in recv_x], ctypes.c_int64)
    sptrs = _table([_ptr(sc) for sc in recv_scales], ctypes.c_void_p) if not _is_copy(f) else None
    with _on(h):
        _check(load_library().ep_dispatch_ranks(
            h.handle, t_begin, n, _ptr(x_rows), H, f, ptrs, sptrs, rows, _stream(h.device)),
            "ep_dispatch_ranks")


def ep_combine_ranks(h: EPHandle, t_begin: int, y: list, topk_weights_rows: torch.Tensor,
                     out_rows: torch.Tensor) -> None:
    """Expert-parallel combine of tokens [t_begin, t_begin + len(out_rows)) of
    the last (global) layout, reading each slot's expert output from its
    rank's buffer y[p] (bf16 or fp16, the type of out_rows)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_combine_ranks")
    if out_rows.dim() != 2:
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_ranks: out_rows must be 2-D")
    _rank_list(h, "ep_combine_ranks", y)
    n, H = out_rows.shape
    if (out_rows.dtype not in _DTYPES or not out_rows.is_contiguous() or len(y) != h.R
            or topk_weights_rows.dtype != torch.float32
            or tuple(topk_weights_rows.shape) != (n, h.k) or not topk_weights_rows.is_contiguous()
            or any(t.dtype != out_rows.dtype or t.shape[1] != H or not t.is_contiguous() for t in y)):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_ranks: bad tensor")
    _same_device(h, "ep_combine_ranks", topk_weights_rows, out_rows)
    ptrs = _table([_ptr(t) for t in y], ctypes.c_void_p)
    rows = _table([t.shape[0] for t in y], ctypes.c_int64)
    with _on(h):
        _check(load_library().ep_combine_ranks(
            h.handle, t_begin, n, ptrs, rows, _ptr(topk_weights_rows), H, _DTYPES[out_rows.dtype],
            _ptr(out_rows), _stream(h.device)), "ep_combine_ranks")


def ep_dispatch_ranks_backward(h: EPHandle, t_begin: int, grad_recv: list,
                               grad_x_rows: torch.Tensor) -> None:
    """Backward of ep_dispatch_ranks for tokens [t_begin, t_begin + len(grad_x_rows)):
    the fp32 sum, in slot order, of each token's slot rows of the ranks' gradient
    buffers grad_recv[p], rounded to grad_x_rows' type (bf16 or fp16)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch_ranks_backward")
    if grad_x_rows.dim() != 2:
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_ranks_backward: grad_x_rows must be 2-D")
    _rank_list(h, "ep_dispatch_ranks_backward", grad_recv)
    _same_device(h, "ep_dispatch_ranks_backward", grad_x_rows)
    n, H = grad_x_rows.shape
    if (grad_x_rows.dtype not in _DTYPES or not grad_x_rows.is_contiguous() or
            len(grad_recv) != h.R or any(t.dtype != grad_x_rows.dtype or t.shape[1] != H or
                                         not t.is_contiguous() for t in grad_recv)):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_ranks_backward: bad tensor")
    ptrs = _table([_ptr(t) for t in grad_recv], ctypes.c_void_p)
    rows = _table([t.shape[0] for t in grad_recv], ctypes.c_int64)
    with _on(h):
        _check(load_library().ep_dispatch_ranks_backward(
            h.handle, t_begin, n, ptrs, rows, H, _DTYPES[grad_x_rows.dtype], _ptr(grad_x_rows),
            _stream(h.device)), "ep_dispatch_ranks_backward")


def ep_combine_ranks_backward(h: EPHandle, t_begin: int, grad_out_rows: torch.Tensor, y: list,
                              topk_weights_rows: torch.Tensor, grad_y: list) -> torch.Tensor:
    """Backward of ep_combine_ranks for tokens [t_begin, t_begin + len(grad_out_rows)):
    writes each used slot's row of grad_y[p] (w * grad_out, rounded) and returns
    grad_weights f32 [n, k] (dot products of grad_out with the slots' y rows)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_combine_ranks_backward")
    if grad_out_rows.dim() != 2:
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_ranks_backward: grad_out_rows must be 2-D")
    _rank_list(h, "ep_combine_ranks_backward", list(y) + list(grad_y))
    _same_device(h, "ep_combine_ranks_backward", grad_out_rows, topk_weights_rows)
    n, H = grad_out_rows.shape
    dt = grad_out_rows.dtype
    if (dt not in _DTYPES or not grad_out_rows.is_contiguous() or len(y) != h.R
            or len(grad_y) != h.R or topk_weights_rows.dtype != torch.float32
            or tuple(topk_weights_rows.shape) != (n, h.k) or not topk_weights_rows.is_contiguous()
            or any(t.dtype != dt or t.shape[1] != H or not t.is_contiguous()
                   for t in list(y) + list(grad_y))):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_ranks_backward: bad tensor")
    grad_w = torch.empty((n, h.k), dtype=torch.float32, device=grad_out_rows.device)
    yp = _table([_ptr(t) for t in y], ctypes.c_void_p)
    yr = _table([t.shape[0] for t in y], ctypes.c_int64)
    gp = _table([_ptr(t) for t in grad_y], ctypes.c_void_p)
    gr = _table([t.shape[0] for t in grad_y], ctypes.c_int64)
    with _on(h):
        _check(load_library().ep_combine_ranks_backward(
            h.handle, t_begin, n, _ptr(grad_out_rows), yp, yr, _ptr(topk_weights_rows), H,
            _DTYPES[dt], gp, gr, _ptr(grad_w), _stream(h.device)), "ep_combine_ranks_backward")
    return grad_w


def ep_allgather_topk(topk_idx: torch.Tensor, group=None):
    """All ranks' top-k indices in rank order (the global token order of the
    expert-parallel layout) and this rank's first global token: an all-gather
    of the token counts, then of the index rows (padded to the largest
    count).  Works with any torch.distributed backend the tensors suit."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    n = torch.tensor([topk_idx.shape[0]], dtype=torch.int64, device=topk_idx.device)
    counts = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(counts, n, group=group)
    counts = [int(c.item()) for c in counts]
    most = max(counts) if counts else 0
    pad = torch.full((most, topk_idx.shape[1]), -1, dtype=topk_idx.dtype, device=topk_idx.device)
    pad[:topk_idx.shape[0]] = topk_idx
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    glob = torch.cat([parts[r][:counts[r]] for r in range(world)], dim=0).contiguous()
    return glob, sum(counts[:me])


EP_IPC_HANDLE_BYTES = 64


def ep_ipc_export(t: torch.Tensor):
    """(handle bytes, offset) of a CUDA tensor's memory, for another process's
    ep_ipc_open (the tensor must come from a cudaMalloc allocation, as the
    default caching allocator's are)."""
    if t.device.type != "cuda" or t.numel() == 0:
        raise EPError(EP_ERR_INVALID_ARG, "ep_ipc_export: a non-empty CUDA tensor")
    buf = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    with torch.cuda.device(t.device):
        _check(load_library().ep_ipc_export(t.data_ptr(), buf, ctypes.byref(off)), "ep_ipc_export")
    return bytes(buf.raw), int(off.value)


def ep_ipc_open(handle: bytes, offset: int):
    """Open another process's exported handle on the current device; returns
    (base, ptr) as integers: base for ep_ipc_close, ptr = base + offset."""
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise EPError(EP_ERR_INVALID_ARG, "ep_ipc_open: handle of %d bytes" % EP_IPC_HANDLE_BYTES)
    base, ptr = ctypes.c_void_p(), ctypes.c_void_p()
    _check(load_library().ep_ipc_open(handle, offset, ctypes.byref(base), ctypes.byref(ptr)),
           "ep_ipc_open")
    return int(base.value), int(ptr.value)


def ep_ipc_close(base: int) -> None:
    _check(load_library().ep_ipc_close(base), "ep_ipc_close")


_CAI_TYPE = {torch.bfloat16: ("<i2", torch.bfloat16), torch.float16: ("<f2", torch.float16),
             torch.float32: ("<f4", torch.float32), torch.int32: ("<i4", torch.int32),
             torch.int64: ("<i8", torch.int64), torch.uint8: ("|u1", torch.uint8),
             torch.float8_e4m3fn: ("|u1", torch.float8_e4m3fn)}


class _DeviceArray:
    """A raw device pointer seen by torch.as_tensor (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": tuple(shape),
                                         "typestr": typestr, "strides": None, "version": 3}


class IPCShare:
    """Every rank's buffers, opened in this process: tensors[r][i] is rank r's
    i-th shared tensor (this rank's own tensors as given, the others' as views
    of their IPC mappings).  close() unmaps the peers' allocations; the views
    must not be used after it."""

    def __init__(self, tensors, bases):
        self.tensors = tensors
        self._bases = bases

    def close(self) -> None:
        for base in self._bases:
            ep_ipc_close(base)
        self._bases = []


def ep_ipc_share(local: list, group=None) -> IPCShare:
    """Share this rank's CUDA tensors with the other ranks of a process group
    and open theirs: an all-gather of (handle, offset, shape, dtype) over the
    group, then ep_ipc_open of each peer allocation once (tensors that share
    an allocation share its mapping).  Every rank passes the same number of
    tensors.  The writes to and reads from the views need the caller's own
    ordering across ranks (stream synchronise, then a barrier)."""
    import torch.distributed as dist

    for t in local:
        if t.dtype not in _CAI_TYPE or not t.is_contiguous() or t.device.type != "cuda":
            raise EPError(EP_ERR_INVALID_ARG, "ep_ipc_share: contiguous CUDA tensors")
    mine = [ep_ipc_export(t) + (tuple(t.shape), str(t.dtype)) for t in local]
    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    every = [None] * world
    dist.all_gather_object(every, mine, group=group)
    names = {str(dt): dt for dt in _CAI_TYPE}
    opened = {}
    tensors = []
    for r in range(world):
        if r == me:
            tensors.append(list(local))
            continue
        views = []
        for handle, offset, shape, dname in every[r]:
            if handle not in opened:
                opened[handle] = ep_ipc_open(handle, 0)[0]
            typestr, dt = _CAI_TYPE[names[dname]]
            arr = _DeviceArray(opened[handle] + offset, shape, typestr)
            views.append(torch.as_tensor(arr).view(dt))  # the device of the mapping: no copy
        tensors.append(views)
    return IPCShare(tensors, list(opened.values()))


def ep_dispatch_backward(h: EPHandle, grad_recv: torch.Tensor,
                         grad_x: Optional[torch.Tensor] = None) -> torch.Tensor:
    """grad_x[t] = sum over the used slots of grad_recv[dst_row[t, j]] ([T, H], the type
    of grad_recv: bf16 or fp16)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch_backward")
    if grad_recv.dtype not in _DTYPES or grad_recv.dim() != 2 or not grad_recv.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG,
                      "ep_dispatch_backward: grad_recv must be bf16/fp16 [rows, H]")
    H = grad_recv.shape[1]
    if grad_x is None:
        grad_x = torch.empty((h.T, H), dtype=grad_recv.dtype, device=grad_recv.device)
    if grad_x.dtype != grad_recv.dtype or tuple(grad_x.shape) != (h.T, H) or \
            not grad_x.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_backward: grad_x must be [T, H]")
    _same_device(h, "ep_dispatch_backward", grad_recv, grad_x)
    with _on(h):
        _check(load_library().ep_dispatch_backward_ex(
            h.handle, _ptr(grad_recv), grad_recv.shape[0], H, _DTYPES[grad_recv.dtype],
            _ptr(grad_x), _stream(h.device)), "ep_dispatch_backward")
    return grad_x


def ep_combine_backward(h: EPHandle, grad_out: torch.Tensor, y: torch.Tensor,
                        topk_weights: torch.Tensor, grad_y: Optional[torch.Tensor] = None):
    """(grad_y in the receive layout, grad_weights f32 [T, k]) for ep_combine; the rows
    are bf16 or fp16 (grad_out, y and grad_y of one type)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_combine_backward")
    for name, t in (("grad_out", grad_out), ("y", y)):
        if t.dtype not in _DTYPES or t.dtype != y.dtype or t.dim() != 2 or not t.is_contiguous():
            raise EPError(EP_ERR_INVALID_ARG,
                          "ep_combine_backward: %s must be 2-D bf16/fp16 of y's type" % name)
    if (topk_weights.dtype != torch.float32 or tuple(topk_weights.shape) != (h.T, h.k)
            or not topk_weights.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_backward: topk_weights must be f32 [T, k]")
    H = y.shape[1]
    if tuple(grad_out.shape) != (h.T, H):
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_backward: grad_out must be [T, H]")
    if grad_y is None:
        grad_y = torch.empty_like(y)
    if grad_y.dtype != y.dtype or grad_y.dim() != 2 or grad_y.shape[1] != H or \
            not grad_y.is_contiguous():
        raise EPError(EP_ERR_INVALID_ARG, "ep_combine_backward: grad_y must be [*, H], y's type")
    _same_device(h, "ep_combine_backward", grad_out, y, topk_weights, grad_y)
    grad_w = torch.empty((h.T, h.k), dtype=torch.float32, device=y.device)
    with _on(h):
        _check(load_library().ep_combine_backward_ex(
            h.handle, _ptr(grad_out), _ptr(y), y.shape[0], _ptr(topk_weights), H,
            _DTYPES[y.dtype], _ptr(grad_y), grad_y.shape[0], _ptr(grad_w), _stream(h.device)),
            "ep_combine_backward")
    return grad_y, grad_w


def ep_dispatch_weights(h: EPHandle, topk_weights: torch.Tensor,
                        recv_weights: Optional[torch.Tensor] = None,
                        capacity_rows: Optional[int] = None) -> torch.Tensor:
    """recv_weights[dst_row[t, j]] = topk_weights[t, j] (f32, receive layout)."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_dispatch_weights")
    if (topk_weights.dtype != torch.float32 or tuple(topk_weights.shape) != (h.T, h.k)
            or not topk_weights.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_weights: topk_weights must be f32 [T, k]")
    if recv_weights is None:
        cap = capacity_rows if capacity_rows is not None else \
            ep_recv_rows_upper_bound(h.T, h.k, h.E, h.block_m)
        recv_weights = torch.zeros(cap, dtype=torch.float32, device=topk_weights.device)
    if (recv_weights.dtype != torch.float32 or recv_weights.dim() != 1
            or not recv_weights.is_contiguous()):
        raise EPError(EP_ERR_INVALID_ARG, "ep_dispatch_weights: recv_weights must be f32 [cap]")
    _same_device(h, "ep_dispatch_weights", topk_weights, recv_weights)
    with _on(h):
        _check(load_library().ep_dispatch_weights(h.handle, _ptr(topk_weights), _ptr(recv_weights),
                                                  recv_weights.shape[0], _stream(h.device)),
               "ep_dispatch_weights")
    return recv_weights


def ep_zero_pad_rows(h: EPHandle, rows: torch.Tensor) -> torch.Tensor:
    """Zero the pad rows (receive layout) of a contiguous [capacity, ...] tensor in place."""
    if h.T is None:
        raise EPError(EP_ERR_STATE, "ep_zero_pad_rows")
    if not rows.is_contiguous() or rows.dim() < 1:
        raise EPError(EP_ERR_INVALID_ARG, "ep_zero_pad_rows: rows must be contiguous")
    _same_device(h, "ep_zero_pad_rows", rows)
    row_bytes = rows[0].numel() * rows.element_size() if rows.shape[0] else 1
    with _on(h):
        _check(load_library().ep_zero_pad_rows(h.handle, _ptr(rows), row_bytes, rows.shape[0],
                                               _stream(h.device)), "ep_zero_pad_rows")
    return rows


def ep_handle_check(h: EPHandle, raise_on_error: bool = True) -> int:
    """Synchronise, read and clear the sticky device error word."""
    with _on(h):
        st = load_library().ep_handle_check(h.handle, _stream(h.device))
    if raise_on_error:
        _check(st, "ep_handle_check")
    return st
