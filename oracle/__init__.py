"""CPU oracle for the MoE dispatch-layout / dispatch / combine path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA product path never imports it, and it shares no code with
the CUDA library: the arithmetic lives in ``ep_oracle.c`` (plain C loops,
compiled with gcc, no fast-math, no FMA contraction) and this module only
marshals NumPy arrays through ctypes.

Array conventions (all C-contiguous NumPy arrays):
  * bf16 values travel as their raw bits in ``np.uint16``;
  * e4m3 values travel as raw bytes in ``np.uint8``;
  * indices are ``np.int64`` (top-k) and ``np.int32`` (rows).

Every function cites the passage of the pages it follows in ``ep_oracle.c``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "libep_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libep_oracle_omp.so")  # the same source with -fopenmp
_lock = threading.Lock()
_lib = None
_lib_omp = None
_active = None  # the OpenMP build while `threads` is in effect

OK = 0
ERR_ARG = 1
ERR_CAPACITY = 4
ERR_BAD_INDEX = 5


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile ``ep_oracle.c`` into ``libep_oracle.so`` (gcc, -O2, strict fp),
    or with ``openmp`` into ``libep_oracle_omp.so``: the same source with its
    token loops parallel over tokens, used only to time the oracle on all
    host cores (its outputs are byte-identical, which a test pins)."""
    out = _LIB_OMP if openmp else _LIB
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra",
               "-fopenmp" if openmp else "-Wno-unknown-pragmas", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _load():
    global _lib
    if _active is not None:
        return _active
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _load_omp():
    global _lib_omp
    with _lock:
        if _lib_omp is None:
            _lib_omp = _configure(ctypes.CDLL(build(openmp=True)))
    return _lib_omp


@contextlib.contextmanager
def threads(n: int = 0):
    """Inside the block, oracle calls run on the OpenMP build with n threads
    (0: the OpenMP default, all host cores); yields the thread count.  For
    timing the oracle on the host's cores; the results are the same bytes."""
    global _active
    lib = _load_omp()
    got = int(lib.oracle_set_threads(n))
    prev = _active
    _active = lib
    try:
        yield got
    finally:
        _active = prev


def _configure(lib):
    """Argument and result types of the oracle's C functions."""
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int
    lib.oracle_layout.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i64, P]
    lib.oracle_layout.restype = i32
    lib.oracle_recv_rows_bound.argtypes = [i64, i32, i32, i32]
    lib.oracle_recv_rows_bound.restype = i64
    lib.oracle_dispatch_bf16.argtypes = [P, i64, i32, i64, P, P, i64]
    lib.oracle_dispatch_bf16.restype = i32
    lib.oracle_dispatch_fp8.argtypes = [P, i64, i32, i64, i32, P, P, P, i64]
    lib.oracle_dispatch_fp8.restype = i32
    lib.oracle_quantize_token_fp8.argtypes = [P, i64, i32, P, P]
    lib.oracle_quantize_token_fp8.restype = None
    lib.oracle_expert_scale_bf16.argtypes = [P, P, P, i32, i64, P, P]
    lib.oracle_expert_scale_bf16.restype = None
    lib.oracle_expert_scale_fp8.argtypes = [P, P, P, P, i32, i64, P, P]
    lib.oracle_expert_scale_fp8.restype = None
    lib.oracle_combine.argtypes = [P, i64, P, P, i64, i32, i64, i32, P]
    lib.oracle_combine.restype = i32
    lib.oracle_dispatch_backward.argtypes = [P, i64, P, i64, i32, i64, i32, P]
    lib.oracle_dispatch_backward.restype = i32
    lib.oracle_combine_backward.argtypes = [P, P, i64, P, P, i64, i32, i64, i32, P, P]
    lib.oracle_combine_backward.restype = i32
    lib.oracle_dispatch_weights.argtypes = [P, P, i64, i32, P, i64]
    lib.oracle_dispatch_weights.restype = i32
    lib.oracle_zero_pad_rows.argtypes = [P, i64, P, i64]
    lib.oracle_zero_pad_rows.restype = None
    lib.oracle_dispatch_fp8_mn.argtypes = [P, i64, i32, i64, i32, P, P, P, i64, i64]
    lib.oracle_dispatch_fp8_mn.restype = i32
    for name in ("oracle_f32_to_e4m3_array", "oracle_e4m3_to_f32_array",
                 "oracle_f32_to_bf16_array", "oracle_fp16_to_f32_array",
                 "oracle_f32_to_fp16_array"):
        getattr(lib, name).argtypes = [P, P, i64]
        getattr(lib, name).restype = None
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_set_threads.restype = i32
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed with oracle status %d" % (what, code))
        self.code = code


# ---------------------------------------------------------------- formats

def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp32 -> e4m3 bytes, round-to-nearest-even, saturating to +-448."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_f32_to_e4m3_array(_p(v), _p(q), v.size)
    return q


def e4m3_decode(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    v = np.empty(q.shape, dtype=np.float32)
    _load().oracle_e4m3_to_f32_array(_p(q), _p(v), q.size)
    return v


def bf16_round(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round-to-nearest-even."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    b = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16_array(_p(v), _p(b), v.size)
    return b


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (a shift into the upper half of binary32)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def fp16_round(v: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE binary16 bits, round-to-nearest-even, overflow to infinity."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    h = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_f32_to_fp16_array(_p(v), _p(h), v.size)
    return h


def fp16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of binary16 bits to fp32."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    v = np.empty(h.shape, dtype=np.float32)
    _load().oracle_fp16_to_f32_array(_p(h), _p(v), h.size)
    return v


DTYPES = {"bf16": 0, "fp16": 1}


def to_f32(bits: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """16-bit values of the given type (bf16 or fp16) widened to fp32."""
    return fp16_to_f32(bits) if dtype == "fp16" else bf16_to_f32(bits)


# ---------------------------------------------------------------- layout

@dataclass
class Layout:
    num_tokens_per_expert: np.ndarray  # int32 [E]
    num_tokens_per_rank: np.ndarray    # int32 [R]
    num_rows_per_rank: np.ndarray      # int32 [R]
    expert_off: np.ndarray             # int32 [E+1]
    rank_off: np.ndarray               # int32 [R+1]
    is_token_in_rank: np.ndarray       # uint8 [T, R]
    dst_row: np.ndarray                # int32 [T, k]
    recv_src: np.ndarray               # int32 [P]
    total_rows: int                    # P


def recv_rows_bound(T: int, k: int, E: int, block_m: int = 128) -> int:
    return int(_load().oracle_recv_rows_bound(T, k, E, block_m))


def layout(topk_idx: np.ndarray, E: int, R: int, block_m: int = 128) -> Layout:
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    T, k = topk_idx.shape
    cap = recv_rows_bound(T, k, E, block_m)
    out = dict(
        num_tokens_per_expert=np.zeros(E, np.int32),
        num_tokens_per_rank=np.zeros(R, np.int32),
        num_rows_per_rank=np.zeros(R, np.int32),
        expert_off=np.zeros(E + 1, np.int32),
        rank_off=np.zeros(R + 1, np.int32),
        is_token_in_rank=np.zeros((T, R), np.uint8),
        dst_row=np.zeros((T, k), np.int32),
    )
    recv_src = np.zeros(max(cap, 1), np.int32)
    total = np.zeros(1, np.int32)
    rc = _load().oracle_layout(
        _p(topk_idx), T, k, E, R, block_m,
        _p(out["num_tokens_per_expert"]), _p(out["num_tokens_per_rank"]),
        _p(out["num_rows_per_rank"]), _p(out["expert_off"]), _p(out["rank_off"]),
        _p(out["is_token_in_rank"]), _p(out["dst_row"]), _p(recv_src), cap, _p(total))
    if rc != OK:
        raise OracleError(rc, "oracle_layout")
    P = int(total[0])
    return Layout(recv_src=recv_src[:P].copy(), total_rows=P, **out)


# ---------------------------------------------------------------- dispatch

def dispatch_bf16(x_bits: np.ndarray, dst_row: np.ndarray, recv_rows: int) -> np.ndarray:
    """recv_x[dst_row[t, j]] = x[t]; pad rows are left zero (unspecified)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    T, H = x_bits.shape
    k = dst_row.shape[1]
    recv = np.zeros((max(recv_rows, 1), H), np.uint16)
    rc = _load().oracle_dispatch_bf16(_p(x_bits), T, k, H, _p(dst_row), _p(recv), recv_rows)
    if rc != OK:
        raise OracleError(rc, "oracle_dispatch_bf16")
    return recv[:recv_rows]


def quantize_token_fp8(x_bits_row: np.ndarray, dtype: str = "bf16"):
    """One token row of bf16 or fp16 bits -> (e4m3 codes [H], scales [H/128])."""
    x_bits_row = np.ascontiguousarray(x_bits_row, dtype=np.uint16)
    H = x_bits_row.shape[0]
    q = np.empty(H, np.uint8)
    s = np.empty(max(H // 128, 1), np.float32)
    _load().oracle_quantize_token_fp8(_p(x_bits_row), H, DTYPES[dtype], _p(q), _p(s))
    return q, s[: H // 128]


def dispatch_fp8(x_bits: np.ndarray, dst_row: np.ndarray, recv_rows: int, dtype: str = "bf16"):
    """FP8 e4m3 1x128 dispatch of bf16 or fp16 rows: returns (recv_q uint8 [P, H],
    recv_scales f32 [P, H/128])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    T, H = x_bits.shape
    k = dst_row.shape[1]
    q = np.zeros((max(recv_rows, 1), H), np.uint8)
    s = np.zeros((max(recv_rows, 1), H // 128), np.float32)
    rc = _load().oracle_dispatch_fp8(_p(x_bits), T, k, H, DTYPES[dtype], _p(dst_row), _p(q),
                                     _p(s), recv_rows)
    if rc != OK:
        raise OracleError(rc, "oracle_dispatch_fp8")
    return q[:recv_rows], s[:recv_rows]


# ---------------------------------------------------------------- stand-in expert

def expert_scale_bf16(recv_x: np.ndarray, lay: Layout, c: np.ndarray) -> np.ndarray:
    recv_x = np.ascontiguousarray(recv_x, dtype=np.uint16)
    P, H = recv_x.shape
    y = np.zeros((max(P, 1), H), np.uint16)
    c = np.ascontiguousarray(c, dtype=np.float32)
    E = lay.expert_off.shape[0] - 1
    _load().oracle_expert_scale_bf16(_p(recv_x), _p(np.ascontiguousarray(lay.recv_src)),
                                     _p(lay.expert_off), E, H, _p(c), _p(y))
    return y[:P]


def expert_scale_fp8(recv_q: np.ndarray, recv_scales: np.ndarray, lay: Layout,
                     c: np.ndarray) -> np.ndarray:
    recv_q = np.ascontiguousarray(recv_q, dtype=np.uint8)
    recv_scales = np.ascontiguousarray(recv_scales, dtype=np.float32)
    P, H = recv_q.shape
    y = np.zeros((max(P, 1), H), np.uint16)
    c = np.ascontiguousarray(c, dtype=np.float32)
    E = lay.expert_off.shape[0] - 1
    _load().oracle_expert_scale_fp8(_p(recv_q), _p(recv_scales),
                                    _p(np.ascontiguousarray(lay.recv_src)),
                                    _p(lay.expert_off), E, H, _p(c), _p(y))
    return y[:P]


# ---------------------------------------------------------------- combine

def combine(y_bits: np.ndarray, topk_weights: np.ndarray, dst_row: np.ndarray,
            dtype: str = "bf16") -> np.ndarray:
    """out[t] = rn(sum_j w[t, j] * y[dst_row[t, j]]), fp32 fma chain in slot order; y and
    out are bf16 or fp16 bits."""
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    P, H = y_bits.shape
    T, k = dst_row.shape
    out = np.zeros((T, H), np.uint16)
    if P == 0:
        y_bits = np.zeros((1, H), np.uint16)
    rc = _load().oracle_combine(_p(y_bits), P, _p(w), _p(dst_row), T, k, H, DTYPES[dtype],
                                _p(out))
    if rc != OK:
        raise OracleError(rc, "oracle_combine")
    return out


# ---------------------------------------------------------------- backward

def dispatch_backward(grad_recv_bits: np.ndarray, dst_row: np.ndarray,
                      dtype: str = "bf16") -> np.ndarray:
    """grad_x[t] = rn16(sum over used slots of grad_recv[dst_row[t, j]]), fp32 in slot
    order; bf16 or fp16 bits."""
    g = np.ascontiguousarray(grad_recv_bits, dtype=np.uint16)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    rows, H = g.shape
    T, k = dst_row.shape
    out = np.zeros((T, H), np.uint16)
    if rows == 0:
        g = np.zeros((1, H), np.uint16)
    rc = _load().oracle_dispatch_backward(_p(g), rows, _p(dst_row), T, k, H, DTYPES[dtype],
                                          _p(out))
    if rc != OK:
        raise OracleError(rc, "oracle_dispatch_backward")
    return out


def combine_backward(grad_out_bits: np.ndarray, y_bits: np.ndarray, topk_weights: np.ndarray,
                     dst_row: np.ndarray, dtype: str = "bf16"):
    """(grad_y bits [rows, H] with pad rows zero, grad_w f32 [T, k]); bf16 or fp16 rows."""
    g = np.ascontiguousarray(grad_out_bits, dtype=np.uint16)
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    rows, H = y.shape
    T, k = dst_row.shape
    gy = np.zeros((max(rows, 1), H), np.uint16)
    gw = np.zeros((T, k), np.float32)
    if rows == 0:
        y = np.zeros((1, H), np.uint16)
    rc = _load().oracle_combine_backward(_p(g), _p(y), rows, _p(w), _p(dst_row), T, k, H,
                                         DTYPES[dtype], _p(gy), _p(gw))
    if rc != OK:
        raise OracleError(rc, "oracle_combine_backward")
    return gy[:rows], gw


# ---------------------------------------------------------------- GEMM-ready layout

def dispatch_weights(topk_weights: np.ndarray, dst_row: np.ndarray, recv_rows: int,
                     fill: float = 0.0) -> np.ndarray:
    """recv_w[dst_row[t, j]] = w[t, j]; pad rows keep `fill`."""
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    T, k = dst_row.shape
    out = np.full(max(recv_rows, 1), fill, np.float32)
    rc = _load().oracle_dispatch_weights(_p(w), _p(dst_row), T, k, _p(out), recv_rows)
    if rc != OK:
        raise OracleError(rc, "oracle_dispatch_weights")
    return out[:recv_rows]


def zero_pad_rows(recv_src: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """A copy of `rows` (any dtype, [P, ...]) with every pad row zeroed."""
    recv_src = np.ascontiguousarray(recv_src, dtype=np.int32)
    out = np.ascontiguousarray(rows).copy()
    P = recv_src.shape[0]
    if P:
        _load().oracle_zero_pad_rows(_p(recv_src), P, _p(out.view(np.uint8)),
                                     out.nbytes // out.shape[0])
    return out


def dispatch_fp8_mn(x_bits: np.ndarray, dst_row: np.ndarray, recv_rows: int, ld: int,
                    dtype: str = "bf16"):
    """FP8 dispatch with MN-major scales: (recv_q [P, H], scales_mn [H/128, ld])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    T, H = x_bits.shape
    k = dst_row.shape[1]
    q = np.zeros((max(recv_rows, 1), H), np.uint8)
    s = np.zeros((H // 128, max(ld, 1)), np.float32)
    rc = _load().oracle_dispatch_fp8_mn(_p(x_bits), T, k, H, DTYPES[dtype], _p(dst_row), _p(q),
                                        _p(s), ld, recv_rows)
    if rc != OK:
        raise OracleError(rc, "oracle_dispatch_fp8_mn")
    return q[:recv_rows], s[:, :ld]


def pipeline(x_bits, topk_idx, topk_weights, E, R, fmt, c, block_m=128):
    """Whole path on the CPU: layout -> dispatch -> stand-in expert -> combine."""
    lay = layout(topk_idx, E, R, block_m)
    if fmt == "bf16":
        recv = dispatch_bf16(x_bits, lay.dst_row, lay.total_rows)
        scales = None
        y = expert_scale_bf16(recv, lay, c)
    else:
        recv, scales = dispatch_fp8(x_bits, lay.dst_row, lay.total_rows)
        y = expert_scale_fp8(recv, scales, lay, c)
    out = combine(y, topk_weights, lay.dst_row)
    return dict(layout=lay, recv=recv, scales=scales, y=y, out=out)
