"""The C-ABI library builds, loads and exports every symbol ep.h declares;
host-side argument checks return their status codes without touching a GPU.

No call here launches work: every ep_* call below is rejected (or answered)
by host code before any CUDA runtime call, so these run on a CPU-only box.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep.h")


@pytest.fixture(scope="module")
def lib():
    from combine_ep_layout_08_b200 import _build, load_library

    _build.build()
    return load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("ep_layout", "ep_dispatch", "ep_combine", "ep_handle_create",
                 "ep_workspace_bytes", "ep_handle_check", "ep_strerror"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from combine_ep_layout_08_b200 import library_path

    out = subprocess.run(["nm", "-D", "--defined-only", library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_sm100a_only():
    from combine_ep_layout_08_b200 import library_path

    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", library_path()],
                         capture_output=True, text=True).stdout
    assert "sm_100a" in out
    for other in ("sm_80", "sm_90", "sm_89"):
        assert other not in out


def test_workspace_bytes_and_bounds(lib, oracle):
    from combine_ep_layout_08_b200 import ep_recv_rows_upper_bound, ep_workspace_bytes

    assert ep_workspace_bytes(8192, 8, 256, 8) > 0
    assert ep_workspace_bytes(0, 8, 256, 8) > 0
    for bad in [(-1, 8, 256, 8, 128), (8, 0, 256, 8, 128), (8, 33, 256, 8, 128),
                (8, 8, 0, 8, 128), (8, 8, 256, 7, 128), (8, 8, 256, 512, 128),
                (8, 8, 256, 8, 0), (8, 8, 8193, 1, 128), (1 << 30, 8, 256, 8, 128)]:
        assert ep_workspace_bytes(*bad) == 0, bad
    rng = np.random.default_rng(0)
    for _ in range(50):
        T, k, E, B = (int(rng.integers(0, 5000)), int(rng.integers(1, 9)),
                      int(rng.choice([8, 64, 256])), int(rng.choice([1, 64, 128])))
        assert ep_recv_rows_upper_bound(T, k, E, B) == oracle.recv_rows_bound(T, k, E, B)
    assert ep_recv_rows_upper_bound(-1, 8, 256, 128) == -1


def _create(lib, ws, nbytes, *shape):
    h = ctypes.c_void_p()
    st = lib.ep_handle_create(ctypes.c_void_p(ws), nbytes, *shape, ctypes.byref(h))
    return st, h


def test_handle_create_validation(lib):
    from combine_ep_layout_08_b200 import (EP_ERR_ALIGNMENT, EP_ERR_INVALID_ARG, EP_OK,
                                           EP_ERR_WORKSPACE_TOO_SMALL, ep_workspace_bytes)

    need = ep_workspace_bytes(1024, 8, 256, 8)
    fake = 0x7f0000000000  # never dereferenced by host code
    st, h = _create(lib, fake, need, 1024, 8, 256, 8, 128)
    assert st == EP_OK and h.value
    lib.ep_handle_destroy(h)
    st, h = _create(lib, fake + 16, need, 1024, 8, 256, 8, 128)
    assert st == EP_ERR_ALIGNMENT and not h.value
    st, h = _create(lib, fake, need - 1, 1024, 8, 256, 8, 128)
    assert st == EP_ERR_WORKSPACE_TOO_SMALL
    st, h = _create(lib, 0, need, 1024, 8, 256, 8, 128)
    assert st == EP_ERR_INVALID_ARG
    st, h = _create(lib, fake, need, 1024, 8, 256, 3, 128)
    assert st == EP_ERR_INVALID_ARG
    assert lib.ep_handle_create(ctypes.c_void_p(fake), need, 1024, 8, 256, 8, 128, None) == \
        EP_ERR_INVALID_ARG


def test_calls_rejected_before_any_launch(lib):
    from combine_ep_layout_08_b200 import (EP_ERR_ALIGNMENT, EP_ERR_INVALID_ARG, EP_ERR_STATE,
                                           ep_workspace_bytes)

    need = ep_workspace_bytes(64, 2, 16, 4)
    st, h = _create(lib, 0x7f0000000000, need, 64, 2, 16, 4, 128)
    assert st == 0
    P = ctypes.c_void_p
    # no layout yet
    assert lib.ep_dispatch(h, P(0x1000), 256, 0, P(0x2000), None, 10, None) == EP_ERR_STATE
    assert lib.ep_combine(h, P(0x1000), 10, P(0x2000), 256, P(0x3000), None) == EP_ERR_STATE
    assert lib.ep_handle_read_counts(h, None, None, None, None, None) == EP_ERR_STATE
    # bad layout arguments
    assert lib.ep_layout(h, P(0x1000), 65, None) == EP_ERR_INVALID_ARG   # T > max_tokens
    assert lib.ep_layout(h, P(0x1000), -1, None) == EP_ERR_INVALID_ARG
    assert lib.ep_layout(h, None, 5, None) == EP_ERR_INVALID_ARG
    assert lib.ep_layout(h, P(0x1004), 5, None) == EP_ERR_ALIGNMENT
    assert lib.ep_layout(None, P(0x1000), 5, None) == EP_ERR_INVALID_ARG
    # ep_handle_check before anything ran needs no device
    assert lib.ep_handle_check(h, None) == 0
    lib.ep_handle_destroy(h)


def test_views_point_into_the_workspace(lib):
    from combine_ep_layout_08_b200 import VIEWS, ep_workspace_bytes

    need = ep_workspace_bytes(100, 8, 256, 8)
    base = 0x7f0000000000
    st, h = _create(lib, base, need, 100, 8, 256, 8, 128)
    assert st == 0
    spans = []
    for name, (code, _) in VIEWS.items():
        n = ctypes.c_int64()
        p = lib.ep_handle_view(h, code, ctypes.byref(n))
        assert p and base <= p < base + need, name
        assert p % 256 == 0, name
        spans.append((p, name))
    assert len(set(p for p, _ in spans)) == len(spans)
    assert lib.ep_handle_view(h, 99, None) is None
    n = ctypes.c_int64()
    assert lib.ep_handle_view(h, 9, ctypes.byref(n)) and n.value == 3
    lib.ep_handle_destroy(h)


def test_strerror(lib):
    from combine_ep_layout_08_b200 import ep_strerror

    assert ep_strerror(0) == "EP_OK"
    assert "BAD_INDEX" in ep_strerror(5)
    assert ep_strerror(1234) == "unknown ep_status_t"


def test_newer_entry_points_rejected_before_any_launch(lib):
    """The FP16, expert-parallel, backward and GEMM-layout calls check their
    arguments (and that a layout exists) on the host, before any launch."""
    from combine_ep_layout_08_b200 import (EP_ERR_INVALID_ARG, EP_ERR_STATE,
                                           ep_workspace_bytes)

    need = ep_workspace_bytes(64, 2, 16, 4)
    st, h = _create(lib, 0x7f0000000000, need, 64, 2, 16, 4, 128)
    assert st == 0
    P = ctypes.c_void_p
    tab = (ctypes.c_void_p * 4)(0x1000, 0x2000, 0x3000, 0x4000)
    rows = (ctypes.c_int64 * 4)(8, 8, 8, 8)
    # no layout yet: every data call reports the state error
    assert lib.ep_dispatch_ex(h, P(0x1000), 1, 256, 3, P(0x2000), None, 8, None) == EP_ERR_STATE
    assert lib.ep_combine_ex(h, P(0x1000), 8, P(0x2000), 256, 1, P(0x3000), None) == EP_ERR_STATE
    assert lib.ep_dispatch_ranks(h, 0, 0, P(0x1000), 256, 0, tab, None, rows, None) == EP_ERR_STATE
    assert lib.ep_combine_ranks(h, 0, 0, tab, rows, P(0x2000), 256, 0, P(0x3000), None) \
        == EP_ERR_STATE
    assert lib.ep_dispatch_backward(h, P(0x1000), 8, 256, P(0x2000), None) == EP_ERR_STATE
    # bad sizes and types are rejected before the state is looked at
    assert lib.ep_dispatch_ranks(h, 0, 0, P(0x1000), 200, 0, tab, None, rows, None) \
        == EP_ERR_INVALID_ARG                                   # H % 16 != 0
    assert lib.ep_combine_ranks(h, 0, 0, tab, rows, P(0x2000), 256, 7, P(0x3000), None) \
        == EP_ERR_INVALID_ARG                                   # unknown dtype
    assert lib.ep_combine_ex(h, P(0x1000), 8, P(0x2000), 250, 0, P(0x3000), None) \
        == EP_ERR_INVALID_ARG                                   # H % 8 != 0
    assert lib.ep_layout_dispatch(h, P(0x1000), 65, P(0x2000), 256, 0, P(0x3000), None, 8, None) \
        == EP_ERR_INVALID_ARG                                   # T > max_tokens
    lib.ep_handle_destroy(h)


def test_backward_ex_rejected_before_any_launch(lib):
    from combine_ep_layout_08_b200 import EP_ERR_INVALID_ARG, EP_ERR_STATE, ep_workspace_bytes

    need = ep_workspace_bytes(64, 2, 16, 4)
    st, h = _create(lib, 0x7f0000000000, need, 64, 2, 16, 4, 128)
    assert st == 0
    P = ctypes.c_void_p
    assert lib.ep_dispatch_backward_ex(h, P(0x1000), 8, 256, 1, P(0x2000), None) == EP_ERR_STATE
    assert lib.ep_dispatch_backward_ex(h, P(0x1000), 8, 256, 3, P(0x2000), None) \
        == EP_ERR_INVALID_ARG                                   # unknown dtype
    assert lib.ep_combine_backward_ex(h, P(0x1000), P(0x2000), 8, P(0x3000), 256, 1, P(0x4000),
                                      8, P(0x5000), None) == EP_ERR_STATE
    lib.ep_handle_destroy(h)


def test_ranks_backward_rejected_before_any_launch(lib):
    from combine_ep_layout_08_b200 import EP_ERR_INVALID_ARG, EP_ERR_STATE, ep_workspace_bytes

    need = ep_workspace_bytes(64, 2, 16, 4)
    st, h = _create(lib, 0x7f0000000000, need, 64, 2, 16, 4, 128)
    assert st == 0
    P = ctypes.c_void_p
    tab = (ctypes.c_void_p * 4)(0x1000, 0x2000, 0x3000, 0x4000)
    rows = (ctypes.c_int64 * 4)(8, 8, 8, 8)
    assert lib.ep_dispatch_ranks_backward(h, 0, 0, tab, rows, 256, 0, P(0x5000), None) \
        == EP_ERR_STATE
    assert lib.ep_combine_ranks_backward(h, 0, 0, P(0x5000), tab, rows, P(0x6000), 256, 0, tab,
                                         rows, P(0x7000), None) == EP_ERR_STATE
    assert lib.ep_combine_ranks_backward(h, 0, 0, P(0x5000), tab, rows, P(0x6000), 200, 0, tab,
                                         rows, P(0x7000), None) == EP_ERR_INVALID_ARG  # H % 16
    lib.ep_handle_destroy(h)


def test_binding_constants_match_the_header():
    """Status codes, formats, dtypes and limits the binding mirrors equal the
    header's (parsed from the text)."""
    import combine_ep_layout_08_b200 as ep

    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    enums = dict((m.group(1), int(m.group(2)))
                 for m in re.finditer(r"\b(EP_[A-Z0-9_]+)\s*=\s*(\d+)", src))
    defines = dict((m.group(1), int(m.group(2)))
                   for m in re.finditer(r"#define\s+(EP_[A-Z0-9_]+)\s+(\d+)", src))
    for name in dir(ep):
        if name.startswith(("EP_ERR_", "EP_FMT_", "EP_DTYPE_")) or name == "EP_OK":
            assert name in enums, name
            assert getattr(ep, name) == enums[name], name
    assert enums["EP_FMT_FP16"] == ep._FMTS["fp16"]
    assert defines["EP_MAX_RANK_TABLE"] >= 8
    assert set(ep._DTYPES.values()) == {enums["EP_DTYPE_BF16"], enums["EP_DTYPE_FP16"]}


def test_ipc_calls_reject_bad_arguments_without_a_gpu(lib):
    """The IPC mapping calls refuse null pointers before any CUDA call, and the
    binding's constant and checks mirror the header."""
    import torch

    import combine_ep_layout_08_b200 as ep
    from combine_ep_layout_08_b200 import EP_ERR_INVALID_ARG

    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    m = re.search(r"#define\s+EP_IPC_HANDLE_BYTES\s+(\d+)", src)
    assert m and int(m.group(1)) == ep.EP_IPC_HANDLE_BYTES == 64
    P = ctypes.c_void_p
    off = ctypes.c_uint64(0)
    buf = ctypes.create_string_buffer(64)
    assert lib.ep_ipc_export(None, buf, ctypes.byref(off)) == EP_ERR_INVALID_ARG
    assert lib.ep_ipc_export(P(0x7f0000000000), None, ctypes.byref(off)) == EP_ERR_INVALID_ARG
    base, ptr = P(), P()
    assert lib.ep_ipc_open(None, 0, ctypes.byref(base), ctypes.byref(ptr)) == EP_ERR_INVALID_ARG
    assert lib.ep_ipc_close(None) == EP_ERR_INVALID_ARG
    with pytest.raises(ep.EPError):
        ep.ep_ipc_export(torch.zeros(4))                  # host memory
    with pytest.raises(ep.EPError):
        ep.ep_ipc_open(b"too short", 0)
