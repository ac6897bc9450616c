"""ep.h is enough for a non-Python caller to drive the device path: a C99
program (tests/c_device_consumer.c) allocates its own device buffers, runs
ep_handle_create -> ep_layout -> ep_dispatch (BF16 and FP8) -> ep_combine ->
ep_handle_check on a non-default stream of its own, and writes the results
back; everything it produced is compared here with the oracle, bit-exact.
The inputs come from the seeded workload generators; the program never sees
Python or PyTorch."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from workloads import make_workload, make_x

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_device_consumer.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    from combine_ep_layout_08_b200 import _build

    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    libdir = os.path.dirname(_build.build())
    out = str(tmp_path_factory.mktemp("cdev") / "c_device_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, "-L", libdir, "-lep",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + libdir,
           "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, " ".join(cmd) + "\n" + r.stderr
    return out


def _run(exe, tmp_path, w, y):
    T, k = w.topk_idx.shape
    P = y.shape[0]
    fin, fout = str(tmp_path / "in.bin"), str(tmp_path / "out.bin")
    with open(fin, "wb") as f:
        f.write(np.array([T, k, w.E, w.R, w.H, P], np.int32).tobytes())
        f.write(np.ascontiguousarray(w.topk_idx, np.int64).tobytes())
        f.write(np.ascontiguousarray(w.x_bits, np.uint16).tobytes())
        f.write(np.ascontiguousarray(w.topk_weights, np.float32).tobytes())
        f.write(np.ascontiguousarray(y, np.uint16).tobytes())
    r = subprocess.run([exe, fin, fout], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    buf = open(fout, "rb").read()
    at = 0

    def take(dtype, n):
        nonlocal at
        a = np.frombuffer(buf, dtype=dtype, count=n, offset=at)
        at += a.nbytes
        return a

    res = {"status": take(np.int32, 6)}
    total = int(take(np.int32, 1)[0])
    res["total"] = total
    res["expert_off"] = take(np.int32, w.E + 1)
    res["dst_row"] = take(np.int32, T * k).reshape(T, k)
    res["recv_src"] = take(np.int32, total)
    res["recv_bf16"] = take(np.uint16, total * w.H).reshape(total, w.H)
    res["recv_q"] = take(np.uint8, total * w.H).reshape(total, w.H)
    res["recv_scales"] = take(np.float32, total * (w.H // 128)).reshape(total, w.H // 128)
    res["out"] = take(np.uint16, T * w.H).reshape(T, w.H)
    assert at == len(buf)
    return res


@pytest.mark.parametrize("name,T,H", [
    ("tiny", 128, 256),      # one-CTA layout
    ("dsv3", 520, 1024),     # 4160 entries, past the one-CTA limit: the single-launch tile layout
    ("8k", 2048, 7168),      # the metric's row width
])
def test_c_program_drives_the_device_path(oracle, exe, tmp_path, name, T, H):
    w = make_workload(name, 0, T=T, H=H)
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    P = lay.total_rows
    y = make_x(P, w.H, np.random.default_rng(41))    # expert outputs in the receive layout
    res = _run(exe, tmp_path, w, y)
    assert res["status"].tolist() == [0] * 6
    assert res["total"] == P
    assert np.array_equal(res["expert_off"], lay.expert_off)
    assert np.array_equal(res["dst_row"], lay.dst_row)
    assert np.array_equal(res["recv_src"], lay.recv_src)
    rows = lay.dst_row[lay.dst_row >= 0]
    ref_bf16 = oracle.dispatch_bf16(w.x_bits, lay.dst_row, P)
    assert np.array_equal(res["recv_bf16"][rows], ref_bf16[rows])
    ref_q, ref_s = oracle.dispatch_fp8(w.x_bits, lay.dst_row, P)
    assert np.array_equal(res["recv_q"][rows], ref_q[rows])
    assert np.array_equal(res["recv_scales"][rows].view(np.uint32), ref_s[rows].view(np.uint32))
    assert np.array_equal(res["out"], oracle.combine(y, w.topk_weights, lay.dst_row))
