"""A process whose first library launches are captured in a CUDA graph (the
one-time set-up of the launch paths -- occupancy queries, shared-memory
limits, the cooperative launch form -- then runs under capture): layout,
BF16 and FP8 dispatch and combine replayed from the graph match the oracle
bit for bit."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_first_launches_inside_a_graph_capture(oracle, tmp_path):
    path = str(tmp_path / "graph_first_call.npz")
    r = subprocess.run([sys.executable, os.path.join(HERE, "graph_first_call_child.py"), path],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    d = np.load(path)
    E, R, B = int(d["E"]), int(d["R"]), int(d["block_m"])
    lay = oracle.layout(d["idx"], E, R, B)
    assert np.array_equal(d["dst_row"], lay.dst_row)
    rows = lay.dst_row[lay.dst_row >= 0]
    exp = oracle.dispatch_bf16(d["x"], lay.dst_row, lay.total_rows)
    assert np.array_equal(d["recv"][rows], exp[rows])
    q, s = oracle.dispatch_fp8(d["x"], lay.dst_row, lay.total_rows)
    assert np.array_equal(d["recv8"][rows], q[rows])
    assert np.array_equal(d["scales"][rows].view(np.uint32), s[rows].view(np.uint32))
    assert np.array_equal(d["out"], oracle.combine(d["y"], d["wt"], lay.dst_row))
