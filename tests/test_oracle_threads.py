"""The oracle's OpenMP build (the same C source compiled with -fopenmp, used
only to time the oracle on all host cores) gives byte-identical results to
the single-threaded build that the parity tests use: every token is computed
by one thread with the same sequence of operations, and the layout stays
serial.  Checked on every function whose token loop runs in parallel, with
several thread counts, unused slots and both 16-bit input types."""
import numpy as np
import pytest

from workloads import make_workload, make_x, make_x_fp16, random_topk


def _all_outputs(oracle, w, dtype):
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    x = w.x_bits if dtype == "bf16" else make_x_fp16(w.T, w.H, np.random.default_rng(5))
    out = {"dst_row": lay.dst_row}
    if dtype == "bf16":
        out["recv_bf16"] = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)
    q, s = oracle.dispatch_fp8(x, lay.dst_row, lay.total_rows, dtype=dtype)
    out["recv_q"], out["recv_s"] = q, s
    rng = np.random.default_rng(9)
    y = make_x(lay.total_rows, w.H, rng) if dtype == "bf16" else make_x_fp16(lay.total_rows, w.H, rng)
    out["combine"] = oracle.combine(y, w.topk_weights, lay.dst_row, dtype=dtype)
    out["dispatch_backward"] = oracle.dispatch_backward(y, lay.dst_row, dtype=dtype)
    g = make_x(w.T, w.H, rng) if dtype == "bf16" else make_x_fp16(w.T, w.H, rng)
    gy, gw = oracle.combine_backward(g, y, w.topk_weights, lay.dst_row, dtype=dtype)
    out["grad_y"], out["grad_w"] = gy, gw
    return out


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_openmp_build_gives_identical_bytes(oracle, dtype):
    w = make_workload("skewed", 0, T=300, H=1024)
    rng = np.random.default_rng(4)
    w.topk_idx[rng.random(w.topk_idx.shape) < 0.1] = -1    # some unused slots
    ref = _all_outputs(oracle, w, dtype)
    for n in (2, 3, 0):                                     # 0: all host cores
        with oracle.threads(n) as used:
            assert used >= 1
            got = _all_outputs(oracle, w, dtype)
        for key in ref:
            a, b = np.asarray(ref[key]), np.asarray(got[key])
            assert a.shape == b.shape and a.dtype == b.dtype, key
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), (n, key)


def test_openmp_build_refuses_the_same_capacity_errors(oracle):
    idx, _ = random_topk(40, 16, 2, np.random.default_rng(1))
    lay = oracle.layout(idx, 16, 4)
    x = make_x(40, 256, np.random.default_rng(2))
    short = int(lay.dst_row.max())                          # one row short of the last used row
    with oracle.threads(4):
        with pytest.raises(oracle.OracleError):
            oracle.dispatch_bf16(x, lay.dst_row, short)
    with pytest.raises(oracle.OracleError):
        oracle.dispatch_bf16(x, lay.dst_row, short)
