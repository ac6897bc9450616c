"""Pins for the oracle's GEMM-ready receive-layout helpers.

Per-row weights: every used slot's weight lands on its row (a scatter that a
brute-force loop over the layout reproduces), pad rows keep their fill.
Zero pad rows: exactly the rows with recv_src == -1 become zero, others are
untouched.  MN-major scales: the transpose of the row-major FP8 scales, with
identical codes.
"""
import numpy as np

from workloads import make_x, random_topk


def test_dispatch_weights_scatter(oracle):
    rng = np.random.default_rng(61)
    T, E, k = 70, 16, 4
    idx, w = random_topk(T, E, k, rng, p_unused=0.2)
    lay = oracle.layout(idx, E, 4, 8)
    rw = oracle.dispatch_weights(w, lay.dst_row, lay.total_rows, fill=-7.0)
    seen = np.zeros(lay.total_rows, bool)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                assert rw[d] == w[t, j]
                seen[d] = True
    assert np.all(rw[~seen] == -7.0)
    assert np.array_equal(~seen, lay.recv_src < 0)


def test_zero_pad_rows(oracle):
    rng = np.random.default_rng(67)
    idx, _ = random_topk(40, 8, 3, rng)
    lay = oracle.layout(idx, 8, 2, 16)
    rows = make_x(lay.total_rows, 24, rng)
    z = oracle.zero_pad_rows(lay.recv_src, rows)
    pad = lay.recv_src < 0
    assert np.all(z[pad] == 0) and np.array_equal(z[~pad], rows[~pad])
    f = rng.random((lay.total_rows, 3)).astype(np.float32) + 1
    zf = oracle.zero_pad_rows(lay.recv_src, f)
    assert np.all(zf[pad] == 0) and np.array_equal(zf[~pad], f[~pad])


def test_fp8_mn_major_is_the_transpose(oracle):
    rng = np.random.default_rng(71)
    T, H, E, k = 30, 640, 16, 3
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 4, 8)
    P = lay.total_rows
    ld = P + 4
    q1, s1 = oracle.dispatch_fp8(x, lay.dst_row, P)
    q2, s2 = oracle.dispatch_fp8_mn(x, lay.dst_row, P, ld)
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(q1[rows], q2[rows])
    assert np.array_equal(s2[:, rows].T, s1[rows])
    assert s2.shape == (H // 128, ld)
