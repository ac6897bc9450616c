"""Pins for the oracle's backward functions (gradients of dispatch and combine).

dispatch backward: grad_x[t] = sum over used slots of grad_recv[dst_row[t, j]]
(fp32 in slot order, bf16 out).  Pinned by the k = 1 gather, a hand-built
cancellation that fixes the slot order, and the exact fp64 sum within the
fp32 accumulation bound.

combine backward: grad_y[dst_row[t, j]] = bf16(w[t, j] * grad_out[t]) and
grad_w[t, j] = <grad_out[t], y[dst_row[t, j]]>.  Pinned by exact scalings
(w = 1 and powers of two), the adjoint identity
<combine(y, w), G> = sum_rows <y_row, grad_y_row> (exact for power-of-two
weights), and NumPy's float64 dot product for grad_w.
"""
import numpy as np
import pytest

from workloads import make_x, random_topk


def _f(oracle, bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


def test_dispatch_backward_k1_is_a_gather(oracle):
    rng = np.random.default_rng(41)
    idx, _ = random_topk(60, 16, 1, rng)
    lay = oracle.layout(idx, 16, 4, 8)
    g = make_x(lay.total_rows, 64, rng)
    gx = oracle.dispatch_backward(g, lay.dst_row)
    assert np.array_equal(gx, g[lay.dst_row[:, 0]])


def test_dispatch_backward_slot_order_cancellation(oracle):
    g = oracle.bf16_round(np.array([[1.0] * 8, [2.0 ** 25] * 8, [-(2.0 ** 25)] * 8], np.float32))
    fwd = oracle.dispatch_backward(g, np.array([[0, 1, 2]], np.int32))
    rev = oracle.dispatch_backward(g, np.array([[2, 1, 0]], np.int32))
    assert np.all(oracle.bf16_to_f32(fwd) == 0.0)   # fp32, slot order: 1 is absorbed
    assert np.all(oracle.bf16_to_f32(rev) == 1.0)


def test_dispatch_backward_within_fp32_bound_and_skips_unused(oracle):
    rng = np.random.default_rng(43)
    T, H, E, k = 50, 128, 16, 6
    idx, _ = random_topk(T, E, k, rng, p_unused=0.2)
    lay = oracle.layout(idx, E, 4, 8)
    g = make_x(lay.total_rows, H, rng)
    gx = _f(oracle, oracle.dispatch_backward(g, lay.dst_row))
    gf = _f(oracle, g)
    exact = np.zeros((T, H))
    absum = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                exact[t] += gf[d]
                absum[t] += np.abs(gf[d])
    acc_err = k * 2.0 ** -24 * absum * (1 + 1e-6)
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(exact) + acc_err)[1] - 9)
    assert np.all(np.abs(gx - exact) <= acc_err + half_ulp)


def test_combine_backward_unit_and_power_of_two_weights_scale_exactly(oracle):
    rng = np.random.default_rng(47)
    T, H, E, k = 40, 64, 8, 3
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, 2, 4)
    y = make_x(lay.total_rows, H, rng)
    g = make_x(T, H, rng)
    gy, _ = oracle.combine_backward(g, y, np.ones((T, k), np.float32), lay.dst_row)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(gy[lay.dst_row[t, j]], g[t])
    w = (2.0 ** rng.integers(-3, 4, size=(T, k))).astype(np.float32) * \
        rng.choice([-1, 1], size=(T, k)).astype(np.float32)
    gy, _ = oracle.combine_backward(g, y, w, lay.dst_row)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(_f(oracle, gy[lay.dst_row[t, j]]), w[t, j] * _f(oracle, g[t]))


def test_combine_backward_adjoint_identity(oracle):
    # <sum_j w_tj y_row(t,j), G_t> summed over t equals sum over rows of
    # <y_row, grad_y_row> when grad_y is exact (power-of-two weights).
    rng = np.random.default_rng(53)
    T, H, E, k = 30, 96, 12, 4
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 3, 8)
    y = make_x(lay.total_rows, H, rng)
    g = make_x(T, H, rng)
    w = (2.0 ** rng.integers(-2, 3, size=(T, k))).astype(np.float32)
    gy, _ = oracle.combine_backward(g, y, w, lay.dst_row)
    yf, gf, gyf = _f(oracle, y), _f(oracle, g), _f(oracle, gy)
    lhs = sum(float(w[t, j]) * float(yf[lay.dst_row[t, j]] @ gf[t])
              for t in range(T) for j in range(k) if lay.dst_row[t, j] >= 0)
    rhs = float(np.sum(yf * gyf))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs))


def test_combine_backward_grad_w_is_the_dot_product(oracle):
    rng = np.random.default_rng(59)
    T, H, E, k = 25, 7168, 32, 8
    idx, wt = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 4, 16)
    y = make_x(lay.total_rows, H, rng)
    g = make_x(T, H, rng)
    _, gw = oracle.combine_backward(g, y, wt, lay.dst_row)
    yf, gf = _f(oracle, y), _f(oracle, g)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d < 0:
                assert gw[t, j] == 0.0
                continue
            ref = np.float32(np.dot(gf[t], yf[d]))       # library fp64 dot, one rounding
            assert abs(gw[t, j] - ref) <= abs(ref) * 2.0 ** -23 + 1e-30


def test_combine_backward_leaves_pad_rows_alone(oracle):
    idx = np.array([[0, -1], [1, 0]], np.int64)
    lay = oracle.layout(idx, 2, 1, 4)
    y = oracle.bf16_round(np.ones((lay.total_rows, 8), np.float32))
    g = oracle.bf16_round(np.full((2, 8), 3.0, np.float32))
    gy, gw = oracle.combine_backward(g, y, np.array([[0.5, 9.0], [2.0, 0.25]], np.float32),
                                     lay.dst_row)
    pad = lay.recv_src < 0
    assert np.all(gy[pad] == 0)
    assert gw[0, 1] == 0.0 and gw[0, 0] == 24.0 and gw[1, 0] == 24.0
