"""Pins for the oracle's FP16 input support: IEEE binary16 widening and
rounding, FP8 e4m3 1x128 quantisation of binary16 rows, and combine with
binary16 expert outputs and result.

binary16 is written from its definition in the oracle; here it is checked
against NumPy's float16 (a library routine, run, not read): every one of the
65 536 bit patterns for widening, and for rounding the whole binary16 grid,
every midpoint between neighbours (ties to even), the fp32 neighbours of each
midpoint, random fp32 values over all binades and the overflow edge.  FP8 of
binary16 rows is pinned by PyTorch's e4m3 cast of the quotients, the amax
code and the dequantisation bound; combine by one-hot weights, slot-order
cancellation, overflow to infinity and the exact fp64 sum within the fp32
accumulation bound plus half a binary16 ulp.
"""
import numpy as np
import pytest
import torch

from workloads import make_x_fp16, random_topk


def f16_bits(vals):
    with np.errstate(over="ignore"):
        return np.asarray(vals, np.float32).astype(np.float16).view(np.uint16)


# ------------------------------------------------------------------ binary16

def test_fp16_widen_every_pattern_vs_numpy(oracle):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.fp16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got.view(np.uint32)[~nan], ref.view(np.uint32)[~nan])


def _numpy_round(v):
    with np.errstate(over="ignore"):   # overflow to infinity is the point of some cases
        return np.asarray(v, np.float32).astype(np.float16).view(np.uint16)


def test_fp16_round_grid_midpoints_and_neighbours_vs_numpy(oracle):
    h = np.arange(0, 0x7c00, dtype=np.uint32).astype(np.uint16)       # +0 .. 65504
    grid = h.view(np.float16).astype(np.float64)
    mids = (grid[:-1] + grid[1:]) / 2                                   # exact in fp32
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)
    up = np.nextafter(mids32, np.float32(np.inf))
    down = np.nextafter(mids32, np.float32(0))
    top = np.float32(65520.0)                                           # 65504 + half a step
    vals = np.concatenate([grid.astype(np.float32), mids32, up, down,
                           [top, np.nextafter(top, np.float32(0)), np.float32(65536.0),
                            np.float32(1e30), np.float32(np.inf)]])
    vals = np.concatenate([vals, -vals])
    assert np.array_equal(oracle.fp16_round(vals), _numpy_round(vals))


def test_fp16_round_random_fp32_vs_numpy(oracle):
    rng = np.random.default_rng(101)
    bits = rng.integers(0, 2 ** 32, size=400_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]
    assert np.array_equal(oracle.fp16_round(v), _numpy_round(v))


def test_fp16_round_special_values(oracle):
    cases = [(65504.0, 0x7BFF), (65519.99609375, 0x7BFF), (65520.0, 0x7C00), (-65520.0, 0xFC00),
             (2.0 ** -24, 0x0001), (2.0 ** -25, 0x0000),            # tie to even: 0
             (3 * 2.0 ** -25, 0x0002),                              # tie to even: 2 units
             (2.0 ** -14, 0x0400), (-0.0, 0x8000), (1.0 + 2.0 ** -11, 0x3C00),
             (1.0 + 3 * 2.0 ** -11, 0x3C02)]
    for v, code in cases:
        assert int(oracle.fp16_round(np.array([v], np.float32))[0]) == code, v
    n = oracle.fp16_round(np.array([np.nan, -np.nan], np.float32))
    assert np.all((n & 0x7C00) == 0x7C00) and np.all((n & 0x03FF) != 0)


# ------------------------------------------------------------------ FP8 of binary16 rows

def _fp8_reference_by_torch_fp16(x_bits):
    xf = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.float16).float()
    T, H = xf.shape
    blk = xf.view(T, H // 128, 128)
    amax = blk.abs().amax(dim=2)
    s = amax / 448.0
    safe = torch.where(s == 0, torch.ones_like(s), s)
    q = (blk / safe.unsqueeze(2)).to(torch.float8_e4m3fn).view(torch.uint8)
    q[s == 0] = 0
    return q.view(T, H).numpy(), s.numpy()


def test_fp8_of_fp16_matches_torch_cast(oracle):
    rng = np.random.default_rng(103)
    T, H = 48, 1024
    xf = rng.standard_normal((T, H), dtype=np.float32)
    # magnitudes over the binary16 range, subnormal inputs included
    scale = np.float32(2.0) ** rng.integers(-22, 13, size=(T, H // 128, 1)).astype(np.float32)
    xf = (xf.reshape(T, H // 128, 128) * scale).reshape(T, H)
    xf[2, 256:384] = 0.0
    xf[3, :128] = -0.0
    x = f16_bits(xf)
    q_ref, s_ref = _fp8_reference_by_torch_fp16(x)
    for t in range(T):
        q, s = oracle.quantize_token_fp8(x[t], dtype="fp16")
        assert np.array_equal(s.view(np.uint32), s_ref[t].view(np.uint32)), t
        assert np.array_equal(q, q_ref[t]), t


def test_fp8_of_fp16_amax_code_and_error_bound(oracle):
    rng = np.random.default_rng(107)
    x = make_x_fp16(16, 1024, rng)
    slack = 1 + 2.0 ** -20
    for t in range(16):
        q, s = oracle.quantize_token_fp8(x[t], dtype="fp16")
        xf = oracle.fp16_to_f32(x[t]).astype(np.float64).reshape(8, 128)
        qb = q.reshape(8, 128)
        for b in range(8):
            i = int(np.argmax(np.abs(xf[b])))
            assert qb[b, i] == (0xFE if xf[b, i] < 0 else 0x7E)
        deq = oracle.e4m3_decode(q).astype(np.float64).reshape(8, 128) * s.astype(np.float64)[:, None]
        err = np.abs(deq - xf)
        normal = np.abs(xf) >= 2.0 ** -6 * s[:, None]
        assert np.all(err[normal] <= slack * 2.0 ** -4 * np.abs(xf[normal]))
        assert np.all(err[~normal] <= slack * 2.0 ** -10 * np.broadcast_to(s[:, None], xf.shape)[~normal])


def test_fp8_of_fp16_differs_from_bf16_reading(oracle):
    # the same bits read as bf16 give other values: the dtype is honoured
    x = f16_bits(np.linspace(-3, 3, 128, dtype=np.float32))
    q16, s16 = oracle.quantize_token_fp8(x, dtype="fp16")
    qb, sb = oracle.quantize_token_fp8(x, dtype="bf16")
    assert s16[0] == np.float32(np.float32(3.0) / np.float32(448.0))
    assert s16[0] != sb[0]


def test_dispatch_fp8_of_fp16_rows_and_mn_scales(oracle):
    rng = np.random.default_rng(109)
    T, H, E, k = 30, 512, 8, 3
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 2, 8)
    x = make_x_fp16(T, H, rng)
    q, s = oracle.dispatch_fp8(x, lay.dst_row, lay.total_rows, dtype="fp16")
    cap = (lay.total_rows + 3) // 4 * 4
    qm, sm = oracle.dispatch_fp8_mn(x, lay.dst_row, cap, cap, dtype="fp16")
    for t in range(T):
        qt, st = oracle.quantize_token_fp8(x[t], dtype="fp16")
        for j in range(k):
            d = lay.dst_row[t, j]
            if d < 0:
                continue
            assert np.array_equal(q[d], qt) and np.array_equal(s[d], st)
            assert np.array_equal(qm[d], qt) and np.array_equal(sm[:, d], st)


# ------------------------------------------------------------------ combine, binary16

def test_combine_fp16_one_hot_and_k1(oracle):
    rng = np.random.default_rng(113)
    T, H, E, k = 20, 64, 8, 4
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, 2, 4)
    y = make_x_fp16(lay.total_rows, H, rng)
    for j in range(k):
        w = np.zeros((T, k), np.float32)
        w[:, j] = 1.0
        out = oracle.combine(y, w, lay.dst_row, dtype="fp16")
        assert np.array_equal(out, y[lay.dst_row[:, j]])


def test_combine_fp16_slot_order_overflow_and_rounding(oracle):
    dst = np.array([[0, 1, 2]], np.int32)
    y = f16_bits([[1.0], [1.0], [1.0]])
    # fp32 chain in slot order: 1 + 2^25 absorbs the 1, then cancels to 0
    out = oracle.combine(y, np.array([[1.0, 2.0 ** 25, -(2.0 ** 25)]], np.float32), dst, dtype="fp16")
    assert oracle.fp16_to_f32(out)[0, 0] == 0.0
    out = oracle.combine(y, np.array([[2.0 ** 25, -(2.0 ** 25), 1.0]], np.float32), dst, dtype="fp16")
    assert oracle.fp16_to_f32(out)[0, 0] == 1.0
    # a sum past 65520 rounds to infinity in binary16
    y2 = f16_bits([[60000.0], [60000.0]])
    out = oracle.combine(y2, np.ones((1, 2), np.float32), np.array([[0, 1]], np.int32), dtype="fp16")
    assert np.isinf(oracle.fp16_to_f32(out)[0, 0])
    # the result is rounded to binary16, ties to even: 1 + 2^-11 -> 1
    y3 = f16_bits([[1.0], [2.0 ** -11]])
    out = oracle.combine(y3, np.ones((1, 2), np.float32), np.array([[0, 1]], np.int32), dtype="fp16")
    assert int(out[0, 0]) == 0x3C00


def test_combine_fp16_within_bound_of_exact_sum(oracle):
    rng = np.random.default_rng(127)
    T, H, E, k = 40, 256, 16, 8
    idx, w = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 4, 16)
    y = make_x_fp16(lay.total_rows, H, rng)
    out = oracle.fp16_to_f32(oracle.combine(y, w, lay.dst_row, dtype="fp16")).astype(np.float64)
    yf = oracle.fp16_to_f32(y).astype(np.float64)
    exact = np.zeros((T, H))
    absum = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                exact[t] += float(w[t, j]) * yf[d]
                absum[t] += abs(float(w[t, j])) * np.abs(yf[d])
    acc_err = k * 2.0 ** -24 * absum * (1 + 1e-6)
    # half a binary16 ulp of the result (normal range; subnormal step 2^-25)
    half_ulp = np.maximum(np.ldexp(1.0, np.frexp(np.abs(exact) + acc_err)[1] - 12), 2.0 ** -25)
    assert np.all(np.abs(out - exact) <= acc_err + half_ulp)


# ------------------------------------------------------------------ backward, binary16

def test_dispatch_backward_fp16_gather_and_bound(oracle):
    rng = np.random.default_rng(131)
    T, H, E, k = 40, 128, 16, 4
    idx1, _ = random_topk(T, E, 1, rng)
    lay1 = oracle.layout(idx1, E, 4, 8)
    g1 = make_x_fp16(lay1.total_rows, H, rng)
    assert np.array_equal(oracle.dispatch_backward(g1, lay1.dst_row, dtype="fp16"),
                          g1[lay1.dst_row[:, 0]])                      # k = 1: a gather
    idx, _ = random_topk(T, E, k, rng, p_unused=0.2)
    lay = oracle.layout(idx, E, 4, 8)
    g = make_x_fp16(lay.total_rows, H, rng)
    gx = oracle.fp16_to_f32(oracle.dispatch_backward(g, lay.dst_row, dtype="fp16")).astype(np.float64)
    gf = oracle.fp16_to_f32(g).astype(np.float64)
    exact = np.zeros((T, H))
    absum = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                exact[t] += gf[d]
                absum[t] += np.abs(gf[d])
    acc_err = k * 2.0 ** -24 * absum * (1 + 1e-6)
    half_ulp = np.maximum(np.ldexp(1.0, np.frexp(np.abs(exact) + acc_err)[1] - 12), 2.0 ** -25)
    assert np.all(np.abs(gx - exact) <= acc_err + half_ulp)


def test_combine_backward_fp16_scaling_and_dot(oracle):
    rng = np.random.default_rng(137)
    T, H, E, k = 30, 256, 8, 3
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, 2, 4)
    y = make_x_fp16(lay.total_rows, H, rng)
    g = make_x_fp16(T, H, rng)
    # power-of-two weights scale grad_out exactly (within the binary16 range)
    w = (2.0 ** rng.integers(-3, 3, size=(T, k))).astype(np.float32)
    gy, gw = oracle.combine_backward(g, y, w, lay.dst_row, dtype="fp16")
    gf = oracle.fp16_to_f32(g).astype(np.float64)
    yf = oracle.fp16_to_f32(y).astype(np.float64)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            assert np.array_equal(oracle.fp16_to_f32(gy[d]).astype(np.float64), w[t, j] * gf[t])
            ref = np.float32(np.dot(gf[t], yf[d]))
            assert abs(gw[t, j] - ref) <= abs(ref) * 2.0 ** -23 + 1e-30
    # the bf16 reading of the same bits differs: the type is honoured
    _, gw_b = oracle.combine_backward(g, y, w, lay.dst_row, dtype="bf16")
    assert not np.array_equal(gw, gw_b)
