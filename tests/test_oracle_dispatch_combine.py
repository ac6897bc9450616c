"""Pins for the oracle's dispatch (BF16 copy, FP8 e4m3 1x128) and combine.

Dispatch BF16 is pinned by the byte-copy invariant.  FP8 is pinned by a
hand-worked block (tests/golden/fp8_block_example.txt), by PyTorch's e4m3
cast applied to the quotients, by the dequantisation error bound of a 3-bit
mantissa, and by invariances a wrong block size, index or scale direction
breaks.  Combine is pinned by closed forms: identity expert with weights
summing to one returns x, one-hot weights return the chosen row, the fp32
slot-order and fused multiply-add semantics on hand-built cancellations, and
an exact fp64 sum within the fp32 accumulation bound.
"""
import os

import numpy as np
import pytest
import torch

from workloads import make_workload, make_x, random_topk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_bits(v):
    return np.asarray(v, np.float32).view(np.uint32)


# ------------------------------------------------------------------ dispatch

def test_dispatch_bf16_copies_rows(oracle):
    rng = np.random.default_rng(1)
    T, H, E, R, k = 37, 64, 8, 2, 3
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.2)
    lay = oracle.layout(idx, E, R, 16)
    recv = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                assert np.array_equal(recv[d], x[t])
    pad_rows = lay.recv_src < 0
    assert np.all(recv[pad_rows] == 0)


def _parse_fp8_golden():
    blocks = {}
    with open(os.path.join(GOLDEN, "fp8_block_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, body = line.split(":", 1)
            _, b, what = head.split()
            b = int(b)
            d = blocks.setdefault(b, {})
            if what == "scale":
                d["scale"] = body.strip()
            else:
                d[what] = dict(tok.split("=") for tok in body.split())
    return blocks


def test_fp8_hand_worked_block(oracle):
    g = _parse_fp8_golden()
    vals = np.zeros(256, np.float32)
    for b, d in g.items():
        for i, v in d["values"].items():
            vals[b * 128 + int(i)] = float.fromhex(v) if "0x" in v else float(v)
    x = bf16_bits(vals)
    assert np.array_equal(oracle.bf16_to_f32(x), vals), "golden values must be exact bf16"
    q, s = oracle.quantize_token_fp8(x)
    for b, d in g.items():
        codes = np.full(128, int(d["codes"].get("rest", "0"), 16), np.uint8)
        for i, c in d["codes"].items():
            if i != "rest":
                codes[int(i)] = int(c, 16)
        assert np.array_equal(q[b * 128:(b + 1) * 128], codes), "block %d" % b
        if d["scale"] == "0":
            assert s[b] == 0.0 and not np.signbit(s[b])
        else:
            num, den = d["scale"].split("/")
            assert s[b] == np.float32(np.float32(num) / np.float32(den))


def _fp8_reference_by_torch(x_bits):
    """Library cross-check: torch's amax, fp32 division and e4m3 cast."""
    xf = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).float()
    T, H = xf.shape
    blk = xf.view(T, H // 128, 128)
    amax = blk.abs().amax(dim=2)
    s = amax / 448.0
    safe = torch.where(s == 0, torch.ones_like(s), s)
    qf = blk / safe.unsqueeze(2)
    q = qf.to(torch.float8_e4m3fn).view(torch.uint8)
    q[s == 0] = 0
    return q.view(T, H).numpy(), s.numpy()


def test_fp8_matches_torch_cast_on_random_tokens(oracle):
    rng = np.random.default_rng(5)
    T, H = 64, 1024
    x = make_x(T, H, rng)
    # spread magnitudes over many binades, including subnormal quotients
    scale = np.float32(2.0) ** rng.integers(-20, 20, size=(T, H // 128, 1)).astype(np.float32)
    xf = (oracle.bf16_to_f32(x).reshape(T, H // 128, 128) * scale).reshape(T, H)
    xf[3, 128:256] = 0.0          # an all-zero block
    xf[4, :128] = -0.0            # an all-negative-zero block
    xf[5, 5] = 0.0
    x = oracle.bf16_round(xf)
    q_ref, s_ref = _fp8_reference_by_torch(x)
    for t in range(T):
        q, s = oracle.quantize_token_fp8(x[t])
        assert np.array_equal(f32_bits(s), f32_bits(s_ref[t])), t
        assert np.array_equal(q, q_ref[t]), t
    q4, s4 = oracle.quantize_token_fp8(x[4])
    assert s4[0] == 0 and np.all(q4[:128] == 0)


def test_fp8_amax_element_encodes_to_448(oracle):
    rng = np.random.default_rng(9)
    x = make_x(16, 512, rng)
    for t in range(16):
        q, s = oracle.quantize_token_fp8(x[t])
        xf = oracle.bf16_to_f32(x[t]).reshape(4, 128)
        qb = q.reshape(4, 128)
        for b in range(4):
            i = int(np.argmax(np.abs(xf[b])))
            assert qb[b, i] == (0xFE if xf[b, i] < 0 else 0x7E)


def test_fp8_dequant_error_bound(oracle):
    # |q*s - x| <= 2^-4 |x| (half a unit of a 3-bit mantissa) in E4M3's normal
    # range, and <= 2^-10 s (half a subnormal step) below it; a little slack
    # covers the fp32 rounding of s and of x / s.
    rng = np.random.default_rng(13)
    x = make_x(32, 1024, rng)
    slack = 1 + 2.0 ** -20
    for t in range(32):
        q, s = oracle.quantize_token_fp8(x[t])
        xf = oracle.bf16_to_f32(x[t]).astype(np.float64).reshape(8, 128)
        deq = oracle.e4m3_decode(q).astype(np.float64).reshape(8, 128) * s.astype(np.float64)[:, None]
        err = np.abs(deq - xf)
        normal = np.abs(xf) >= 2.0 ** -6 * s[:, None]
        assert np.all(err[normal] <= slack * 2.0 ** -4 * np.abs(xf[normal]))
        assert np.all(err[~normal] <= slack * 2.0 ** -10 * np.broadcast_to(s[:, None], xf.shape)[~normal])


def test_fp8_invariances(oracle):
    rng = np.random.default_rng(17)
    x = make_x(1, 512, rng)[0]
    q, s = oracle.quantize_token_fp8(x)
    xf = oracle.bf16_to_f32(x)
    # power-of-two scaling of one block: codes unchanged, its scale scales
    y = xf.copy()
    y[128:256] *= np.float32(2.0 ** 5)
    q2, s2 = oracle.quantize_token_fp8(oracle.bf16_round(y))
    assert np.array_equal(q2, q)
    assert s2[1] == s[1] * np.float32(32) and np.array_equal(np.delete(s2, 1), np.delete(s, 1))
    # negation flips sign bits only (zeros included), scales unchanged
    q3, s3 = oracle.quantize_token_fp8(x ^ np.uint16(0x8000))
    assert np.array_equal(q3, q ^ np.uint8(0x80)) and np.array_equal(s3, s)
    # blocks are independent: changing block 2 leaves blocks 0, 1, 3 alone
    z = xf.copy()
    z[256:384] = rng.standard_normal(128).astype(np.float32) * 50
    q4, s4 = oracle.quantize_token_fp8(oracle.bf16_round(z))
    keep = np.r_[0:256, 384:512]
    assert np.array_equal(q4[keep], q[keep]) and s4[0] == s[0] and s4[1] == s[1] and s4[3] == s[3]


def test_dispatch_fp8_rows_and_scales(oracle):
    rng = np.random.default_rng(19)
    T, H, E, R, k = 20, 384, 8, 4, 2
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, R, 4)
    q, s = oracle.dispatch_fp8(x, lay.dst_row, lay.total_rows)
    assert q.shape == (lay.total_rows, H) and s.shape == (lay.total_rows, H // 128)
    for t in range(T):
        qt, st = oracle.quantize_token_fp8(x[t])
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                assert np.array_equal(q[d], qt) and np.array_equal(s[d], st)


# ------------------------------------------------------------------ combine

def test_combine_identity_expert_returns_x(oracle):
    # Tiny config: identity expert, weights renormalised to sum 1, so the
    # combine must return x up to the rounding of the weights (1 bf16 ulp).
    w = make_workload("tiny", 0)
    res = oracle.pipeline(w.x_bits, w.topk_idx, w.topk_weights, w.E, w.R, w.fmt, w.expert_c)
    out = oracle.bf16_to_f32(res["out"]).astype(np.float64)
    x = oracle.bf16_to_f32(w.x_bits).astype(np.float64)
    ulp = np.ldexp(1.0, np.frexp(np.abs(x))[1] - 8)
    assert np.all(np.abs(out - x) <= ulp)
    assert np.mean(res["out"] == w.x_bits) > 0.99


def test_combine_one_hot_weights_pick_the_row(oracle):
    rng = np.random.default_rng(23)
    T, H, E, k = 16, 64, 8, 4
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, 2, 8)
    y = make_x(lay.total_rows, H, rng)
    for jj in range(k):
        w = np.zeros((T, k), np.float32)
        w[:, jj] = 1.0
        out = oracle.combine(y, w, lay.dst_row)
        assert np.array_equal(out, y[lay.dst_row[:, jj]])


def test_combine_k1_is_a_gather(oracle):
    rng = np.random.default_rng(29)
    T, H, E = 50, 32, 16
    idx, _ = random_topk(T, E, 1, rng)
    lay = oracle.layout(idx, E, 4, 128)
    y = make_x(lay.total_rows, H, rng)
    out = oracle.combine(y, np.ones((T, 1), np.float32), lay.dst_row)
    assert np.array_equal(out, y[lay.dst_row[:, 0]])


def test_combine_fp32_slot_order_and_fma(oracle):
    dst = np.array([[0, 1, 2]], np.int32)
    # fp32 accumulation in slot order: 1 + 2^25 rounds away the 1, then the
    # big terms cancel -> 0 (an fp64 or reversed-order sum would give 1).
    y = bf16_bits([[1.0], [2.0 ** 25], [-(2.0 ** 25)]])
    out = oracle.combine(y, np.ones((1, 3), np.float32), dst)
    assert oracle.bf16_to_f32(out)[0, 0] == 0.0
    y_rev = bf16_bits([[-(2.0 ** 25)], [2.0 ** 25], [1.0]])
    out_rev = oracle.combine(y_rev, np.ones((1, 3), np.float32), dst)
    assert oracle.bf16_to_f32(out_rev)[0, 0] == 1.0
    # fused multiply-add: w1*y1 = 1 + 2^-7 + 2^-23 + 2^-30 exactly; a rounded
    # product would cancel to 0 against acc = -(1 + 2^-7 + 2^-23).
    w = np.array([[1.0 + 2.0 ** -7 + 2.0 ** -23, 1.0 + 2.0 ** -23]], np.float32)
    y = bf16_bits([[-1.0], [1.0 + 2.0 ** -7]])
    out = oracle.combine(y, w, np.array([[0, 1]], np.int32))
    assert oracle.bf16_to_f32(out)[0, 0] == np.float32(2.0 ** -30)


def test_combine_within_fp32_bound_of_exact_sum(oracle):
    rng = np.random.default_rng(31)
    T, H, E, k = 40, 256, 16, 8
    idx, w = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, 4, 16)
    y = make_x(lay.total_rows, H, rng)
    out = oracle.bf16_to_f32(oracle.combine(y, w, lay.dst_row)).astype(np.float64)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    exact = np.zeros((T, H))
    absum = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d >= 0:
                exact[t] += float(w[t, j]) * yf[d]
                absum[t] += abs(float(w[t, j])) * np.abs(yf[d])
    # fp32 fma chain of <= k terms: |acc - exact| <= k 2^-24 sum|w y| (first
    # order); then one bf16 rounding: half an ulp of the result.
    acc_err = k * 2.0 ** -24 * absum * (1 + 1e-6)
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(exact) + acc_err)[1] - 9)
    assert np.all(np.abs(out - exact) <= acc_err + half_ulp)


def test_combine_skips_unused_slots(oracle):
    y = bf16_bits([[3.0], [5.0]])
    w = np.array([[100.0, 0.5, 2.0]], np.float32)
    out = oracle.combine(y, w, np.array([[-1, 0, 1]], np.int32))
    assert oracle.bf16_to_f32(out)[0, 0] == 11.5
