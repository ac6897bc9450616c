"""GPU parity of ep_dispatch (BF16 and FP8 e4m3 1x128) and ep_combine against
the oracle.

Bars: dispatch payload, FP8 bytes and fp32 scales bit-exact on every non-pad
row; combine within 1 bf16 ulp per element (the tolerance the design states;
the fused multiply-add chain in slot order is expected to match exactly, and
the exact-match fraction is asserted too).  Pad rows and guard bands around
the receive buffer must keep their sentinel bytes.
"""
import numpy as np
import pytest
import torch

from workloads import make_workload, make_x, make_x_scale_sweep, random_topk

pytestmark = pytest.mark.gpu

SENTINEL = 0x5A


def _handle(T, k, E, R, B=128):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV

    return ep.ep_handle_create(max(T, 1), k, E, R, B, device=DEV)


def _guarded(rows, H, dtype, guard_rows=4):
    """A receive buffer with guard rows on both sides, all bytes = SENTINEL."""
    from gpu_util import DEV

    esize = torch.empty((), dtype=dtype).element_size()
    raw = torch.full(((rows + 2 * guard_rows) * H * esize,), SENTINEL, dtype=torch.uint8,
                     device=DEV)
    full = raw.view(dtype).view(rows + 2 * guard_rows, H)
    return full, full[guard_rows: guard_rows + rows]


def _check_guards(full, guard_rows=4):
    b = full.view(torch.uint8).view(full.shape[0], -1)
    assert bool((b[:guard_rows] == SENTINEL).all()), "write below the receive buffer"
    assert bool((b[-guard_rows:] == SENTINEL).all()), "write above the receive buffer"


def dispatch_case(oracle, x_bits, idx, E, R, fmt, B=128, x_offset=0):
    """x_offset > 0 places x that many bf16 elements past an aligned base, so a
    16-byte but not 32-byte aligned x takes the 16-byte kernels."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16, nonpad_rows

    T, H = x_bits.shape
    k = idx.shape[1]
    lay = oracle.layout(idx, E, R, B)
    h = _handle(T, k, E, R, B)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    P = lay.total_rows
    if x_offset:
        base = torch.empty(T * H + x_offset, dtype=torch.bfloat16, device=DEV)
        x = base[x_offset:].view(T, H)
        x.copy_(bits_to_bf16(x_bits))
        assert x.data_ptr() % 32 != 0 and x.data_ptr() % 16 == 0
    else:
        x = bits_to_bf16(x_bits)
    rows = nonpad_rows(lay)
    padr = np.nonzero(lay.recv_src < 0)[0]
    if fmt == "bf16":
        full, recv = _guarded(P, H, torch.bfloat16)
        ep.ep_dispatch(h, x, "bf16", recv_x=recv)
        ep.ep_handle_check(h)
        got = recv.view(torch.int16).cpu().numpy().view(np.uint16)
        exp = oracle.dispatch_bf16(x_bits, lay.dst_row, P)
        assert np.array_equal(got[rows], exp[rows])
    else:
        full, recv = _guarded(P, H, torch.float8_e4m3fn)
        sfull, scales = _guarded(P, H // 128, torch.float32)
        ep.ep_dispatch(h, x, "fp8", recv_x=recv, recv_scales=scales)
        ep.ep_handle_check(h)
        got_q = recv.view(torch.uint8).cpu().numpy()
        got_s = scales.cpu().numpy()
        exp_q, exp_s = oracle.dispatch_fp8(x_bits, lay.dst_row, P)
        if not np.array_equal(got_q[rows], exp_q[rows]):
            bad = np.argwhere(got_q[rows] != exp_q[rows])[:5]
            raise AssertionError("fp8 bytes differ at %s: got %s expected %s" % (
                bad.tolist(), got_q[rows][tuple(bad.T)], exp_q[rows][tuple(bad.T)]))
        assert np.array_equal(got_s[rows].view(np.uint32), exp_s[rows].view(np.uint32))
        sb = scales.view(torch.uint8).view(P, -1).cpu().numpy()
        assert np.all(sb[padr] == SENTINEL), "a pad row's scales were written"
        _check_guards(sfull)
    b = recv.view(torch.uint8).view(P, -1).cpu().numpy()
    assert np.all(b[padr] == SENTINEL), "a pad row was written"
    _check_guards(full)
    return h, lay


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("tiny", 3), ("decode", 0), ("decode", 1),
                                       ("dsv3", 0)])
def test_dispatch_configs(oracle, name, seed):
    w = make_workload(name, seed)
    dispatch_case(oracle, w.x_bits, w.topk_idx, w.E, w.R, w.fmt)


@pytest.mark.parametrize("T,H,E,R,k,fmt,p_unused", [
    (1, 8, 4, 2, 2, "bf16", 0.0),
    (45, 264, 16, 4, 3, "bf16", 0.1),     # H/8 = 33 vectors: a ragged unit tail
    (300, 2056, 32, 8, 8, "bf16", 0.0),   # 257 vectors
    (64, 7168, 256, 8, 8, "bf16", 0.3),
    (1, 128, 4, 2, 2, "fp8", 0.0),
    (45, 384, 16, 4, 3, "fp8", 0.1),      # 3 blocks: a partial unit of 8 blocks
    (70, 1152, 32, 8, 8, "fp8", 0.0),     # 9 blocks
    (33, 7168, 256, 32, 8, "fp8", 0.2),
    (40, 2048, 64, 8, 20, "fp8", 0.0),    # k = 20 > 8
])
def test_dispatch_fuzz(oracle, T, H, E, R, k, fmt, p_unused):
    rng = np.random.default_rng(T * 31 + H)
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=p_unused)
    dispatch_case(oracle, x, idx, E, R, fmt)


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_dispatch_16byte_kernels_on_unaligned_x(oracle, fmt):
    rng = np.random.default_rng(11)
    T, H, E, R, k = 150, 1024, 32, 8, 8
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    dispatch_case(oracle, x, idx, E, R, fmt, x_offset=8)


def test_dispatch_fp8_special_values(oracle):
    rng = np.random.default_rng(77)
    T, H, E, R, k = 16, 1024, 16, 4, 2
    xf = rng.standard_normal((T, H)).astype(np.float32)
    xf[0, :128] = 0.0                       # amax = 0
    xf[1, :128] = -0.0                      # amax = 0 with negative zeros
    xf[2, :] *= 2.0 ** -126                 # subnormal-range bf16 inputs, tiny scales
    xf[3, :128] = 0.0
    xf[3, 5] = 2.0 ** -133                  # smallest bf16 subnormal as amax
    xf[4, :] *= 3.0e37                      # near the top of the bf16 range
    xf[5, ::2] = 0.0
    xf[6, :128] = 1.0                       # every element equals amax
    xf[7, :] = np.round(xf[7, :] * 4) / 4   # many exact ties after scaling
    x = oracle.bf16_round(xf)
    idx, _ = random_topk(T, E, k, rng)
    dispatch_case(oracle, x, idx, E, R, "fp8")


@pytest.mark.parametrize("x_offset", [0, 8])  # the 32-byte and the 16-byte kernels
def test_dispatch_fp8_scale_sweep(oracle, x_offset):
    rng = np.random.default_rng(2024 + x_offset)
    T, H, E, R, k = 512, 7168, 16, 4, 2
    x = make_x_scale_sweep(T, H, rng)
    idx, _ = random_topk(T, E, k, rng)
    dispatch_case(oracle, x, idx, E, R, "fp8", x_offset=x_offset)


def test_dispatch_capacity_overflow_is_reported_and_bounded(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16

    rng = np.random.default_rng(3)
    T, H, E, R, k = 200, 256, 16, 4, 4
    x_bits = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, R)
    cap = lay.total_rows // 2
    h = _handle(T, k, E, R)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    full, recv = _guarded(cap, H, torch.bfloat16)
    ep.ep_dispatch(h, bits_to_bf16(x_bits), "bf16", recv_x=recv)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY
    _check_guards(full)
    exp = oracle.dispatch_bf16(x_bits, lay.dst_row, lay.total_rows)
    got = recv.view(torch.int16).cpu().numpy().view(np.uint16)
    rows = lay.dst_row[(lay.dst_row >= 0) & (lay.dst_row < cap)]
    assert np.array_equal(got[rows], exp[rows])
    # the same for FP8, and for combine with too few y rows
    full, recv = _guarded(cap, H, torch.float8_e4m3fn)
    sfull, sc = _guarded(cap, H // 128, torch.float32)
    ep.ep_dispatch(h, bits_to_bf16(x_bits), "fp8", recv_x=recv, recv_scales=sc)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY
    _check_guards(full)
    _check_guards(sfull)
    y = torch.zeros((cap, H), dtype=torch.bfloat16, device=DEV)
    w = torch.ones((T, k), dtype=torch.float32, device=DEV)
    ep.ep_combine(h, y, w)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY


def combine_case(oracle, y_bits, w, idx, E, R, B=128, exact_frac=1.0):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bf16_ulp_diff, bits_to_bf16

    T, k = idx.shape
    H = y_bits.shape[1]
    lay = oracle.layout(idx, E, R, B)
    h = _handle(T, k, E, R, B)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    out = ep.ep_combine(h, bits_to_bf16(y_bits), torch.from_numpy(w).to(DEV))
    ep.ep_handle_check(h)
    got = bf16_to_bits(out)
    exp = oracle.combine(y_bits, w, lay.dst_row)
    d = bf16_ulp_diff(got, exp)
    assert d.max(initial=0) <= 1, "combine differs by %d bf16 ulp" % d.max()
    assert (got == exp).mean() >= exact_frac if got.size else True
    return got, exp


@pytest.mark.parametrize("T,H,E,R,k,p_unused", [
    (1, 8, 4, 2, 2, 0.0),
    (100, 264, 16, 4, 3, 0.1),
    (257, 1024, 64, 8, 8, 0.0),
    (64, 7168, 256, 8, 8, 0.2),
    (50, 512, 64, 8, 32, 0.1),       # k = 32 takes the general path
    (80, 136, 8, 2, 1, 0.0),         # k = 1
])
def test_combine_random_y(oracle, T, H, E, R, k, p_unused):
    # y rows are independent draws (mixed signs: cancellation inside the
    # fp32 chain), weights U(0,1); the fma chain in slot order is expected to
    # match the oracle bit for bit.
    rng = np.random.default_rng(T + H + k)
    idx, w = random_topk(T, E, k, rng, p_unused=p_unused)
    P = oracle.layout(idx, E, R).total_rows
    y = make_x(max(P, 1), H, rng)
    combine_case(oracle, y, w, idx, E, R)


def test_combine_right_after_a_new_layout(oracle):
    """Layouts of two different routings alternate on one handle with no
    synchronisation, each followed at once by a combine: a combine starts
    while the layout ahead of it still writes dst_row, so the rows it
    prefetches before its dependent-launch wait may be the previous
    routing's.  Every result must be the one of its own routing (bit-exact)."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    rng = np.random.default_rng(5150)
    T, H, E, R, k = 128, 7168, 256, 16, 8
    idx_a, w_a = random_topk(T, E, k, rng)
    idx_b, w_b = random_topk(T, E, k, rng)
    idx_b[::7] = idx_a[::7]  # some tokens keep their rows, most move
    lays = [oracle.layout(idx_a, E, R), oracle.layout(idx_b, E, R)]
    P = max(l.total_rows for l in lays)
    y_bits = make_x(P, H, rng)
    y = bits_to_bf16(y_bits)
    h = _handle(T, k, E, R)
    idx_d = [torch.from_numpy(i).to(DEV) for i in (idx_a, idx_b)]
    w_d = [torch.from_numpy(w).to(DEV) for w in (w_a, w_b)]
    outs = [torch.empty((T, H), dtype=torch.bfloat16, device=DEV) for _ in range(20)]
    for i in range(20):
        ep.ep_layout(h, idx_d[i % 2])
        ep.ep_combine(h, y, w_d[i % 2], out=outs[i])
    ep.ep_handle_check(h)
    exp = [oracle.combine(y_bits, w, l.dst_row) for w, l in zip((w_a, w_b), lays)]
    for i in range(20):
        assert np.array_equal(bf16_to_bits(outs[i]), exp[i % 2]), "combine %d" % i


def test_combine_cancellation_and_fma_cases(oracle):
    # Expert e's rows all hold vals[e]; the expected values are closed forms
    # (the same cases pin the oracle): fp32 slot order gives 0 and 1 for the
    # two orders of 1, 2^25, -2^25, and the fused multiply-add keeps 2^-30.
    vals = np.array([1.0, 2.0 ** 25, -(2.0 ** 25), -1.0, 1.0 + 2.0 ** -7], np.float32)
    idx = np.array([[0, 1, 2], [2, 1, 0], [3, 4, -1]], np.int64)
    w = np.array([[1, 1, 1], [1, 1, 1],
                  [1.0 + 2.0 ** -7 + 2.0 ** -23, 1.0 + 2.0 ** -23, 5.0]], np.float32)
    lay = oracle.layout(idx, 5, 1, 1)
    row_expert = np.searchsorted(lay.expert_off[1:], np.arange(lay.total_rows), side="right")
    y = oracle.bf16_round(np.repeat(vals[row_expert][:, None], 8, axis=1))
    got, exp = combine_case(oracle, y, w, idx, 5, 1, B=1)
    f = oracle.bf16_to_f32(got)[:, 0]
    assert f[0] == 0.0 and f[1] == 1.0 and f[2] == np.float32(2.0 ** -30)


def test_combine_identity_returns_x(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    w = make_workload("tiny", 2)
    h = _handle(w.T, w.k, w.E, w.R)
    ep.ep_layout(h, torch.from_numpy(w.topk_idx).to(DEV))
    recv, _ = ep.ep_dispatch(h, bits_to_bf16(w.x_bits), "bf16")
    out = ep.ep_combine(h, recv, torch.from_numpy(w.topk_weights).to(DEV))
    ep.ep_handle_check(h)
    got = oracle.bf16_to_f32(bf16_to_bits(out)).astype(np.float64)
    x = oracle.bf16_to_f32(w.x_bits).astype(np.float64)
    ulp = np.ldexp(1.0, np.frexp(np.abs(x))[1] - 8)
    assert np.all(np.abs(got - x) <= ulp)


def test_non_default_stream(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    w = make_workload("decode", 3)
    s = torch.cuda.Stream(device=DEV)
    with torch.cuda.stream(s):
        h = _handle(w.T, w.k, w.E, w.R)
        x = bits_to_bf16(w.x_bits)
        idx = torch.from_numpy(w.topk_idx).to(DEV)
        ep.ep_layout(h, idx)
        recv, sc = ep.ep_dispatch(h, x, "fp8")
    s.synchronize()
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    exp_q, exp_s = oracle.dispatch_fp8(w.x_bits, lay.dst_row, lay.total_rows)
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], exp_q[rows])
    assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), exp_s[rows].view(np.uint32))


@pytest.mark.parametrize("fmt", ["fp8", "fp8_mn"])
def test_dispatch_fp8_receive_rows_16_byte_aligned(oracle, fmt):
    """A receive buffer that is 16- but not 32-byte aligned (the API's
    minimum): codes and scales bit-exact, nothing written outside it."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16

    rng = np.random.default_rng(29)
    T, H, E, R, k = 90, 1024, 32, 8, 8
    x_bits = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, R)
    P = lay.total_rows
    cap = (P + 3) // 4 * 4
    h = _handle(T, k, E, R)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    raw = torch.full((cap * H + 32,), SENTINEL, dtype=torch.uint8, device=DEV)
    recv = raw[16:16 + cap * H].view(cap, H).view(torch.float8_e4m3fn)
    assert recv.data_ptr() % 32 == 16
    rows = lay.dst_row[lay.dst_row >= 0]
    if fmt == "fp8":
        sc = torch.empty((cap, H // 128), dtype=torch.float32, device=DEV)
        ep.ep_dispatch(h, bits_to_bf16(x_bits), "fp8", recv_x=recv, recv_scales=sc)
        q_ref, s_ref = oracle.dispatch_fp8(x_bits, lay.dst_row, cap)
        assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s_ref[rows].view(np.uint32))
    else:
        sc = torch.empty((H // 128, cap), dtype=torch.float32, device=DEV)
        ep.ep_dispatch(h, bits_to_bf16(x_bits), "fp8_mn", recv_x=recv, recv_scales=sc)
        q_ref, s_ref = oracle.dispatch_fp8_mn(x_bits, lay.dst_row, cap, cap)
        assert np.array_equal(sc.cpu().numpy()[:, rows].view(np.uint32),
                              s_ref[:, rows].view(np.uint32))
    ep.ep_handle_check(h)
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q_ref[rows])
    b = raw.cpu().numpy()
    assert np.all(b[:16] == SENTINEL) and np.all(b[16 + cap * H:] == SENTINEL)
