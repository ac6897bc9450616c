"""GPU parity of the FP16-input paths against the oracle: the fp16 row copy
(ep_dispatch / ep_layout_dispatch / ep_dispatch_range with the fp16 format),
FP8 e4m3 1x128 quantisation of fp16 rows (ep_dispatch_ex, row-major and
MN-major scales, 32-byte and 16-byte kernels), and combine of fp16 expert
outputs (ep_combine_ex).

Bars: copies, FP8 bytes and scales bit-exact on every used row; combine
bit-exact (the fp32 fused multiply-add chain in slot order, then binary16
round-to-nearest-even, the oracle's own order); pad rows and guard bands
keep their sentinels; mismatched type and format are rejected.
"""
import numpy as np
import pytest
import torch

from workloads import make_x_fp16, make_x_scale_sweep, random_topk

pytestmark = pytest.mark.gpu

SENTINEL = 0x5A


def _f16(bits, device="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).to(device)


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _guarded(rows, cols, dtype, guard=4):
    esize = torch.empty((), dtype=dtype).element_size()
    raw = torch.full(((rows + 2 * guard) * cols * esize,), SENTINEL, dtype=torch.uint8,
                     device="cuda:0")
    full = raw.view(dtype).view(rows + 2 * guard, cols)
    return full, full[guard:guard + rows]


def _guards_ok(full, guard=4):
    b = full.view(torch.uint8).view(full.shape[0], -1)
    return bool((b[:guard] == SENTINEL).all()) and bool((b[-guard:] == SENTINEL).all())


def _setup(oracle, T, H, E, R, k, seed, p_unused=0.1, x_bits=None):
    import combine_ep_layout_08_b200 as ep

    rng = np.random.default_rng(seed)
    x = make_x_fp16(T, H, rng) if x_bits is None else x_bits
    idx, w = random_topk(T, E, k, rng, p_unused=p_unused)
    lay = oracle.layout(idx, E, R)
    h = ep.ep_handle_create(max(T, 1), k, E, R, device="cuda:0")
    ep.ep_layout(h, torch.from_numpy(idx).to("cuda:0"))
    return h, lay, x, idx, w, rng


@pytest.mark.parametrize("T,H,E,R,k", [(1, 8, 4, 2, 2), (77, 1032, 32, 8, 8), (64, 7168, 256, 8, 8)])
def test_fp16_copy_dispatch(oracle, T, H, E, R, k):
    import combine_ep_layout_08_b200 as ep

    h, lay, x, idx, _, _ = _setup(oracle, T, H, E, R, k, T + H)
    P = lay.total_rows
    full, recv = _guarded(P, H, torch.float16)
    ep.ep_dispatch(h, _f16(x), "fp16", recv_x=recv)
    ep.ep_handle_check(h)
    rows = lay.dst_row[lay.dst_row >= 0]
    exp = oracle.dispatch_bf16(x, lay.dst_row, P)    # a 16-bit row copy, whatever the type
    got = _bits(recv)
    assert np.array_equal(got[rows], exp[rows])
    pad = np.nonzero(lay.recv_src < 0)[0]
    assert np.all(recv.view(torch.uint8).view(P, -1).cpu().numpy()[pad] == SENTINEL)
    assert _guards_ok(full)


def test_fp16_copy_fused_and_ranges(oracle):
    import combine_ep_layout_08_b200 as ep

    T, H, E, R, k = 128, 2048, 256, 16, 8
    rng = np.random.default_rng(5)
    x = make_x_fp16(T, H, rng)
    idx, _ = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, R)
    exp = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)
    rows = lay.dst_row[lay.dst_row >= 0]
    h = ep.ep_handle_create(T, k, E, R, device="cuda:0")
    recv, _ = ep.ep_layout_dispatch(h, torch.from_numpy(idx).to("cuda:0"), _f16(x), "fp16")
    ep.ep_handle_check(h)
    assert recv.dtype == torch.float16
    assert np.array_equal(_bits(recv)[rows], exp[rows])
    recv2 = torch.zeros_like(recv)
    xd = _f16(x)
    for t0 in range(0, T, 40):
        ep.ep_dispatch_range(h, t0, xd[t0:t0 + 40].contiguous(), "fp16", recv2)
    ep.ep_handle_check(h)
    assert np.array_equal(_bits(recv2)[rows], exp[rows])


@pytest.mark.parametrize("fmt", ["fp8", "fp8_mn"])
@pytest.mark.parametrize("T,H,E,R,k,x_offset", [
    (1, 128, 4, 2, 2, 0),
    (45, 384, 16, 4, 3, 0),       # 3 blocks: a partial unit
    (70, 7168, 256, 8, 8, 0),
    (40, 1024, 32, 8, 8, 8),      # 16-byte aligned x: the 16-byte kernel
])
def test_fp8_of_fp16_rows(oracle, fmt, T, H, E, R, k, x_offset):
    import combine_ep_layout_08_b200 as ep

    h, lay, x, idx, _, _ = _setup(oracle, T, H, E, R, k, 3 * T + H)
    P = lay.total_rows
    if x_offset:
        base = torch.empty(T * H + x_offset, dtype=torch.float16, device="cuda:0")
        xd = base[x_offset:].view(T, H)
        xd.copy_(_f16(x))
        assert xd.data_ptr() % 32 != 0
    else:
        xd = _f16(x)
    rows = lay.dst_row[lay.dst_row >= 0]
    if fmt == "fp8":
        full, recv = _guarded(P, H, torch.float8_e4m3fn)
        sfull, sc = _guarded(P, H // 128, torch.float32)
        ep.ep_dispatch(h, xd, "fp8", recv_x=recv, recv_scales=sc)
        ep.ep_handle_check(h)
        q_ref, s_ref = oracle.dispatch_fp8(x, lay.dst_row, P, dtype="fp16")
        assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s_ref[rows].view(np.uint32))
        assert _guards_ok(sfull)
    else:
        cap = (P + 3) // 4 * 4
        full, recv = _guarded(cap, H, torch.float8_e4m3fn)
        sc = torch.full((H // 128, cap), float("nan"), dtype=torch.float32, device="cuda:0")
        ep.ep_dispatch(h, xd, "fp8_mn", recv_x=recv, recv_scales=sc)
        ep.ep_handle_check(h)
        q_ref, s_ref = oracle.dispatch_fp8_mn(x, lay.dst_row, cap, cap, dtype="fp16")
        assert np.array_equal(sc.cpu().numpy()[:, rows].view(np.uint32),
                              s_ref[:, rows].view(np.uint32))
    got = recv.view(torch.uint8).cpu().numpy()
    assert np.array_equal(got[rows], q_ref[rows])
    assert _guards_ok(full)


@pytest.mark.parametrize("x_offset", [0, 8])  # the 32-byte and the 16-byte kernels
def test_fp8_of_fp16_scale_sweep(oracle, x_offset):
    """Block maxima over every binade of binary16 (all of them take the
    corrected-reciprocal division): codes and scales bit-exact."""
    import combine_ep_layout_08_b200 as ep

    T, H, E, R, k = 256, 7168, 16, 4, 2
    x = make_x_scale_sweep(T, H, np.random.default_rng(99 + x_offset), fmt="fp16")
    h, lay, x, idx, _, _ = _setup(oracle, T, H, E, R, k, 5, p_unused=0.0, x_bits=x)
    P = lay.total_rows
    if x_offset:
        base = torch.empty(T * H + x_offset, dtype=torch.float16, device="cuda:0")
        xd = base[x_offset:].view(T, H)
        xd.copy_(_f16(x))
    else:
        xd = _f16(x)
    rows = lay.dst_row[lay.dst_row >= 0]
    full, recv = _guarded(P, H, torch.float8_e4m3fn)
    sfull, sc = _guarded(P, H // 128, torch.float32)
    ep.ep_dispatch(h, xd, "fp8", recv_x=recv, recv_scales=sc)
    ep.ep_handle_check(h)
    q_ref, s_ref = oracle.dispatch_fp8(x, lay.dst_row, P, dtype="fp16")
    assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s_ref[rows].view(np.uint32))
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q_ref[rows])
    assert _guards_ok(full) and _guards_ok(sfull)


def test_fp8_of_fp16_special_values(oracle):
    T, H, E, R, k = 12, 1024, 16, 4, 2
    rng = np.random.default_rng(91)
    xf = rng.standard_normal((T, H)).astype(np.float32)
    xf[0, :128] = 0.0                        # amax = 0
    xf[1, :128] = -0.0
    xf[2, :] *= 2.0 ** -18                   # fp16 subnormal inputs
    xf[3, :128] = 0.0
    xf[3, 7] = 2.0 ** -24                    # smallest fp16 subnormal as amax
    xf[4, :] = np.clip(xf[4, :] * 30000.0, -65504.0, 65504.0)   # near the top of fp16
    xf[5, :128] = 65504.0
    xf[6, ::2] = 0.0
    xf[7, :] = np.round(xf[7, :] * 4) / 4
    with np.errstate(over="ignore"):
        x = xf.astype(np.float16).view(np.uint16)
    import combine_ep_layout_08_b200 as ep

    h, lay, _, idx, _, _ = _setup(oracle, T, H, E, R, k, 92, p_unused=0.0, x_bits=x)
    P = lay.total_rows
    recv, sc = ep.ep_dispatch(h, _f16(x), "fp8")
    ep.ep_handle_check(h)
    q_ref, s_ref = oracle.dispatch_fp8(x, lay.dst_row, P, dtype="fp16")
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q_ref[rows])
    assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s_ref[rows].view(np.uint32))


@pytest.mark.parametrize("T,H,E,R,k,p_unused", [
    (1, 8, 4, 2, 2, 0.0),
    (100, 1032, 32, 8, 8, 0.1),    # 129 vectors: ragged unit, some unused slots
    (64, 7168, 256, 8, 8, 0.0),
    (30, 512, 64, 8, 20, 0.2),     # k > 8: the general path
])
def test_combine_fp16_bit_exact(oracle, T, H, E, R, k, p_unused):
    import combine_ep_layout_08_b200 as ep

    h, lay, _, idx, w, rng = _setup(oracle, T, H, E, R, k, 7 * T + k, p_unused=p_unused)
    y = make_x_fp16(max(lay.total_rows, 1), H, rng)
    out = ep.ep_combine(h, _f16(y), torch.from_numpy(w).to("cuda:0"))
    ep.ep_handle_check(h)
    assert out.dtype == torch.float16
    assert np.array_equal(_bits(out), oracle.combine(y, w, lay.dst_row, dtype="fp16"))


def test_combine_fp16_overflow_to_infinity(oracle):
    import combine_ep_layout_08_b200 as ep

    T, H, E, R, k = 8, 64, 4, 2, 2
    idx = np.array([[0, 1]] * T, np.int64)
    lay = oracle.layout(idx, E, R)
    y = np.full((lay.total_rows, H), np.float16(60000.0).view(np.uint16), np.uint16)
    w = np.ones((T, k), np.float32)
    h = ep.ep_handle_create(T, k, E, R, device="cuda:0")
    ep.ep_layout(h, torch.from_numpy(idx).to("cuda:0"))
    out = ep.ep_combine(h, _f16(y), torch.from_numpy(w).to("cuda:0"))
    ep.ep_handle_check(h)
    ref = oracle.combine(y, w, lay.dst_row, dtype="fp16")
    assert np.array_equal(_bits(out), ref) and np.all(ref == 0x7C00)


def test_type_and_format_mismatch_rejected(oracle):
    import combine_ep_layout_08_b200 as ep

    h, lay, x, idx, w, _ = _setup(oracle, 16, 256, 8, 2, 2, 1)
    with pytest.raises(ep.EPError):
        ep.ep_dispatch(h, _f16(x), "bf16")          # fp16 rows as a bf16 copy
    xb = _f16(x).view(torch.bfloat16)
    with pytest.raises(ep.EPError):
        ep.ep_dispatch(h, xb, "fp16")               # bf16 rows as an fp16 copy
    with pytest.raises(ep.EPError):
        ep.ep_layout_dispatch(h, torch.from_numpy(idx).to("cuda:0"), _f16(x), "fp8")
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
