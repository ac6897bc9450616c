"""GPU parity of the backward entry points against the oracle.

ep_dispatch_backward: bit-exact (fp32 sum in slot order, like combine).
ep_combine_backward: grad_y bit-exact on every used row (one fp32 product,
then bf16); pad rows keep their sentinel; grad_weights within the error bound
of the kernel's own reduction tree -- gamma_n * sum|grad_out * y| with
gamma_n = n u / (1 - n u), u = 2^-24 and n the roundings on the longest path
from a product to the result (each lane's chain of fused multiply-adds, the
xor-shuffle tree, and for the 16-byte kernel the sum over warps) -- plus the
oracle's one rounding of its fp64 dot product, and bitwise repeatable.  At
H = 7168 that is n = 229, tight enough that one dropped 16-channel vector
(an error of about N(0, 16) against a bound near 0.06) fails the check.
"""
import numpy as np
import pytest
import torch

from gpu_util import grad_w_bound
from workloads import make_workload, make_x, random_topk

pytestmark = pytest.mark.gpu


def _setup(idx, E, R, B=128):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV

    T, k = idx.shape
    h = ep.ep_handle_create(max(T, 1), k, E, R, B, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    return h


@pytest.mark.parametrize("T,H,E,R,k,p_unused", [
    (1, 8, 4, 2, 2, 0.0),
    (200, 1032, 32, 8, 8, 0.1),     # 129 vectors: a ragged unit
    (64, 7168, 256, 8, 8, 0.0),
    (50, 512, 64, 8, 20, 0.2),      # k > 8: the general path
])
def test_dispatch_backward_bit_exact(oracle, T, H, E, R, k, p_unused):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import bf16_to_bits, bits_to_bf16

    rng = np.random.default_rng(T + H + k)
    idx, _ = random_topk(T, E, k, rng, p_unused=p_unused)
    lay = oracle.layout(idx, E, R)
    g = make_x(max(lay.total_rows, 1), H, rng)
    h = _setup(idx, E, R)
    gx = ep.ep_dispatch_backward(h, bits_to_bf16(g))
    ep.ep_handle_check(h)
    assert np.array_equal(bf16_to_bits(gx), oracle.dispatch_backward(g, lay.dst_row))


def _combine_backward_case(oracle, idx, E, R, H, rng, w=None):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    T, k = idx.shape
    lay = oracle.layout(idx, E, R)
    P = lay.total_rows
    y = make_x(max(P, 1), H, rng)
    g = make_x(T, H, rng)
    if w is None:
        w = rng.random((T, k)).astype(np.float32)
    h = _setup(idx, E, R)
    gy_dev = torch.full((max(P, 1), H), 0, dtype=torch.int16, device=DEV)
    gy_dev.fill_(0x5A5A)
    gy_dev = gy_dev.view(torch.bfloat16)
    gy, gw = ep.ep_combine_backward(h, bits_to_bf16(g), bits_to_bf16(y),
                                    torch.from_numpy(w).to(DEV), grad_y=gy_dev)
    ep.ep_handle_check(h)
    gy_ref, gw_ref = oracle.combine_backward(g, y, w, lay.dst_row)
    got = bf16_to_bits(gy)
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(got[rows], gy_ref[rows])
    pad = np.setdiff1d(np.arange(P), rows)
    assert np.all(got[pad] == 0x5A5A), "a pad row of grad_y was written"
    gw_got = gw.cpu().numpy()
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    gf = oracle.bf16_to_f32(g).astype(np.float64)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d < 0:
                assert gw_got[t, j] == 0.0
                continue
            bound = grad_w_bound(H, float(np.abs(gf[t] * yf[d]).sum()), float(gw_ref[t, j]))
            assert abs(float(gw_got[t, j]) - float(gw_ref[t, j])) <= bound + 1e-30, (t, j)
    # bitwise repeatable
    _, gw2 = ep.ep_combine_backward(h, bits_to_bf16(g), bits_to_bf16(y),
                                    torch.from_numpy(w).to(DEV))
    assert np.array_equal(gw2.cpu().numpy().view(np.uint32), gw_got.view(np.uint32))
    return gw_got, gw_ref


@pytest.mark.parametrize("T,H,E,R,k,p_unused", [
    (1, 8, 4, 2, 2, 0.0),
    (120, 1032, 32, 8, 8, 0.1),
    (48, 7168, 256, 8, 8, 0.0),
    (40, 2048, 64, 8, 20, 0.2),      # k > 8: slots in batches of 8
    (30, 64, 16, 4, 1, 0.0),
])
def test_combine_backward(oracle, T, H, E, R, k, p_unused):
    rng = np.random.default_rng(3 * T + H + k)
    idx, _ = random_topk(T, E, k, rng, p_unused=p_unused)
    _combine_backward_case(oracle, idx, E, R, H, rng)


def test_combine_backward_full_dsv3_shape(oracle):
    w = make_workload("dsv3", 0, T=512)
    rng = np.random.default_rng(77)
    gw, ref = _combine_backward_case(oracle, w.topk_idx, w.E, w.R, w.H, rng, w.topk_weights)
    # typical error is far inside the worst-case bound
    rel = np.abs(gw - ref) / np.maximum(np.abs(ref), 1e-6)
    assert np.median(rel) < 1e-5


def _f16(bits):
    from gpu_util import DEV

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).to(DEV)


def _f16_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("T,H,E,R,k,p_unused", [
    (200, 1032, 32, 8, 8, 0.1),     # 16-byte rows: the fallback kernels
    (64, 7168, 256, 8, 8, 0.0),     # 32-byte rows
    (40, 2048, 64, 8, 20, 0.2),     # k > 8: slots in batches of 8
])
def test_backward_fp16(oracle, T, H, E, R, k, p_unused):
    """fp16 rows: dispatch backward bit-exact; combine backward grad_y
    bit-exact, grad_w within the reduction tree's bound of the fp64 dot."""
    import combine_ep_layout_08_b200 as ep
    from workloads import make_x_fp16

    rng = np.random.default_rng(5 * T + H + k)
    idx, w = random_topk(T, E, k, rng, p_unused=p_unused)
    lay = oracle.layout(idx, E, R)
    P = max(lay.total_rows, 1)
    h = _setup(idx, E, R)
    g = make_x_fp16(P, H, rng)
    gx = ep.ep_dispatch_backward(h, _f16(g))
    ep.ep_handle_check(h)
    assert gx.dtype == torch.float16
    assert np.array_equal(_f16_bits(gx), oracle.dispatch_backward(g, lay.dst_row, dtype="fp16"))

    y = make_x_fp16(P, H, rng)
    go = make_x_fp16(T, H, rng)
    from gpu_util import DEV

    gy, gw = ep.ep_combine_backward(h, _f16(go), _f16(y), torch.from_numpy(w).to(DEV))
    ep.ep_handle_check(h)
    gy_ref, gw_ref = oracle.combine_backward(go, y, w, lay.dst_row, dtype="fp16")
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(_f16_bits(gy)[rows], gy_ref[rows])
    gwg = gw.cpu().numpy()
    yf = oracle.fp16_to_f32(y).astype(np.float64)
    gf = oracle.fp16_to_f32(go).astype(np.float64)
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d < 0:
                assert gwg[t, j] == 0.0
                continue
            bound = grad_w_bound(H, float(np.abs(gf[t] * yf[d]).sum()), float(gw_ref[t, j]))
            assert abs(float(gwg[t, j]) - float(gw_ref[t, j])) <= bound + 1e-30, (t, j)
