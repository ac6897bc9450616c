"""GPU parity of the GEMM-ready receive-layout helpers against the oracle:
MN-major FP8 scales (both FP8 kernels), the per-row weight scatter, and
zeroing of pad rows (16-byte and byte paths)."""
import numpy as np
import pytest
import torch

from workloads import make_workload, make_x, random_topk

pytestmark = pytest.mark.gpu

SENT = 0x5A


def _handle(idx, E, R, B=128):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV

    T, k = idx.shape
    h = ep.ep_handle_create(max(T, 1), k, E, R, B, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    return h


@pytest.mark.parametrize("T,H,E,R,k,x_offset", [
    (100, 7168, 256, 8, 8, 0),
    (57, 384, 16, 4, 3, 0),
    (64, 1024, 32, 8, 8, 8),     # 16-byte aligned x: the 16-byte kernel
])
def test_fp8_mn_major_scales(oracle, T, H, E, R, k, x_offset):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16

    rng = np.random.default_rng(T + H)
    x_bits = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=0.1)
    lay = oracle.layout(idx, E, R)
    P = lay.total_rows
    cap = (P + 4 + 3) // 4 * 4
    h = _handle(idx, E, R)
    base = torch.empty(T * H + x_offset, dtype=torch.bfloat16, device=DEV)
    x = base[x_offset:].view(T, H)
    x.copy_(bits_to_bf16(x_bits))
    recv = torch.full((cap, H), SENT, dtype=torch.uint8, device=DEV).view(torch.float8_e4m3fn)
    sc = torch.full((H // 128 * cap * 4,), SENT, dtype=torch.uint8, device=DEV).view(torch.float32)
    sc = sc.view(H // 128, cap)
    ep.ep_dispatch(h, x, "fp8_mn", recv_x=recv, recv_scales=sc)
    ep.ep_handle_check(h)
    q_ref, s_ref = oracle.dispatch_fp8_mn(x_bits, lay.dst_row, P, cap)
    rows = lay.dst_row[lay.dst_row >= 0]
    got_q = recv.view(torch.uint8).cpu().numpy()
    got_s = sc.cpu().numpy()
    assert np.array_equal(got_q[rows], q_ref[rows])
    assert np.array_equal(got_s[:, rows].view(np.uint32), s_ref[:, rows].view(np.uint32))
    others = np.setdiff1d(np.arange(cap), rows)
    assert np.all(np.ascontiguousarray(got_s[:, others]).view(np.uint8) == SENT), \
        "an MN scale outside the used rows"


def test_fp8_mn_requires_capacity_multiple_of_4(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16

    w = make_workload("decode", 0, H=256)
    h = _handle(w.topk_idx, w.E, w.R)
    recv = torch.empty((4094, 256), dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty((2, 4094), dtype=torch.float32, device=DEV)
    with pytest.raises(ep.EPError):
        ep.ep_dispatch(h, bits_to_bf16(w.x_bits), "fp8_mn", recv_x=recv, recv_scales=sc)


def test_dispatch_weights_scatter(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV

    rng = np.random.default_rng(5)
    T, E, R, k = 3000, 256, 8, 8
    idx, w = random_topk(T, E, k, rng, p_unused=0.05)
    lay = oracle.layout(idx, E, R)
    h = _handle(idx, E, R)
    cap = lay.total_rows + 3
    rw = torch.full((cap,), -7.0, dtype=torch.float32, device=DEV)
    ep.ep_dispatch_weights(h, torch.from_numpy(w).to(DEV), rw)
    ep.ep_handle_check(h)
    ref = oracle.dispatch_weights(w, lay.dst_row, cap, fill=-7.0)
    assert np.array_equal(rw.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    small = torch.zeros(lay.total_rows // 2, dtype=torch.float32, device=DEV)
    ep.ep_dispatch_weights(h, torch.from_numpy(w).to(DEV), small)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY


@pytest.mark.parametrize("shape,dtype", [
    ((7168,), torch.bfloat16),     # recv_x rows: 16-byte stores
    ((56,), torch.float32),        # row-major scales at H = 7168: 224 bytes
    ((3,), torch.float32),         # 12-byte rows: byte stores
    ((3,), torch.uint8),
])
def test_zero_pad_rows(oracle, shape, dtype):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV

    w = make_workload("decode", 1, H=128)   # ~97 % pad rows
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    h = _handle(w.topk_idx, w.E, w.R)
    P = lay.total_rows
    esize = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape))
    raw = torch.full((P * n * esize,), SENT, dtype=torch.uint8, device=DEV)
    rows = raw.view(dtype).view(P, *shape)
    ep.ep_zero_pad_rows(h, rows)
    ep.ep_handle_check(h)
    got = raw.view(P, n * esize).cpu().numpy()
    ref = oracle.zero_pad_rows(lay.recv_src, np.full((P, n * esize), SENT, np.uint8))
    assert np.array_equal(got, ref)
