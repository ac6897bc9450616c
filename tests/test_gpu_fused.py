"""The fused low-latency path ep_layout_dispatch: the same layout and receive
buffers as ep_layout + ep_dispatch, bit-exact against the oracle, on the
one-launch path (small batches, 32-byte rows) and on the fallback path."""
import numpy as np
import pytest
import torch

from workloads import make_workload, make_x, make_x_scale_sweep, random_topk

pytestmark = pytest.mark.gpu
SENT = 0x5A


def fused_case(oracle, x_bits, idx, E, R, fmt, B=128):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, assert_layout_equal, bits_to_bf16, gpu_layout

    T, H = x_bits.shape
    k = idx.shape[1]
    lay = oracle.layout(idx, E, R, B)
    P = lay.total_rows
    cap = (P + 8 + 3) // 4 * 4
    h = ep.ep_handle_create(max(T, 1), k, E, R, B, device=DEV)
    x = bits_to_bf16(x_bits)
    if fmt == "bf16":
        recv = torch.full((cap * H * 2,), SENT, dtype=torch.uint8, device=DEV)
        recv = recv.view(torch.bfloat16).view(cap, H)
        sc = None
    else:
        recv = torch.full((cap, H), SENT, dtype=torch.uint8, device=DEV).view(torch.float8_e4m3fn)
        shape = (cap, H // 128) if fmt == "fp8" else (H // 128, cap)
        sc = torch.full((cap * (H // 128) * 4,), SENT, dtype=torch.uint8, device=DEV)
        sc = sc.view(torch.float32).view(*shape)
    ep.ep_layout_dispatch(h, torch.from_numpy(idx).to(DEV), x, fmt, recv_x=recv, recv_scales=sc)
    ep.ep_handle_check(h)
    assert_layout_equal(gpu_layout(h), lay)
    rows = lay.dst_row[lay.dst_row >= 0]
    pad = np.setdiff1d(np.arange(cap), rows)
    if fmt == "bf16":
        got = recv.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got[rows], oracle.dispatch_bf16(x_bits, lay.dst_row, P)[rows])
    elif fmt == "fp8":
        q, s = oracle.dispatch_fp8(x_bits, lay.dst_row, P)
        assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q[rows])
        assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s[rows].view(np.uint32))
    else:
        q, s = oracle.dispatch_fp8_mn(x_bits, lay.dst_row, P, cap)
        assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q[rows])
        assert np.array_equal(sc.cpu().numpy()[:, rows].view(np.uint32), s[:, rows].view(np.uint32))
    b = recv.view(torch.uint8).view(cap, -1).cpu().numpy()
    assert np.all(b[pad] == SENT), "a row outside the used rows was written"
    return h


@pytest.mark.parametrize("name,seed", [("decode", 0), ("decode", 3), ("tiny", 1)])
def test_fused_configs(oracle, name, seed):
    w = make_workload(name, seed)
    fused_case(oracle, w.x_bits, w.topk_idx, w.E, w.R, w.fmt)


@pytest.mark.parametrize("T,H,E,R,k,fmt,p_unused", [
    (1, 16, 4, 2, 2, "bf16", 0.0),
    (37, 1040, 32, 8, 8, "bf16", 0.1),    # 65 vectors: ragged unit
    (512, 2048, 256, 16, 8, "fp8", 0.0),  # 4096 entries: the one-launch limit
    (100, 384, 16, 4, 3, "fp8_mn", 0.1),
    (130, 7168, 1024, 64, 8, "fp8", 0.0), # E = 1024
    (600, 256, 64, 8, 8, "bf16", 0.0),    # 4800 entries: two launches
    (40, 264, 16, 4, 2, "bf16", 0.0),     # H % 16 != 0: two launches
    (148, 1024, 256, 16, 8, "fp8", 0.05), # one CTA per token on every SM
    (60, 512, 64, 8, 32, "bf16", 0.1),    # k = 32 slots per token
    (149, 1024, 256, 16, 8, "bf16", 0.0), # one token more than SMs: the replicated layout
    (100, 512, 256, 64, 8, "fp8", 0.1),   # one CTA per token, R > 32 ranks
    (90, 512, 32, 32, 5, "bf16", 0.0),    # one CTA per token, R = E = 32, k not dividing 32
])
def test_fused_shapes(oracle, T, H, E, R, k, fmt, p_unused):
    rng = np.random.default_rng(T * 7 + H)
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, p_unused=p_unused)
    fused_case(oracle, x, idx, E, R, fmt)


@pytest.mark.parametrize("T,H", [(128, 7168),   # one CTA per token (decode kernel)
                                 (300, 2048)])  # the replicated-layout kernel
def test_fused_fp8_scale_sweep(oracle, T, H):
    rng = np.random.default_rng(T + H)
    x = make_x_scale_sweep(T, H, rng)
    idx, _ = random_topk(T, 256, 8, rng)
    fused_case(oracle, x, idx, 256, 16, "fp8")


def _decode_shapes(n, seed):
    """Batches that take the one-CTA-per-token kernel (T <= 148, E <= 512):
    duplicate experts in a token, unused slots, k up to 32, R above and
    below 32, block_m not a power of two."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        E = int(rng.choice([1, 2, 5, 16, 64, 100, 256, 320, 512]))
        R = int(rng.choice([r for r in range(1, min(E, 64) + 1) if E % r == 0]))
        k = int(rng.choice([1, 2, 3, 6, 8, 13, 32]))
        T = int(rng.integers(1, 149))
        B = int(rng.choice([1, 7, 64, 128]))
        distinct = bool(rng.random() < 0.5) and k <= E
        p_unused = float(rng.choice([0.0, 0.2]))
        fmt = str(rng.choice(["bf16", "fp8"]))
        H = int(rng.choice([128, 1024, 7168]))
        out.append((T, H, E, R, k, B, distinct, p_unused, fmt))
    return out


@pytest.mark.parametrize("T,H,E,R,k,B,distinct,p_unused,fmt", _decode_shapes(24, 31337))
def test_fused_decode_kernel_random_shapes(oracle, T, H, E, R, k, B, distinct, p_unused, fmt):
    rng = np.random.default_rng(T * 13 + E * 3 + k)
    x = make_x(T, H, rng)
    idx, _ = random_topk(T, E, k, rng, distinct=distinct, p_unused=p_unused)
    fused_case(oracle, x, idx, E, R, fmt, B=B)


def test_fused_errors(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16

    rng = np.random.default_rng(1)
    x = make_x(64, 256, rng)
    idx, _ = random_topk(64, 16, 4, rng)
    idx[5, 2] = 99
    h = ep.ep_handle_create(64, 4, 16, 4, device=DEV)
    ep.ep_layout_dispatch(h, torch.from_numpy(idx).to(DEV), bits_to_bf16(x), "bf16")
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_BAD_INDEX
    idx[5, 2] = 3
    lay = oracle.layout(idx, 16, 4)
    small = torch.empty((lay.total_rows // 2, 256), dtype=torch.bfloat16, device=DEV)
    ep.ep_layout_dispatch(h, torch.from_numpy(idx).to(DEV), bits_to_bf16(x), "bf16", recv_x=small)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY


def test_fused_under_cuda_graph(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    w = make_workload("decode", 2)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, device=DEV)
    x = bits_to_bf16(w.x_bits)
    idx = torch.from_numpy(w.topk_idx).to(DEV)
    wt = torch.from_numpy(w.topk_weights).to(DEV)
    cap = ep.ep_recv_rows_upper_bound(w.T, w.k, w.E)
    recv = torch.empty((cap, w.H), dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty((cap, w.H // 128), dtype=torch.float32, device=DEV)
    y = bits_to_bf16(make_x(cap, w.H, np.random.default_rng(9)))
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=DEV)

    def step():
        ep.ep_layout_dispatch(h, idx, x, "fp8", recv_x=recv, recv_scales=sc)
        ep.ep_combine(h, y, wt, out=out)

    s = torch.cuda.Stream(device=DEV)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    recv.view(torch.uint8).zero_()
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    rows = lay.dst_row[lay.dst_row >= 0]
    q, _ = oracle.dispatch_fp8(w.x_bits, lay.dst_row, lay.total_rows)
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q[rows])
    assert np.array_equal(bf16_to_bits(out), oracle.combine(bf16_to_bits(y), w.topk_weights,
                                                            lay.dst_row))
    del g
