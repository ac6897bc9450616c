"""The whole path on the GPU -- layout -> dispatch -> stand-in expert ->
combine -- against the oracle's whole path, on all five configs at their full
sizes (the launch configuration the benchmark times), under CUDA-graph
replay, and run twice for determinism."""
import numpy as np
import pytest
import torch

from workloads import make_workload

pytestmark = pytest.mark.gpu


def gpu_pipeline(w, h=None):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bits_to_bf16, expert_op_torch

    if h is None:
        h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=DEV)
    x = bits_to_bf16(w.x_bits)
    idx = torch.from_numpy(w.topk_idx).to(DEV)
    wt = torch.from_numpy(w.topk_weights).to(DEV)
    c = torch.from_numpy(w.expert_c).to(DEV)
    ep.ep_layout(h, idx)
    recv, scales = ep.ep_dispatch(h, x, w.fmt)
    P = int(ep.ep_handle_view(h, "total_recv_rows").item())
    y = expert_op_torch(recv, scales, ep.ep_handle_view(h, "expert_off"), c, P)
    out = ep.ep_combine(h, y, wt)
    ep.ep_handle_check(h)
    return h, recv, scales, y, out, P


@pytest.mark.parametrize("name", ["tiny", "decode", "dsv3", "8k", "skewed"])
def test_full_config_pipeline(oracle, name):
    from gpu_util import assert_layout_equal, bf16_to_bits, bf16_ulp_diff, gpu_layout

    w = make_workload(name, 0)
    h, recv, scales, y, out, P = gpu_pipeline(w)
    ref = oracle.pipeline(w.x_bits, w.topk_idx, w.topk_weights, w.E, w.R, w.fmt, w.expert_c)
    lay = ref["layout"]
    assert_layout_equal(gpu_layout(h), lay)
    rows = lay.dst_row[lay.dst_row >= 0]
    if w.fmt == "bf16":
        got = recv[:P].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got[rows], ref["recv"][rows])
    else:
        got = recv[:P].view(torch.uint8).cpu().numpy()
        assert np.array_equal(got[rows], ref["recv"][rows])
        gs = scales[:P].cpu().numpy()
        assert np.array_equal(gs[rows].view(np.uint32), ref["scales"][rows].view(np.uint32))
    # the stand-in expert sees identical inputs, so y must match bit for bit
    gy = bf16_to_bits(y[:P])
    assert np.array_equal(gy[rows], ref["y"][rows])
    go = bf16_to_bits(out)
    d = bf16_ulp_diff(go, ref["out"])
    assert d.max() <= 1
    assert (go == ref["out"]).mean() == 1.0


@pytest.mark.parametrize("name", ["decode", "dsv3"])  # one-CTA and cooperative layouts
def test_cuda_graph_replay_matches_eager(oracle, name):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16

    w = make_workload(name, 0, H=1024)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, device=DEV)
    x = bits_to_bf16(w.x_bits)
    idx = torch.from_numpy(w.topk_idx).to(DEV)
    wt = torch.from_numpy(w.topk_weights).to(DEV)
    cap = ep.ep_recv_rows_upper_bound(w.T, w.k, w.E)
    recv = torch.empty((cap, w.H), dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty((cap, w.H // 128), dtype=torch.float32, device=DEV)
    from workloads import make_x

    y = bits_to_bf16(make_x(cap, w.H, np.random.default_rng(1)))
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=DEV)

    def step():
        ep.ep_layout(h, idx)
        ep.ep_dispatch(h, x, "fp8", recv_x=recv, recv_scales=sc)
        ep.ep_combine(h, y, wt, out=out)

    s = torch.cuda.Stream(device=DEV)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside capture (first call zeroes the error word)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager_out = bf16_to_bits(out).copy()
    eager_q = recv.view(torch.uint8).cpu().numpy().copy()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_()
    recv.view(torch.uint8).zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    assert np.array_equal(bf16_to_bits(out), eager_out)
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], eager_q[rows])
    exp = oracle.combine(bf16_to_bits(y), w.topk_weights, lay.dst_row)
    assert np.array_equal(eager_out, exp)
    del g


def test_pipeline_bitwise_deterministic():
    import combine_ep_layout_08_b200 as ep
    from gpu_util import bf16_to_bits

    w = make_workload("skewed", 1, T=2048)
    h, recv1, sc1, _, out1, P = gpu_pipeline(w)
    rows = ep.ep_handle_view(h, "dst_row").cpu().numpy().reshape(-1)
    a = (recv1.view(torch.uint8).cpu().numpy()[rows], sc1.cpu().numpy()[rows], bf16_to_bits(out1))
    _, recv2, sc2, _, out2, _ = gpu_pipeline(w, h)
    b = (recv2.view(torch.uint8).cpu().numpy()[rows], sc2.cpu().numpy()[rows], bf16_to_bits(out2))
    for u, v in zip(a, b):
        assert np.array_equal(u.view(np.uint8), v.view(np.uint8))


@pytest.mark.parametrize("name,T,H", [("8k", 1000, 1024), ("skewed", 2048, 1024)])
def test_token_ranges_match_the_whole_call(oracle, name, T, H):
    """Dispatch and combine of token ranges (uneven, one empty, on two streams)
    write exactly what the whole-batch calls write."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, bf16_to_bits, bits_to_bf16
    from workloads import make_x

    w = make_workload(name, 0, T=T, H=H)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, device=DEV)
    x = bits_to_bf16(w.x_bits)
    wt = torch.from_numpy(w.topk_weights).to(DEV)
    ep.ep_layout(h, torch.from_numpy(w.topk_idx).to(DEV))
    recv_full, sc_full = ep.ep_dispatch(h, x, w.fmt)
    cap = recv_full.shape[0]
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    y = bits_to_bf16(make_x(max(lay.total_rows, 1), H, np.random.default_rng(4)))
    out_full = ep.ep_combine(h, y, wt)
    recv = torch.empty_like(recv_full)
    sc = None if sc_full is None else torch.empty_like(sc_full)
    out = torch.empty_like(out_full)
    cuts = [0, 300, 300, 777, T]
    streams = [torch.cuda.Stream(device=DEV), torch.cuda.Stream(device=DEV)]
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        with torch.cuda.stream(streams[i % 2]):
            ep.ep_dispatch_range(h, a, x[a:b], w.fmt, recv, sc)
            ep.ep_combine_range(h, a, y, wt[a:b], out[a:b])
    torch.cuda.synchronize()
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows],
                          recv_full.view(torch.uint8).cpu().numpy()[rows])
    if sc is not None:
        assert np.array_equal(sc.cpu().numpy()[rows], sc_full.cpu().numpy()[rows])
    assert np.array_equal(bf16_to_bits(out), bf16_to_bits(out_full))
    assert np.array_equal(bf16_to_bits(out_full), oracle.combine(bf16_to_bits(y), w.topk_weights,
                                                                 lay.dst_row))
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_range(h, T - 10, x[:20], w.fmt, recv, sc)   # past the last token
