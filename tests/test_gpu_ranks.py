"""GPU parity of the expert-parallel entry points (ep_dispatch_ranks,
ep_combine_ranks) on one GPU: R source ranks are emulated as token ranges of
the global order, and the R receive buffers are separate allocations (on R
GPUs they would be peer views).  No kernel waits on another.

Expected values come from the oracle's single-buffer path over the global
token order: rank p's buffer must equal rows [rank_off[p], rank_off[p+1]) of
the oracle's receive buffer, and each source's combined rows the oracle's
combine of its tokens.  Bars: bit-exact (copies, FP8 codes and scales,
combine -- the same fma chain in slot order); rows past a rank's block keep
their sentinel; a rank buffer that is too small reports EP_ERR_CAPACITY.
"""
import numpy as np
import pytest
import torch

from gpu_util import grad_w_bound
from workloads import make_x, make_x_fp16, random_topk

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SENT = 0x5A


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _setup(oracle, counts, E, R, k, H, seed, p_unused=0.1):
    import combine_ep_layout_08_b200 as ep

    rng = np.random.default_rng(seed)
    T = sum(counts)
    idx, w = random_topk(T, E, k, rng, p_unused=p_unused)
    x = make_x(T, H, rng)
    lay = oracle.layout(idx, E, R)
    h = ep.ep_handle_create(max(T, 1), k, E, R, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(int)
    return h, lay, idx, w, x, rng, starts


def _rank_rows(lay, R):
    return [(int(lay.rank_off[p]), int(lay.rank_off[p + 1])) for p in range(R)]


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
@pytest.mark.parametrize("counts,E,R,k,H", [
    ([50, 0, 77, 31], 32, 4, 8, 1024),     # an empty source rank
    ([128] * 8, 256, 8, 8, 7168),          # the decode shape over 8 ranks
    ([40, 41], 16, 2, 3, 2048),
])
def test_dispatch_ranks_matches_the_global_layout(oracle, fmt, counts, E, R, k, H):
    import combine_ep_layout_08_b200 as ep

    h, lay, idx, _, x, _, starts = _setup(oracle, counts, E, R, k, H, sum(counts) + H)
    blocks = _rank_rows(lay, R)
    extra = 5                                          # rows past each block: must stay untouched
    dt = torch.bfloat16 if fmt == "bf16" else torch.float8_e4m3fn
    esz = 2 if fmt == "bf16" else 1
    recv = [torch.full(((b - a + extra) * H * esz,), SENT, dtype=torch.uint8, device=DEV)
            .view(dt).view(b - a + extra, H) for a, b in blocks]
    scales = None
    if fmt == "fp8":
        scales = [torch.full(((b - a + extra) * (H // 128) * 4,), SENT, dtype=torch.uint8,
                             device=DEV).view(torch.float32).view(b - a + extra, H // 128)
                  for a, b in blocks]
    xd = _bf16(x)
    for s, n in zip(starts, counts):                   # each source rank, its own tokens
        ep.ep_dispatch_ranks(h, int(s), xd[s:s + n].contiguous(), fmt, recv, scales)
    ep.ep_handle_check(h)
    if fmt == "bf16":
        ref = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)
    else:
        ref, sref = oracle.dispatch_fp8(x, lay.dst_row, lay.total_rows)
    used = np.zeros(lay.total_rows, bool)
    used[lay.dst_row[lay.dst_row >= 0]] = True
    for p, (a, b) in enumerate(blocks):
        rows = np.nonzero(used[a:b])[0]
        got = recv[p].view(torch.uint8).view(b - a + extra, -1).cpu().numpy()
        exp = ref[a:b].view(np.uint8).reshape(b - a, -1)
        assert np.array_equal(got[rows], exp[rows]), "rank %d" % p
        assert np.all(got[b - a:] == SENT), "rank %d: a row past its block was written" % p
        pad = np.nonzero(~used[a:b])[0]
        assert np.all(got[pad] == SENT), "rank %d: a pad row was written" % p
        if fmt == "fp8":
            gs = scales[p].cpu().numpy()
            assert np.array_equal(gs[rows].view(np.uint32), sref[a:b][rows].view(np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("counts,E,R,k,H", [
    ([50, 0, 77, 31], 32, 4, 8, 1024),
    ([64] * 8, 256, 8, 8, 7168),
    ([30, 33], 16, 2, 12, 264),            # k > 8: two slot batches; a ragged unit
])
def test_combine_ranks_matches_the_global_combine(oracle, dtype, counts, E, R, k, H):
    import combine_ep_layout_08_b200 as ep

    h, lay, idx, w, _, rng, starts = _setup(oracle, counts, E, R, k, H, 3 * sum(counts) + k)
    P = max(lay.total_rows, 1)
    y = make_x(P, H, rng) if dtype == "bf16" else make_x_fp16(P, H, rng)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    yd = torch.from_numpy(y.view(np.int16)).view(tdt).to(DEV)
    blocks = _rank_rows(lay, R)
    ys = [yd[a:b].clone() if b > a else torch.zeros((1, H), dtype=tdt, device=DEV)
          for a, b in blocks]
    out = torch.full((sum(counts), H), 0, dtype=torch.int16, device=DEV).view(tdt)
    wd = torch.from_numpy(w).to(DEV)
    for s, n in zip(starts, counts):
        ep.ep_combine_ranks(h, int(s), ys, wd[s:s + n].contiguous(), out[s:s + n])
    ep.ep_handle_check(h)
    ref = oracle.combine(y, w, lay.dst_row, dtype=dtype)
    assert np.array_equal(_bits(out), ref)


def test_one_rank_equals_the_single_buffer_path(oracle):
    import combine_ep_layout_08_b200 as ep

    T, E, k, H = 200, 64, 8, 2048
    rng = np.random.default_rng(9)
    idx, w = random_topk(T, E, k, rng)
    x = make_x(T, H, rng)
    h = ep.ep_handle_create(T, k, E, 1, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    single, sc1 = ep.ep_dispatch(h, _bf16(x), "fp8")
    P = int(ep.ep_handle_view(h, "total_recv_rows").item())
    recv = torch.zeros_like(single)
    sc = torch.zeros_like(sc1)
    ep.ep_dispatch_ranks(h, 0, _bf16(x), "fp8", [recv], [sc])
    ep.ep_handle_check(h)
    lay = oracle.layout(idx, E, 1)
    rows = lay.dst_row[lay.dst_row >= 0]
    assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows],
                          single.view(torch.uint8).cpu().numpy()[rows])
    assert np.array_equal(sc.cpu().numpy()[rows], sc1.cpu().numpy()[rows])


def test_rank_buffer_too_small_reports_capacity(oracle):
    import combine_ep_layout_08_b200 as ep

    counts, E, R, k, H = [60, 60], 16, 2, 4, 256
    h, lay, idx, _, x, _, starts = _setup(oracle, counts, E, R, k, H, 77, p_unused=0.0)
    blocks = _rank_rows(lay, R)
    recv = [torch.zeros((b - a, H), dtype=torch.bfloat16, device=DEV) for a, b in blocks]
    recv[1] = recv[1][: max(1, (blocks[1][1] - blocks[1][0]) // 2)].contiguous()
    ep.ep_dispatch_ranks(h, 0, _bf16(x), "bf16", recv)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_CAPACITY


def test_rank_table_is_checked(oracle):
    import combine_ep_layout_08_b200 as ep

    counts, E, R, k, H = [20, 20], 16, 2, 2, 256
    h, lay, idx, _, x, _, _ = _setup(oracle, counts, E, R, k, H, 5)
    blocks = _rank_rows(lay, R)
    recv = [torch.zeros((b - a + 1, H), dtype=torch.bfloat16, device=DEV) for a, b in blocks]
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_ranks(h, 0, _bf16(x), "bf16", recv[:1])            # one buffer for two ranks
    raw = torch.zeros(((blocks[0][1] + 2) * H * 2 + 16,), dtype=torch.uint8, device=DEV)
    off = raw[16:16 + (blocks[0][1] - blocks[0][0] + 1) * H * 2].view(torch.bfloat16).view(-1, H)
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_ranks(h, 0, _bf16(x), "bf16", [off, recv[1]])      # 16-byte aligned only
    assert ep.ep_handle_check(h, raise_on_error=False) == 0


def test_ranks_fp16_copy_and_cuda_graph_replay(oracle):
    """fp16 rows through the rank table, captured once in a CUDA graph and
    replayed with new inputs written into the same buffers (the table is
    passed by value, so the graph keeps it)."""
    import combine_ep_layout_08_b200 as ep

    counts, E, R, k, H = [70, 58], 32, 2, 4, 512
    rng = np.random.default_rng(31)
    T = sum(counts)
    idx, w = random_topk(T, E, k, rng)
    lay = oracle.layout(idx, E, R)
    blocks = _rank_rows(lay, R)
    h = ep.ep_handle_create(T, k, E, R, device=DEV)
    d_idx = torch.from_numpy(idx).to(DEV)
    xd = torch.empty((T, H), dtype=torch.float16, device=DEV)
    recv = [torch.zeros((b - a, H), dtype=torch.float16, device=DEV) for a, b in blocks]
    ys = [torch.empty((b - a, H), dtype=torch.float16, device=DEV) for a, b in blocks]
    wd = torch.from_numpy(w).to(DEV)
    out = torch.empty((T, H), dtype=torch.float16, device=DEV)

    def step():
        ep.ep_layout(h, d_idx)
        for s0, n in ((0, counts[0]), (counts[0], counts[1])):
            ep.ep_dispatch_ranks(h, s0, xd[s0:s0 + n], "fp16", recv)
        for s0, n in ((0, counts[0]), (counts[0], counts[1])):
            ep.ep_combine_ranks(h, s0, ys, wd[s0:s0 + n], out[s0:s0 + n])

    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        step()
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    used = lay.dst_row[lay.dst_row >= 0]
    for rep in range(2):
        x = make_x_fp16(T, H, rng)
        y = make_x_fp16(lay.total_rows, H, rng)
        xd.copy_(torch.from_numpy(x.view(np.int16)).view(torch.float16))
        for p, (a, b) in enumerate(blocks):
            ys[p].copy_(torch.from_numpy(y[a:b].view(np.int16)).view(torch.float16))
        g.replay()
        torch.cuda.synchronize()
        ep.ep_handle_check(h)
        ref = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)   # a 16-bit row copy
        for p, (a, b) in enumerate(blocks):
            rows = used[(used >= a) & (used < b)] - a
            assert np.array_equal(_bits(recv[p])[rows], ref[a:b][rows]), (rep, p)
        assert np.array_equal(_bits(out), oracle.combine(y, w, lay.dst_row, dtype="fp16")), rep
    del g


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("counts,E,R,k,H", [
    ([50, 0, 77, 31], 32, 4, 8, 1024),
    ([30, 33], 16, 2, 12, 256),            # k > 8: two slot batches
])
def test_backward_ranks_matches_the_global_backward(oracle, dtype, counts, E, R, k, H):
    """Per-rank backward: dispatch backward bit-exact; combine backward grad_y
    bit-exact on every used row and grad_w within the bound of the kernel's
    reduction tree around the oracle's fp64 dot product."""
    import combine_ep_layout_08_b200 as ep

    h, lay, idx, w, _, rng, starts = _setup(oracle, counts, E, R, k, H, 9 * sum(counts) + k)
    P = max(lay.total_rows, 1)
    gen = make_x if dtype == "bf16" else make_x_fp16
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    to_dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).to(DEV)
    blocks = _rank_rows(lay, R)
    T = sum(counts)
    # dispatch backward
    g = gen(P, H, rng)
    gd = to_dev(g)
    gr = [gd[a:b].clone() if b > a else torch.zeros((1, H), dtype=tdt, device=DEV) for a, b in blocks]
    gx = torch.zeros((T, H), dtype=tdt, device=DEV)
    for s, n in zip(starts, counts):
        ep.ep_dispatch_ranks_backward(h, int(s), gr, gx[s:s + n])
    ep.ep_handle_check(h)
    assert np.array_equal(_bits(gx), oracle.dispatch_backward(g, lay.dst_row, dtype=dtype))
    # combine backward
    y = gen(P, H, rng)
    go = gen(T, H, rng)
    yd = to_dev(y)
    ys = [yd[a:b].clone() if b > a else torch.zeros((1, H), dtype=tdt, device=DEV) for a, b in blocks]
    gys = [torch.zeros_like(t) for t in ys]
    god = to_dev(go)
    wd = torch.from_numpy(w).to(DEV)
    gw = torch.zeros((T, k), dtype=torch.float32, device=DEV)
    for s, n in zip(starts, counts):
        gw[s:s + n] = ep.ep_combine_ranks_backward(h, int(s), god[s:s + n].contiguous(), ys,
                                                   wd[s:s + n].contiguous(), gys)
    ep.ep_handle_check(h)
    gy_ref, gw_ref = oracle.combine_backward(go, y, w, lay.dst_row, dtype=dtype)
    used = lay.dst_row[lay.dst_row >= 0]
    for p, (a, b) in enumerate(blocks):
        rows = used[(used >= a) & (used < b)]
        assert np.array_equal(_bits(gys[p])[rows - a], gy_ref[rows]), p
    to32 = oracle.bf16_to_f32 if dtype == "bf16" else oracle.fp16_to_f32
    yf, gf, gwg = to32(y).astype(np.float64), to32(go).astype(np.float64), gw.cpu().numpy()
    for t in range(T):
        for j in range(k):
            d = lay.dst_row[t, j]
            if d < 0:
                assert gwg[t, j] == 0.0
                continue
            bound = grad_w_bound(H, float(np.abs(gf[t] * yf[d]).sum()), float(gw_ref[t, j]))
            assert abs(float(gwg[t, j]) - float(gw_ref[t, j])) <= bound + 1e-30, (t, j)
