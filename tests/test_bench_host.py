"""Host logic of bench.py on the CPU: the algorithmic byte model, and the
max-over-ranks reduction used for multi-GPU timing (world_size 2, gloo)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_algorithmic_bytes_match_the_stated_model():
    # dispatch = T*2H read + T*k*rowB written; combine = T*k*2H read + T*2H written
    assert bench.algo_bytes(8192, 7168, 8, "bf16") == (1056964608, 1056964608)
    assert bench.algo_bytes(8192, 7168, 8, "fp8") == (601882624, 1056964608)
    assert bench.algo_bytes(4096, 7168, 8, "fp8") == (300941312, 528482304)
    assert bench.algo_bytes(128, 7168, 8, "fp8") == (9404416, 16515072)
    assert bench.algo_bytes(128, 256, 2, "bf16") == (196608, 196608)
    # the pages' per-stage volume: batch x top_k x hidden x sizeof(dtype)
    T, H, k = 8192, 7168, 8
    d, c = bench.algo_bytes(T, H, k, "bf16")
    assert d - T * 2 * H == T * k * H * 2 == c - T * 2 * H


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [3.5, 7.25][rank]
        got = bench.aggregate_max(local)
        q.put((rank, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_aggregate_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 7.25, 1: 7.25}


def test_aggregate_max_single_process_is_identity():
    assert bench.aggregate_max(1.5) == 1.5


def test_marginal_cost_is_the_step_minus_the_step_without_the_kernel():
    # per-step times in ms, as time_gpu returns them
    tm = {"step": [0.330, 0.334], "step_no_layout": [0.325, 0.325],
          "step_no_dispatch": [0.172, 0.174], "step_no_combine": [0.170, 0.172]}
    m = bench.marginal(tm, 1056964608, 1056964608)
    assert m["layout_marginal_us"] == pytest.approx(7.0)
    assert m["dispatch_marginal_us"] == pytest.approx(159.0)
    assert m["combine_marginal_us"] == pytest.approx(161.0)
    assert m["dispatch_marginal_GBps"] == pytest.approx(1056964608 / 159.0e-6 / 1e9, rel=1e-3)
    # the aggregate (max over ranks) is applied to each mean before the difference
    seen = []
    bench.marginal(tm, 1, 1, agg=lambda v: seen.append(v) or v)
    assert len(seen) == 4
    # a kernel that adds nothing has no rate
    tm["step_no_combine"] = tm["step"]
    assert bench.marginal(tm, 1, 1)["combine_marginal_GBps"] is None


def test_kernel_hash_is_stable():
    for k in ("dispatch_bf16_v32_kernel", "combine_kernel"):
        assert bench.kernel_source_hash(k) == bench.kernel_source_hash(k)
        assert len(bench.kernel_source_hash(k)) == 16


def test_kernel_hash_ignores_comments_and_whitespace():
    import bench

    a = "int f(int x) { return x + 1; } // one\n/* block */"
    b = "int f(int x)\n{\n    return x + 1;  /* other words */\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only('s = "// kept";') == 's="// kept";'
    assert bench._code_only("x = 1;") != bench._code_only("x = 2;")


def _gather_worker(rank, world, port, q):
    import os

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import combine_ep_layout_08_b200 as ep

        n = [3, 5][rank]
        idx = torch.arange(n * 2, dtype=torch.int64).view(n, 2) + 100 * rank
        glob, t0 = ep.ep_allgather_topk(idx)
        q.put((rank, glob.tolist(), t0))
    finally:
        dist.destroy_process_group()


def test_allgather_topk_gloo_world_2():
    """The expert-parallel global token order: rank-major concatenation of
    the ranks' top-k rows (unequal counts), and each rank's first token."""
    import multiprocessing as mp
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(2):
        r, glob, t0 = q.get(timeout=120)
        res[r] = (glob, t0)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    exp = [[2 * i, 2 * i + 1] for i in range(3)] + [[100 + 2 * i, 101 + 2 * i] for i in range(5)]
    assert res[0] == (exp, 0) and res[1] == (exp, 3)


def test_routing_stats_closed_form():
    import numpy as np

    import bench

    c = dict(num_tokens_per_expert=np.array([3, 1, 0, 4], np.int32),
             num_tokens_per_rank=np.array([2, 2], np.int32),
             num_rows_per_rank=np.array([4, 4], np.int32), total_recv_rows=16)
    r = bench.routing_stats(c, None)
    assert r["expert_slots_max"] == 4 and r["expert_slots_max_over_mean"] == 2.0
    assert r["rank_rows_max_over_mean"] == 1.0 and r["pad_row_share"] == 0.5
