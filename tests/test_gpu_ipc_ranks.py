"""Expert parallelism across processes: two processes on one GPU, each with
its own CUDA context, exchange rows through CUDA IPC mappings of each
other's buffers (tests/ipc_ranks_child.py).  Each rank owns half of the
tokens and one receive buffer; it all-gathers the top-k indices, computes the
global layout, stores its tokens' rows straight into both ranks' buffers
(ep_dispatch_ranks), runs the stand-in expert on its own rows, and combines
its tokens from both ranks' expert outputs (ep_combine_ranks).  Host-side
ordering only -- stream synchronise and a gloo barrier between the phases --
so no kernel waits on another.

Checked against the oracle over the global token order, bit-exact: each
rank's buffer equals its block of the oracle's receive buffer (BF16 rows, or
FP8 codes and scales), pad rows keep their sentinel, the expert outputs equal
the oracle's stand-in expert, and each rank's combined rows equal the
oracle's combine of its tokens."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

import ipc_ranks_child as child

pytestmark = pytest.mark.gpu

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(tmp_path, case):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=child.run_rank, args=(r, WORLD, port, str(tmp_path), case))
             for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    hung = [p for p in procs if p.is_alive()]
    for p in hung:
        p.terminate()
        p.join(timeout=30)
    errs = [open(os.path.join(tmp_path, f)).read() for f in sorted(os.listdir(tmp_path))
            if f.endswith(".err")]
    assert not hung, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs), "\n".join(errs)
    return [dict(np.load(os.path.join(tmp_path, "rank%d.npz" % r))) for r in range(WORLD)]


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_two_processes_exchange_rows_through_ipc(oracle, tmp_path, fmt):
    case = dict(counts=[300, 217], E=64, k=8, H=1024, fmt=fmt, seed=7)
    res = _run_ranks(tmp_path, case)
    idx, w, x = child.case_inputs(case)
    lay = oracle.layout(idx, case["E"], WORLD)
    P = lay.total_rows
    from workloads import expert_scale_table

    c = expert_scale_table(case["E"])
    if fmt == "bf16":
        ref = oracle.dispatch_bf16(x, lay.dst_row, P)
        y_ref = oracle.expert_scale_bf16(ref, lay, c)
    else:
        ref, ref_s = oracle.dispatch_fp8(x, lay.dst_row, P)
        y_ref = oracle.expert_scale_fp8(ref, ref_s, lay, c)
    used = lay.dst_row[lay.dst_row >= 0]
    y_glob = np.zeros((max(P, 1), case["H"]), np.uint16)
    for p in range(WORLD):
        r = res[p]
        assert int(r["status"][0]) == 0
        a, b = int(lay.rank_off[p]), int(lay.rank_off[p + 1])
        assert int(r["rows"][0]) == b - a
        mine = used[(used >= a) & (used < b)]
        assert np.array_equal(r["recv"][mine - a], ref[mine]), p
        if fmt == "fp8":
            assert np.array_equal(r["scales"][mine - a].view(np.uint32), ref_s[mine].view(np.uint32))
        pad = np.setdiff1d(np.arange(b - a), mine - a)
        sentinel = child.SENT16 if fmt == "bf16" else child.SENT8
        assert np.all(r["recv"][pad] == sentinel), "a pad row of rank %d was written" % p
        assert np.array_equal(r["y"][mine - a], y_ref[mine]), p
        y_glob[a:b] = r["y"]
    out_ref = oracle.combine(y_glob, w, lay.dst_row)
    starts = np.concatenate([[0], np.cumsum(case["counts"])]).astype(int)
    for p in range(WORLD):
        assert np.array_equal(res[p]["out"], out_ref[starts[p]:starts[p + 1]]), p
