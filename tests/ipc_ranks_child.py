"""One rank of the two-process expert-parallel exchange that
tests/test_gpu_ipc_ranks.py runs (a helper module, started with the spawn
method; not a test file).

Each rank is a separate process with its own CUDA context on the same GPU,
owns a contiguous slice of the global tokens and one rank's receive buffer,
and reaches the other rank's buffers only through CUDA IPC mappings
(ep_ipc_share).  No kernel waits on another: the phases are ordered on the
host, each one closed by a stream synchronise and a process-group barrier.
The results are written to OUTDIR/rank<r>.npz for the parent to compare with
the oracle; the stand-in expert op is torch arithmetic (harness, not the
path), checked there too."""
from __future__ import annotations

import datetime
import os
import traceback

import numpy as np


def case_inputs(case):
    """The global inputs of a case (the same seeded draws in every process)."""
    from workloads import make_x, random_topk

    rng = np.random.default_rng(case["seed"])
    T = sum(case["counts"])
    idx, w = random_topk(T, case["E"], case["k"], rng, p_unused=0.05)
    x = make_x(T, case["H"], rng)
    return idx, w, x


SENT16 = 0x5A5A   # receive-row sentinel (bf16 bits)
SENT8 = 0x5A      # receive-row sentinel (fp8 bytes)


def run_rank(rank: int, world: int, port: int, outdir: str, case: dict) -> None:
    try:
        _run(rank, world, port, outdir, case)
    except BaseException:
        with open(os.path.join(outdir, "rank%d.err" % rank), "w") as f:
            f.write(traceback.format_exc())
        raise


def _run(rank, world, port, outdir, case):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    import combine_ep_layout_08_b200 as ep
    from workloads import expert_scale_table

    idx, w, x = case_inputs(case)
    E, k, H, fmt = case["E"], case["k"], case["H"], case["fmt"]
    starts = np.concatenate([[0], np.cumsum(case["counts"])]).astype(int)
    t0, n = int(starts[rank]), int(case["counts"][rank])

    # all ranks' indices in rank order: the global token order
    glob, first = ep.ep_allgather_topk(torch.from_numpy(idx[t0:t0 + n]).contiguous())
    assert first == t0 and glob.shape[0] == idx.shape[0]
    h = ep.ep_handle_create(glob.shape[0], k, E, world, device=dev)
    ep.ep_layout(h, glob.to(dev))
    roff = ep.ep_handle_view(h, "rank_off").cpu().numpy()
    eoff = ep.ep_handle_view(h, "expert_off")
    rows = int(roff[rank + 1] - roff[rank])
    cap = max(rows, 1)

    # this rank's receive buffer, shared with the other rank
    if fmt == "bf16":
        recv = torch.full((cap, H), SENT16, dtype=torch.int16, device=dev).view(torch.bfloat16)
        share = ep.ep_ipc_share([recv])
        ep.ep_dispatch_ranks(h, t0, _bf16(x[t0:t0 + n], dev), "bf16",
                             [share.tensors[p][0] for p in range(world)])
    else:
        recv = torch.full((cap, H), SENT8, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
        scales = torch.full((cap, H // 128), -1.0, dtype=torch.float32, device=dev)
        share = ep.ep_ipc_share([recv, scales])
        ep.ep_dispatch_ranks(h, t0, _bf16(x[t0:t0 + n], dev), "fp8",
                             [share.tensors[p][0] for p in range(world)],
                             [share.tensors[p][1] for p in range(world)])
    torch.cuda.synchronize()
    dist.barrier()                       # every rank's rows are in every buffer

    # stand-in expert op on this rank's own rows: y = bf16(c[e] * x~)
    c = torch.from_numpy(expert_scale_table(E)).to(dev)
    local_rows = torch.arange(rows, device=dev) + int(roff[rank])
    e = torch.searchsorted(eoff[1:].contiguous(), local_rows, right=True)
    y = torch.zeros((cap, H), dtype=torch.bfloat16, device=dev)
    if rows:
        if fmt == "bf16":
            val = recv[:rows].float()
        else:
            val = recv[:rows].float() * scales[:rows].repeat_interleave(128, dim=1)
        y[:rows] = (val * c[e].unsqueeze(1)).to(torch.bfloat16)
    torch.cuda.synchronize()
    yshare = ep.ep_ipc_share([y])        # an all-gather: every rank's y is complete
    dist.barrier()

    out = torch.empty((n, H), dtype=torch.bfloat16, device=dev)
    if n:
        ep.ep_combine_ranks(h, t0, [yshare.tensors[p][0] for p in range(world)],
                            torch.from_numpy(w[t0:t0 + n]).contiguous().to(dev), out)
    torch.cuda.synchronize()
    dist.barrier()                       # no rank unmaps or frees while another reads
    status = ep.ep_handle_check(h, raise_on_error=False)

    res = {"rows": np.array([rows]), "status": np.array([status]),
           "y": y[:rows].view(torch.int16).cpu().numpy().view(np.uint16),
           "out": out.view(torch.int16).cpu().numpy().view(np.uint16)}
    if fmt == "bf16":
        res["recv"] = recv.view(torch.int16).cpu().numpy().view(np.uint16)
    else:
        res["recv"] = recv.view(torch.uint8).cpu().numpy()
        res["scales"] = scales.cpu().numpy()
    np.savez(os.path.join(outdir, "rank%d.npz" % rank), **res)
    share.close()
    yshare.close()
    dist.barrier()
    dist.destroy_process_group()


def _bf16(bits, dev):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
