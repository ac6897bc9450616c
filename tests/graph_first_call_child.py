"""Child process of test_gpu_graph_first_call.py: the library's first kernel
launches of this process happen inside a CUDA graph capture.  Captures
ep_layout + ep_dispatch (BF16 and FP8) + ep_combine, replays the graph twice
and saves the results for the parent to compare with the oracle."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import combine_ep_layout_08_b200 as ep  # noqa: E402
from workloads import make_workload, make_x  # noqa: E402


def main(out_path):
    dev = torch.device("cuda", 0)
    w = make_workload("8k", 0, T=1024)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=dev)
    x = torch.from_numpy(w.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wt = torch.from_numpy(w.topk_weights).to(dev)
    cap = ep.ep_recv_rows_upper_bound(w.T, w.k, w.E, w.block_m)
    recv = torch.zeros((cap, w.H), dtype=torch.bfloat16, device=dev)
    recv8 = torch.zeros((cap, w.H), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
    sc = torch.zeros((cap, w.H // 128), dtype=torch.float32, device=dev)
    y_bits = make_x(cap, w.H, np.random.default_rng(3))
    y = torch.from_numpy(y_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    out = torch.zeros((w.T, w.H), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ep.ep_layout(h, idx)
        ep.ep_dispatch(h, x, "bf16", recv_x=recv)
        ep.ep_dispatch(h, x, "fp8", recv_x=recv8, recv_scales=sc)
        ep.ep_combine(h, y, wt, out=out)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ep.ep_handle_check(h)
    np.savez(out_path,
             dst_row=ep.ep_handle_view(h, "dst_row").cpu().numpy(),
             recv=recv.view(torch.int16).cpu().numpy().view(np.uint16),
             recv8=recv8.view(torch.uint8).cpu().numpy(),
             scales=sc.cpu().numpy(),
             out=out.view(torch.int16).cpu().numpy().view(np.uint16),
             y=y_bits, x=w.x_bits, idx=w.topk_idx, wt=w.topk_weights,
             E=w.E, R=w.R, block_m=w.block_m)
    del g


if __name__ == "__main__":
    main(sys.argv[1])
