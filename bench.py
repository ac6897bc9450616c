"""Benchmark of the MoE permutation path: layout -> dispatch -> combine.

One step = ep_layout + ep_dispatch + ep_combine over one synthetic batch of
the workload "8k": T=8192 tokens, hidden 7168, top-8 of 256 experts over 8
virtual ranks, uniform distinct routing with Dirichlet(1) weights, BF16
dispatch and BF16 combine.  The combine input y (the expert outputs) is made
once before timing by a stand-in expert op y = bf16(c[e] x) on the device;
the expert op is user code, not part of the path, and is not timed.

value = (dispatch bytes + combine bytes) / step time, with
  dispatch bytes = T*2H read + T*k*rowB written (rowB = 2H, or H + 4H/128 for FP8)
  combine bytes  = T*k*2H read + T*2H written
summed over all ranks (each rank runs an independent replica: the path does
not shard across GPUs here, so N GPUs run N replicas and no data crosses
between them).  Timing: CUDA events on the launching stream around each
step, L2 flushed (a 2x L2 write) between steps outside the events, barrier +
synchronize around the timed region, max over ranks.

Prints ONE JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(the plain C reference) instead, on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine GB/s & % of HBM peak; 8192x7168, top-8 of 256 experts"
UNIT = "GB/s"
MAIN_WORKLOAD = "8k"
SECONDARY = ("skewed", "dsv3", "decode")
WORKLOAD_TEXT = {
    "8k": "8K batch: T=8192 H=7168 E=256 R=8 top-8 uniform distinct, Dirichlet(1) weights, "
          "BF16 dispatch + BF16 combine, 128-row expert padding",
    "skewed": "skewed: T=8192 H=7168 E=256 R=32 top-8 Zipf(1.2), FP8 e4m3 1x128 dispatch + "
              "BF16 combine",
    "dsv3": "DeepSeek-V3 shape: T=4096 H=7168 E=256 R=8 group-limited top-8, FP8 dispatch",
    "decode": "decode: T=128 H=7168 E=256 R=16 group-limited top-8, FP8 dispatch",
}
LAUNCHES_PER_STEP = 3  # layout (one cooperative kernel), dispatch, combine


def algo_bytes(T, H, k, fmt):
    row = 2 * H if fmt == "bf16" else H + 4 * (H // 128)
    disp = T * 2 * H + T * k * row
    comb = T * k * 2 * H + T * 2 * H
    return disp, comb


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: torch copy, read+write)"
    return 6650.0, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


KERNEL_FILES = {
    "dispatch_bf16_v32_kernel": ("ep_dispatch.cu", "ep_dispatch_units.cuh", "ep_internal.cuh"),
    "dispatch_fp8_v32_kernel": ("ep_dispatch.cu", "ep_dispatch_units.cuh", "ep_internal.cuh"),
    "combine_kernel": ("ep_combine.cu", "ep_internal.cuh"),
}


def _code_only(text: str) -> str:
    """C/C++ source without comments and whitespace (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            if not text[i].isspace():
                out.append(text[i])
            i += 1
    return "".join(out)


def kernel_source_hash(kernel: str = "dispatch_bf16_v32_kernel"):
    """Hash of the code (comments and whitespace dropped) of the source files
    that make up a kernel (first 16 hex digits)."""
    h = hashlib.sha256()
    for name in KERNEL_FILES[kernel]:
        with open(os.path.join(ROOT, "combine_ep_layout_08_b200", "csrc", name),
                  encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if it
    was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get("kernels", {}).get(kernel)
    if e is None or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during timing."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.proc = None
        self.path = None
        try:
            import tempfile

            fd, self.path = tempfile.mkstemp(prefix="clk", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", "25"]
            if bus_id:
                cmd += ["-i", bus_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
            # nvidia-smi needs a moment to start: wait for its first sample so
            # that the timed region is covered
            deadline = time.time() + 15.0
            while time.time() < deadline and self.proc.poll() is None:
                if self._count_rows() > 0:
                    break
                time.sleep(0.05)
        except Exception:
            self.proc = None

    def _count_rows(self):
        try:
            with open(self.path) as f:
                return sum(1 for line in f if line.count(",") >= 8)
        except OSError:
            return 0

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # let at least one sample land after the timed region
        n0 = self._count_rows()
        deadline = time.time() + 2.0
        while time.time() < deadline and self._count_rows() < n0 + 2:
            time.sleep(0.02)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        import datetime

        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:9]))
            except Exception:
                continue
        os.unlink(self.path)
        inwin = [r for r in rows if t0 - 0.03 <= r[0] <= t1 + 0.03]
        window = "timed"
        if len(inwin) < 2:
            inwin, window = rows, "whole run (timed region shorter than the sampling period)"
        if not inwin:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inwin:
            for n, v in zip(names, r[3][1:]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inwin),
                "sm_max_mhz": max(r[2] for r in inwin), "reasons": sorted(reasons),
                "samples": len(inwin), "window": window}


# ----------------------------------------------------------------- GPU arm

def gpu_setup(name, seed, dev, T=None):
    import torch

    import combine_ep_layout_08_b200 as ep
    from workloads import make_workload

    w = make_workload(name, seed, T=T)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=dev)
    x = torch.from_numpy(w.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wt = torch.from_numpy(w.topk_weights).to(dev)
    cap = ep.ep_recv_rows_upper_bound(w.T, w.k, w.E, w.block_m)
    if w.fmt == "bf16":
        recv = torch.empty((cap, w.H), dtype=torch.bfloat16, device=dev)
        scales = None
    else:
        recv = torch.empty((cap, w.H), dtype=torch.float8_e4m3fn, device=dev)
        scales = torch.empty((cap, w.H // 128), dtype=torch.float32, device=dev)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    # one untimed pass to produce y with the stand-in expert op
    ep.ep_layout(h, idx)
    ep.ep_dispatch(h, x, w.fmt, recv_x=recv, recv_scales=scales)
    P = int(ep.ep_handle_view(h, "total_recv_rows").item())
    rows = torch.arange(P, device=dev)
    off = ep.ep_handle_view(h, "expert_off")
    e = torch.searchsorted(off[1:].contiguous(), rows, right=True)
    c = torch.from_numpy(w.expert_c).to(dev)[e].unsqueeze(1)
    y = torch.empty((cap, w.H), dtype=torch.bfloat16, device=dev)
    if scales is None:
        y[:P] = (recv[:P].float() * c).to(torch.bfloat16)
    else:
        y[:P] = (recv[:P].float() * scales[:P].repeat_interleave(128, 1) * c).to(torch.bfloat16)
    ep.ep_handle_check(h)
    return dict(w=w, h=h, x=x, idx=idx, wt=wt, recv=recv, scales=scales, out=out, y=y, P=P,
                routing=routing_stats(ep.ep_handle_read_counts(h), w))


def routing_stats(c: dict, w) -> dict:
    """Load balance of the layout (read once, untimed): per-expert slot counts and
    per-rank rows as max / mean, and the share of pad rows in the receive buffer."""
    e = np.asarray(c["num_tokens_per_expert"], np.float64)
    r = np.asarray(c["num_rows_per_rank"], np.float64)
    P = max(int(c["total_recv_rows"]), 1)
    return {"expert_slots_max": int(e.max()) if e.size else 0,
            "expert_slots_max_over_mean": round(float(e.max() / max(e.mean(), 1e-9)), 3),
            "rank_rows_max_over_mean": round(float(r.max() / max(r.mean(), 1e-9)), 3),
            "receive_rows": P,
            "pad_row_share": round(1.0 - float(e.sum()) / P, 4)}


NVTX = False  # --nvtx: name the three calls for a profiler's timeline (off when timing)


def _range(name):
    import contextlib

    import torch

    if not NVTX:
        return contextlib.nullcontext()
    return torch.cuda.nvtx.range(name)


def gpu_step(s, ev=None, skip=None):
    """One step: layout, dispatch, combine (skip: leave one of the three out,
    for the marginal timing; without the layout, dispatch and combine use the
    handle's layout of the same routing from the step before)."""
    import combine_ep_layout_08_b200 as ep

    h, w = s["h"], s["w"]
    if ev is not None:
        ev[0].record()
    if skip != "layout":
        with _range("ep_layout"):
            ep.ep_layout(h, s["idx"])
    if ev is not None:
        ev[1].record()
    if skip != "dispatch":
        with _range("ep_dispatch"):
            ep.ep_dispatch(h, s["x"], w.fmt, recv_x=s["recv"], recv_scales=s["scales"])
    if ev is not None:
        ev[2].record()
    if skip != "combine":
        with _range("ep_combine"):
            ep.ep_combine(h, s["y"], s["wt"], out=s["out"])
    if ev is not None:
        ev[3].record()


def time_gpu(s, steps, warmup, flush, barrier):
    """Device timing of `steps` steps, L2 flushed before each (outside the
    events).  Two passes: the step time from events at the two ends of each
    step only (events between kernels keep a kernel from starting while its
    predecessor drains: ~6 us per step at 8k), then the per-kernel split from
    a pass with events between the three kernels.  Returns per-step lists in
    ms and the wall-clock window of both passes."""
    import torch

    for _ in range(warmup):
        flush()
        gpu_step(s)
    ends = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    torch.cuda.synchronize()
    barrier()
    t0 = time.time()
    for i in range(steps):
        flush()
        ends[i][0].record()
        gpu_step(s)
        ends[i][1].record()
    for i in range(steps):
        flush()
        gpu_step(s, evs[i])
    # the step without one of the three kernels, events at its ends only: what
    # each kernel adds to the step when its launch overlaps its neighbours'
    part = {}
    for name, skip in (("no_layout", "layout"), ("no_dispatch", "dispatch"),
                       ("no_combine", "combine")):
        pe = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            flush()
            pe[i][0].record()
            gpu_step(s, skip=skip)
            pe[i][1].record()
        part[name] = pe
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    tot = [e[0].elapsed_time(e[1]) for e in ends]
    lay = [e[0].elapsed_time(e[1]) for e in evs]
    dis = [e[1].elapsed_time(e[2]) for e in evs]
    com = [e[2].elapsed_time(e[3]) for e in evs]
    split = [e[0].elapsed_time(e[3]) for e in evs]
    nol = [e[0].elapsed_time(e[1]) for e in part["no_layout"]]
    nod = [e[0].elapsed_time(e[1]) for e in part["no_dispatch"]]
    noc = [e[0].elapsed_time(e[1]) for e in part["no_combine"]]
    return dict(layout=lay, dispatch=dis, combine=com, step=tot, step_split=split,
                step_no_layout=nol, step_no_dispatch=nod, step_no_combine=noc, wall=(t0, t1))


def marginal(tm, d_bytes, c_bytes, agg=lambda v: v):
    """What each kernel adds to the step: the step time minus the step
    without that kernel, both with events at the ends only."""
    step = agg(statistics.mean(tm["step"]))
    lay = step - agg(statistics.mean(tm["step_no_layout"]))
    d = step - agg(statistics.mean(tm["step_no_dispatch"]))
    c = step - agg(statistics.mean(tm["step_no_combine"]))
    return {"layout_marginal_us": round(lay * 1e3, 2),
            "dispatch_marginal_us": round(d * 1e3, 2),
            "dispatch_marginal_GBps": round(d_bytes / (d / 1e3) / 1e9, 1) if d > 0 else None,
            "combine_marginal_us": round(c * 1e3, 2),
            "combine_marginal_GBps": round(c_bytes / (c / 1e3) / 1e9, 1) if c > 0 else None}


def time_gpu_e2e(s, steps, warmup):
    """The same step through the public API with host buffers, as a stream of
    batches: every step copies topk_idx, weights and x from pinned host memory,
    runs ep_layout, ep_dispatch and ep_combine, and copies out back to pinned
    host memory.  Device staging is double-buffered so that step i's
    device->host copy runs while step i+1's inputs come in (PCIe is full
    duplex); the kernels of one step run between the two.  The timed region
    spans all steps, pipeline fill (the first inputs alone) and drain (the last
    result alone) included; the time per step is the total over steps."""
    import torch

    import combine_ep_layout_08_b200 as ep

    w = s["w"]
    hx = s["x"].cpu().pin_memory()
    hidx = s["idx"].cpu().pin_memory()
    hwt = s["wt"].cpu().pin_memory()
    hout = [torch.empty(s["out"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dx = [torch.empty_like(s["x"]) for _ in range(2)]
    didx = [torch.empty_like(s["idx"]) for _ in range(2)]
    dwt = [torch.empty_like(s["wt"]) for _ in range(2)]
    dout = [torch.empty_like(s["out"]) for _ in range(2)]
    h, y = s["h"], s["y"]
    main = torch.cuda.current_stream()
    s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(device=s["x"].device) for _ in range(3))

    def run(n):
        """n pipelined steps; returns the device time in ms (events on main)."""
        a_ev = torch.cuda.Event(enable_timing=True)
        b_ev = torch.cuda.Event(enable_timing=True)
        a_ev.record(main)
        for st in (s_h2d, s_cmp, s_d2h):
            st.wait_stream(main)
        cmp_done, d2h_done = [], []
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(cmp_done[i - 2])    # buffer b read by step i-2
                didx[b].copy_(hidx, non_blocking=True)
                dwt[b].copy_(hwt, non_blocking=True)
                dx[b].copy_(hx, non_blocking=True)
                in_ev = torch.cuda.Event()
                in_ev.record(s_h2d)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_ev)
                if i >= 2:
                    s_cmp.wait_event(d2h_done[i - 2])   # dout[b] copied out by step i-2
                ep.ep_layout(h, didx[b])
                ep.ep_dispatch(h, dx[b], w.fmt, recv_x=s["recv"], recv_scales=s["scales"])
                ep.ep_combine(h, y, dwt[b], out=dout[b])
                ce = torch.cuda.Event()
                ce.record(s_cmp)
                cmp_done.append(ce)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ce)
                hout[b].copy_(dout[b], non_blocking=True)
                de = torch.cuda.Event()
                de.record(s_d2h)
                d2h_done.append(de)
        main.wait_stream(s_d2h)
        main.wait_stream(s_cmp)
        b_ev.record(main)
        b_ev.synchronize()
        return a_ev.elapsed_time(b_ev)

    run(max(warmup, 3))
    torch.cuda.synchronize()
    total_ms = run(steps)
    h2d = hx.numel() * 2 + hidx.numel() * 8 + hwt.numel() * 4
    d2h = hout[0].numel() * 2
    # the result the device-resident step gives, for the check of both host buffers
    ep.ep_layout(h, s["idx"])
    ep.ep_dispatch(h, s["x"], w.fmt, recv_x=s["recv"], recv_scales=s["scales"])
    ep.ep_combine(h, y, s["wt"], out=s["out"])
    ref = s["out"].cpu()
    assert torch.equal(hout[0], ref) and torch.equal(hout[1], ref), "host copy of out differs"
    return total_ms / steps, h2d, d2h


def fused_step(s):
    """The low-latency form of the step: ep_layout_dispatch (one launch for
    small batches) then ep_combine."""
    import combine_ep_layout_08_b200 as ep

    ep.ep_layout_dispatch(s["h"], s["idx"], s["x"], s["w"].fmt, recv_x=s["recv"],
                          recv_scales=s["scales"])
    ep.ep_combine(s["h"], s["y"], s["wt"], out=s["out"])


def graph_latency_us(s, reps=200, step=None, inner=1):
    """Decode-style latency: a CUDA graph holding `inner` back-to-back steps
    (layout + dispatch + combine each), replayed `reps` times; returns the
    device time per step.  With inner = 1 the replay rate of the host bounds
    the figure; inner = 20 is a decode pass with many MoE layers in one
    graph."""
    import torch

    step = step or gpu_step
    st = torch.cuda.Stream(device=s["x"].device)
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        step(s)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(inner):
            step(s)
    for _ in range(10):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    b.synchronize()
    us = a.elapsed_time(b) * 1000.0 / (reps * inner)
    del g
    return us


def time_ranks(dev, flush, seed, steps):
    """The expert-parallel entry points on one GPU: the 8k workload as R = 8
    ranks, one separately allocated receive buffer per rank (the ranks' own
    buffers, or peer views of them, on 8 GPUs).  Times ep_dispatch_ranks and
    ep_combine_ranks as one launch over all 8192 tokens and as 8 launches of
    1024 tokens (each source rank's own call).  Same bytes as the 8k step."""
    import torch

    import combine_ep_layout_08_b200 as ep
    from workloads import make_workload

    w = make_workload(MAIN_WORKLOAD, seed)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=dev)
    x = torch.from_numpy(w.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wt = torch.from_numpy(w.topk_weights).to(dev)
    ep.ep_layout(h, idx)
    roff = ep.ep_handle_view(h, "rank_off").cpu().tolist()
    recv = [torch.empty((max(roff[p + 1] - roff[p], 1), w.H), dtype=torch.bfloat16, device=dev)
            for p in range(w.R)]
    ys = [torch.randn((r.shape[0], w.H), device=dev).to(torch.bfloat16) for r in recv]
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    src = w.T // w.R
    res = {}
    for name, parts in (("one_launch", [(0, w.T)]),
                        ("per_source_rank", [(s * src, src) for s in range(w.R)])):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(3 + steps):
            flush()
            e = ev[i - 3] if i >= 3 else None
            if e:
                e[0].record()
            for t0, n in parts:
                ep.ep_dispatch_ranks(h, t0, x[t0:t0 + n], "bf16", recv)
            if e:
                e[1].record()
            for t0, n in parts:
                ep.ep_combine_ranks(h, t0, ys, wt[t0:t0 + n], out[t0:t0 + n])
            if e:
                e[2].record()
        torch.cuda.synchronize()
        d_ms = statistics.mean(a[0].elapsed_time(a[1]) for a in ev)
        c_ms = statistics.mean(a[1].elapsed_time(a[2]) for a in ev)
        db, cb = algo_bytes(w.T, w.H, w.k, w.fmt)
        res[name] = {"dispatch_us": round(d_ms * 1e3, 2),
                     "dispatch_GBps": round(db / (d_ms / 1e3) / 1e9, 1),
                     "combine_us": round(c_ms * 1e3, 2),
                     "combine_GBps": round(cb / (c_ms / 1e3) / 1e9, 1)}
    # the backward of both, one launch over all tokens
    gys = [torch.empty_like(t) for t in ys]
    go = torch.randn((w.T, w.H), device=dev).to(torch.bfloat16)
    gx = torch.empty_like(out)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(3 + steps):
        flush()
        e = ev[i - 3] if i >= 3 else None
        if e:
            e[0].record()
        ep.ep_dispatch_ranks_backward(h, 0, recv, gx)
        if e:
            e[1].record()
        ep.ep_combine_ranks_backward(h, 0, go, ys, wt, gys)
        if e:
            e[2].record()
    torch.cuda.synchronize()
    d_ms = statistics.mean(a[0].elapsed_time(a[1]) for a in ev)
    c_ms = statistics.mean(a[1].elapsed_time(a[2]) for a in ev)
    db, _ = algo_bytes(w.T, w.H, w.k, w.fmt)
    # grad_out and k y rows read, k grad_y rows and grad_w written (as time_backward)
    cbb = w.T * 2 * w.H + 2 * w.T * w.k * 2 * w.H + w.T * w.k * 4
    res["backward_one_launch"] = {
        "dispatch_backward_us": round(d_ms * 1e3, 2),
        "dispatch_backward_GBps": round(db / (d_ms / 1e3) / 1e9, 1),
        "combine_backward_us": round(c_ms * 1e3, 2),
        "combine_backward_GBps": round(cbb / (c_ms / 1e3) / 1e9, 1)}
    ep.ep_handle_check(h)
    res["workload"] = ("8k routing as R = 8 ranks on one GPU, 8 separate receive buffers, BF16; "
                       "dispatch_ranks / combine_ranks and their backward (no NVLink: the ranks' "
                       "buffers are local)")
    return res


def time_backward(dev, flush, seed, steps):
    """Backward of the 8k step: ep_dispatch_backward (a k-row sum per token)
    and ep_combine_backward (k scaled rows written, k dot products), each
    timed with CUDA events, L2 flushed before each launch."""
    import torch

    import combine_ep_layout_08_b200 as ep
    from workloads import make_workload

    w = make_workload(MAIN_WORKLOAD, seed, H=16)  # routing only; rows are drawn below
    H = 7168
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=dev)
    ep.ep_layout(h, torch.from_numpy(w.topk_idx).to(dev))
    cap = ep.ep_recv_rows_upper_bound(w.T, w.k, w.E, w.block_m)
    g = torch.randn((cap, H), device=dev).to(torch.bfloat16)
    go = torch.randn((w.T, H), device=dev).to(torch.bfloat16)
    y = torch.randn((cap, H), device=dev).to(torch.bfloat16)
    wt = torch.from_numpy(w.topk_weights).to(dev)
    gx = torch.empty((w.T, H), dtype=torch.bfloat16, device=dev)
    gy = torch.empty_like(y)
    res = {}
    for name, fn, nbytes in (
            ("dispatch_backward", lambda: ep.ep_dispatch_backward(h, g, gx),
             w.T * w.k * 2 * H + w.T * 2 * H),
            ("combine_backward", lambda: ep.ep_combine_backward(h, go, y, wt, gy),
             w.T * 2 * H + 2 * w.T * w.k * 2 * H + w.T * w.k * 4)):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(steps):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.mean(ts)
        res[name + "_us"] = round(ms * 1e3, 2)
        res[name + "_GBps"] = round(nbytes / (ms / 1e3) / 1e9, 1)
    ep.ep_handle_check(h)
    res["workload"] = "8k routing, H=7168, bf16 gradients (random rows)"
    return res


# ----------------------------------------------------------------- profiler cases

KERNEL_CASES = {
    "layout_8k": "ep_layout alone on the 8k routing (8192 tokens, top-8 of 256, 8 ranks): "
                 "only topk_idx and the workspace are allocated",
    "decode_fused": "the decode step in its fused form: ep_layout_dispatch (FP8) + ep_combine",
    "dispatch_2k": "layout + BF16 dispatch + combine on the first 2048 tokens of the 8k workload "
                   "(a quarter of the 8k launch; inputs and outputs larger than L2)",
    "dispatch_fp8_dsv3": "layout + FP8 dispatch + combine on the DeepSeek-V3 shape (4096 tokens, "
                         "group-limited top-8 of 256; inputs and outputs larger than L2)",
}


def run_kernel_case(name, steps, dev):
    """One small case of a kernel, `steps` times, for a profiler capture."""
    import torch

    import combine_ep_layout_08_b200 as ep
    from workloads import make_workload

    if name == "layout_8k":
        w = make_workload(MAIN_WORKLOAD, 0, H=16)
        h = ep.ep_handle_create(w.T, w.k, w.E, w.R, w.block_m, device=dev)
        idx = torch.from_numpy(w.topk_idx).to(dev)
        for _ in range(steps):
            ep.ep_layout(h, idx)
        shape = "T=%d k=%d E=%d R=%d" % (w.T, w.k, w.E, w.R)
    elif name == "decode_fused":
        s = gpu_setup("decode", 0, dev)
        for _ in range(steps):
            fused_step(s)
        h, shape = s["h"], "decode: T=%d H=%d E=%d R=%d k=%d fp8" % (s["w"].T, s["w"].H, s["w"].E,
                                                                   s["w"].R, s["w"].k)
    else:
        s = (gpu_setup(MAIN_WORKLOAD, 0, dev, T=2048) if name == "dispatch_2k"
             else gpu_setup("dsv3", 0, dev))
        torch.cuda.empty_cache()  # the set-up's temporaries: keep the device footprint small
        for _ in range(steps):
            gpu_step(s)
        h, shape = s["h"], "T=%d H=%d E=%d R=%d k=%d %s" % (s["w"].T, s["w"].H, s["w"].E,
                                                            s["w"].R, s["w"].k, s["w"].fmt)
    torch.cuda.synchronize()
    ep.ep_handle_check(h)
    print("kernel case %s (%s), %d steps: %s" % (name, shape, steps, KERNEL_CASES[name]), flush=True)


# ----------------------------------------------------------------- expert parallel

def run_ep(args, rank, world, dev, flush, barrier, peak, peak_src):
    """--ep: expert parallelism over the N ranks.  Every rank owns the 8k
    workload's tokens (weak scaling: N x 8192 tokens in all) and rank p holds
    experts [p E/N, (p+1) E/N).  A step: all-gather of the top-k indices,
    the global layout, ep_dispatch_ranks of this rank's tokens into every
    rank's receive buffer (peer buffers mapped with CUDA IPC), stream
    synchronise + barrier, ep_combine_ranks of this rank's tokens from every
    rank's expert outputs, stream synchronise + barrier.  The expert outputs
    come from the stand-in expert op once, before timing.  Device time per
    step with events, the max over ranks; value = all ranks' dispatch +
    combine bytes / that time."""
    import torch

    import combine_ep_layout_08_b200 as ep
    from workloads import expert_scale_table, make_workload

    w = make_workload(MAIN_WORKLOAD, args.seed + rank)
    x = torch.from_numpy(w.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wt = torch.from_numpy(w.topk_weights).to(dev)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)

    def gather():
        if world == 1:
            return idx, 0
        return ep.ep_allgather_topk(idx)

    glob, t0 = gather()
    h = ep.ep_handle_create(glob.shape[0], w.k, w.E, world, w.block_m, device=dev)
    ep.ep_layout(h, glob)
    roff = ep.ep_handle_view(h, "rank_off").cpu().tolist()
    rows = roff[rank + 1] - roff[rank]
    recv = torch.empty((max(rows, 1), w.H), dtype=torch.bfloat16, device=dev)
    y = torch.zeros_like(recv)
    shares = []

    def table(t):
        if world == 1:
            return [t]
        sh = ep.ep_ipc_share([t])
        shares.append(sh)
        return [sh.tensors[p][0] for p in range(world)]

    recv_tab = table(recv)
    ep.ep_dispatch_ranks(h, t0, x, "bf16", recv_tab)
    torch.cuda.synchronize()
    barrier()
    if rows:  # stand-in expert op on this rank's rows, once
        eoff = ep.ep_handle_view(h, "expert_off")
        e = torch.searchsorted(eoff[1:].contiguous(), torch.arange(rows, device=dev) + roff[rank],
                               right=True)
        c = torch.from_numpy(expert_scale_table(w.E)).to(dev)[e].unsqueeze(1)
        y[:rows] = (recv[:rows].float() * c).to(torch.bfloat16)
    torch.cuda.synchronize()
    y_tab = table(y)
    barrier()

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        g, _ = gather()
        ep.ep_layout(h, g)
        ep.ep_dispatch_ranks(h, t0, x, "bf16", recv_tab)
        if ev is not None:
            ev[1].record()
        torch.cuda.synchronize()
        barrier()
        ep.ep_combine_ranks(h, t0, y_tab, wt, out)
        if ev is not None:
            ev[2].record()
        torch.cuda.synchronize()
        barrier()

    for _ in range(args.warmup):
        flush()
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        step(evs[i])
    torch.cuda.synchronize()
    step_ms = aggregate_max(statistics.mean(e[0].elapsed_time(e[2]) for e in evs))
    dis_ms = aggregate_max(statistics.mean(e[0].elapsed_time(e[1]) for e in evs))
    com_ms = aggregate_max(statistics.mean(e[1].elapsed_time(e[2]) for e in evs))
    ep.ep_handle_check(h)
    for sh in shares:
        sh.close()
    d_bytes, c_bytes = algo_bytes(w.T, w.H, w.k, w.fmt)
    value = world * (d_bytes + c_bytes) / (step_ms / 1e3) / 1e9
    if rank == 0:
        cfg = workload_config(w, world)
        cfg["virtual_ranks"] = world
        cfg["parallelism"] = ("expert parallel over %d rank%s (one per GPU): %d experts each, "
                              "rows exchanged through CUDA IPC peer buffers"
                              % (world, "" if world == 1 else "s", w.E // world))
        line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": cfg,
                "kernels": {"gather_layout_dispatch_us": round(dis_ms * 1e3, 2),
                            "combine_us": round(com_ms * 1e3, 2),
                            "note": "each phase ends with a stream synchronise and a barrier "
                                    "across the ranks (host-side ordering)"},
                "peak": {"hbm_GBps": peak, "source": peak_src},
                "gpu_launches": 3 * args.steps}
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- CPU arm

def oracle_sample(w, tokens):
    """Inputs of an oracle step on the first `tokens` tokens, and the expert
    output y that its combine reads (made by the oracle's stand-in expert;
    not part of any timed step)."""
    import oracle

    idx = np.ascontiguousarray(w.topk_idx[:tokens])
    xb = np.ascontiguousarray(w.x_bits[:tokens])
    wt = np.ascontiguousarray(w.topk_weights[:tokens])
    lay0 = oracle.layout(idx, w.E, w.R, w.block_m)
    if w.fmt == "bf16":
        r0 = oracle.dispatch_bf16(xb, lay0.dst_row, lay0.total_rows)
        y = oracle.expert_scale_bf16(r0, lay0, w.expert_c)
    else:
        q0, s0 = oracle.dispatch_fp8(xb, lay0.dst_row, lay0.total_rows)
        y = oracle.expert_scale_fp8(q0, s0, lay0, w.expert_c)
    return {"tokens": tokens, "idx": idx, "xb": xb, "wt": wt, "y": y}


def oracle_timed_step(w, smp):
    """One oracle step (layout + dispatch + combine) on a prepared sample; seconds."""
    import oracle

    t0 = time.perf_counter()
    lay = oracle.layout(smp["idx"], w.E, w.R, w.block_m)
    if w.fmt == "bf16":
        oracle.dispatch_bf16(smp["xb"], lay.dst_row, lay.total_rows)
    else:
        oracle.dispatch_fp8(smp["xb"], lay.dst_row, lay.total_rows)
    oracle.combine(smp["y"], smp["wt"], lay.dst_row)
    return time.perf_counter() - t0


def oracle_seconds_per_token(w, probe=512):
    """Per-token time of one oracle step, from the second of two steps on the
    first `probe` tokens: the first also pays for first touches of freshly
    mapped output pages and would overstate the cost of a larger sample."""
    smp = oracle_sample(w, min(w.T, probe))
    oracle_timed_step(w, smp)
    return oracle_timed_step(w, smp) / smp["tokens"]


def _oracle_rate(w, budget_s):
    """GB/s of oracle steps on a bounded token sample; (GB/s, tokens, reps)."""
    per_tok = oracle_seconds_per_token(w)
    tokens = int(min(w.T, max(min(w.T, 512), budget_s / 2.0 / max(per_tok, 1e-9))))
    smp = oracle_sample(w, tokens)
    warm = oracle_timed_step(w, smp)                # warm-up; its time bounds the repetitions
    reps = min(5, max(1, int(budget_s / max(warm, 1e-9))))
    times = [oracle_timed_step(w, smp) for _ in range(reps)]
    d, c = algo_bytes(tokens, w.H, w.k, w.fmt)
    return (d + c) / statistics.mean(times) / 1e9, tokens, reps


def cpu_baseline(w, budget_s=12.0):
    """The oracle as it stands, timed twice on bounded token samples: the
    OpenMP build on all host cores (the reported value) and the
    single-threaded build (the parity tests' ground truth)."""
    import oracle

    oracle.build()
    oracle.build(openmp=True)
    one, t1, r1 = _oracle_rate(w, budget_s)
    with oracle.threads(0) as n:
        alln, tn, rn = _oracle_rate(w, budget_s)
    what = ("first %d of %d tokens of the same workload, 1 warm-up + %d timed repetitions, "
            "C oracle (gcc -O2%s), layout (serial) + dispatch + combine")
    return {"value": round(alln, 3), "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": what % (tn, w.T, rn, ", -fopenmp: tokens in parallel"),
            "single_core": {"value": round(one, 3), "unit": UNIT, "cores": 1,
                            "sample": what % (t1, w.T, r1, "")},
            "host": host_cpu()}


def host_cpu() -> dict:
    """The host the CPU numbers come from: logical cores and CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"logical_cores": os.cpu_count(), "cpu_model": model}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    from workloads import make_workload

    import oracle

    oracle.build(openmp=True)
    w = make_workload(MAIN_WORKLOAD, 0)
    with oracle.threads(0) as cores:
        line = _reference_line(args, world, w, cores)
    print(json.dumps(line), flush=True)


def _reference_line(args, world, w, cores):
    """The reference arm's steps (the oracle on `cores` threads) and its JSON line."""
    per_tok = oracle_seconds_per_token(w)
    budget = 120.0                                  # seconds of timed and warm-up steps
    per_step = budget / max(1, args.steps + args.warmup)
    floor = min(w.T, 256)
    tokens = int(max(floor, min(w.T, per_step / per_tok)))
    smp = oracle_sample(w, tokens)
    for _ in range(2):                              # the probe can misjudge a larger sample
        t = oracle_timed_step(w, smp)
        if t <= 1.5 * per_step or tokens == floor:
            break
        tokens = int(max(floor, tokens * per_step / t))
        smp = oracle_sample(w, tokens)
    for _ in range(args.warmup):
        oracle_timed_step(w, smp)
    ts = [oracle_timed_step(w, smp) for _ in range(args.steps)]
    d, c = algo_bytes(tokens, w.H, w.k, w.fmt)
    ms = statistics.mean(ts) * 1e3
    val = (d + c) / (ms / 1e3) / 1e9
    line = {"metric": METRIC, "value": round(val, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "impl": "reference",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": round(val, 3), "unit": UNIT, "cores": cores,
                             "kind": "oracle",
                             "sample": "first %d of %d tokens per step, C oracle (gcc -O2, "
                                       "-fopenmp: tokens in parallel)" % (tokens, w.T),
                             "host": host_cpu()},
            "e2e": {"value": round(val, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    return line


# ----------------------------------------------------------------- main

def workload_config(w, world):
    """The `config` object of the JSON line, the same in both arms."""
    return {"workload": WORKLOAD_TEXT[MAIN_WORKLOAD], "tokens": w.T, "hidden": w.H,
            "experts": w.E, "virtual_ranks": w.R, "topk": w.k, "fmt": w.fmt,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "flushed between steps (write of 2x L2), outside the events"}


def aggregate_max(value: float, group=None) -> float:
    """Max over ranks (a scalar all-reduce; no data-path collective)."""
    import torch
    import torch.distributed as dist

    if group is None and not (dist.is_available() and dist.is_initialized()):
        return value
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--secondary", default="all",
                    help="comma-separated secondary workloads (skewed, dsv3, decode, ranks, backward) "
                         "or all")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--nvtx", action="store_true",
                    help="NVTX ranges around the three calls (for a profiler's timeline)")
    ap.add_argument("--kernel-case", choices=sorted(KERNEL_CASES),
                    help="run one small case of a kernel --steps times and print its shape (for a "
                         "profiler; no timing line)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the N ranks (rows exchanged through CUDA IPC "
                         "peer buffers) instead of N independent replicas")
    args = ap.parse_args()
    global NVTX
    NVTX = args.nvtx

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    from combine_ep_layout_08_b200 import _build

    if rank == 0:
        _build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    barrier()
    props = torch.cuda.get_device_properties(dev)
    flush_buf = torch.empty(2 * int(props.L2_cache_size), dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    peak, peak_src = load_peaks()
    if args.kernel_case:
        run_kernel_case(args.kernel_case, args.steps, dev)
        return
    if args.ep:
        run_ep(args, rank, world, dev, flush, barrier, peak, peak_src)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    s = gpu_setup(MAIN_WORKLOAD, args.seed + rank, dev)
    w = s["w"]
    routing_main = s["routing"]
    bus = None
    try:
        bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except Exception:
        bus = None
    sampler = ClockSampler(bus) if rank == 0 else None
    tm = time_gpu(s, args.steps, args.warmup, flush, barrier)
    clocks = sampler.stop(*tm["wall"]) if sampler else None

    d_bytes, c_bytes = algo_bytes(w.T, w.H, w.k, w.fmt)
    step_ms = aggregate_max(statistics.mean(tm["step"]))
    lay_ms = aggregate_max(statistics.mean(tm["layout"]))
    dis_ms = aggregate_max(statistics.mean(tm["dispatch"]))
    com_ms = aggregate_max(statistics.mean(tm["combine"]))
    marg_main = marginal(tm, d_bytes, c_bytes, aggregate_max)  # every rank: collectives inside
    value = world * (d_bytes + c_bytes) / (step_ms / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        e_steps = max(3, min(args.steps, 100))
        e_ms, h2d, d2h = time_gpu_e2e(s, e_steps, 3)
        e_ms = aggregate_max(e_ms)
        e2e = {"value": round(world * (d_bytes + c_bytes) / (e_ms / 1e3) / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms, 4),
               "steps": e_steps,
               "how": "a stream of steps through the Python API: pinned host x, topk_idx, "
                      "weights in and out back every step; double-buffered device staging on "
                      "3 streams (H2D | ep_layout, ep_dispatch, ep_combine | D2H) so that a "
                      "step's D2H overlaps the next step's H2D; events span all steps incl. "
                      "pipeline fill and drain"}

    secondary = {}
    if not args.no_secondary:
        del s
        torch.cuda.empty_cache()
        chosen = SECONDARY if args.secondary == "all" else \
            [n for n in SECONDARY if n in args.secondary.split(",")]
        for name in chosen:
            s2 = gpu_setup(name, args.seed + rank, dev)
            w2 = s2["w"]
            n = max(3, min(args.steps, 100))
            t2 = time_gpu(s2, n, min(args.warmup, 10), flush, barrier)
            db, cb = algo_bytes(w2.T, w2.H, w2.k, w2.fmt)
            ent = {"workload": WORKLOAD_TEXT[name], "routing": s2["routing"],
                   "step_us": round(statistics.mean(t2["step"]) * 1e3, 2),
                   "layout_us": round(statistics.mean(t2["layout"]) * 1e3, 2),
                   "dispatch_us": round(statistics.mean(t2["dispatch"]) * 1e3, 2),
                   "combine_us": round(statistics.mean(t2["combine"]) * 1e3, 2),
                   "dispatch_GBps": round(db / (statistics.mean(t2["dispatch"]) / 1e3) / 1e9, 1),
                   "combine_GBps": round(cb / (statistics.mean(t2["combine"]) / 1e3) / 1e9, 1),
                   "value_GBps": round((db + cb) / (statistics.mean(t2["step"]) / 1e3) / 1e9, 1),
                   **marginal(t2, db, cb)}
            if name == "decode":
                # per step inside a graph of 20 steps; one-step graphs as well
                ent["graph_step_us"] = round(graph_latency_us(s2, reps=50, inner=20), 2)
                ent["graph_fused_step_us"] = round(
                    graph_latency_us(s2, reps=50, step=fused_step, inner=20), 2)
                ent["graph1_step_us"] = round(graph_latency_us(s2), 2)
                ent["graph1_fused_step_us"] = round(graph_latency_us(s2, step=fused_step), 2)
                ent["graph_note"] = ("graph_*: device time per step in a CUDA graph of 20 "
                                     "back-to-back steps; graph1_*: a one-step graph replayed "
                                     "from the host (bounded by the replay rate)")
            secondary[name] = ent
            del s2
            torch.cuda.empty_cache()

    if not args.no_secondary and (args.secondary == "all" or "ranks" in args.secondary.split(",")):
        secondary["8k_ranks"] = time_ranks(dev, flush, args.seed + rank, max(3, min(args.steps, 50)))
        torch.cuda.empty_cache()
    if not args.no_secondary and (args.secondary == "all" or "backward" in args.secondary.split(",")):
        secondary["8k_backward"] = time_backward(dev, flush, args.seed + rank,
                                                 max(3, min(args.steps, 50)))
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    dom = "dispatch" if dis_ms >= com_ms else "combine"
    dom_ms = max(dis_ms, com_ms)
    dom_bytes = d_bytes if dom == "dispatch" else c_bytes
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    kname = "dispatch_bf16_v32_kernel" if dom == "dispatch" else "combine_kernel"
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": ncu_traffic(kname),
                "kernel": kname, "peak_source": peak_src}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w, world),
            "bytes_per_step": d_bytes + c_bytes,
            "routing": routing_main,
            "pct_of_measured_hbm": round(value / world / peak, 4),
            "pct_of_hbm_spec_8TBps": round(value / world / 8000.0, 4),
            "kernels": {"layout_us": round(lay_ms * 1e3, 2), "dispatch_us": round(dis_ms * 1e3, 2),
                        "combine_us": round(com_ms * 1e3, 2),
                        "dispatch_GBps": round(d_bytes / (dis_ms / 1e3) / 1e9, 1),
                        "combine_GBps": round(c_bytes / (com_ms / 1e3) / 1e9, 1),
                        "dispatch_p50_p95_p99_us": [round(np.percentile(tm["dispatch"], q) * 1e3, 2)
                                                    for q in (50, 95, 99)],
                        "combine_p50_p95_p99_us": [round(np.percentile(tm["combine"], q) * 1e3, 2)
                                                   for q in (50, 95, 99)],
                        "split_step_us": round(statistics.mean(tm["step_split"]) * 1e3, 2),
                        **marg_main,
                        "note": "per-kernel times from a second pass of the same steps with "
                                "events between the kernels (split_step_us is that pass's step); "
                                "value and ms_per_step come from events at the step's ends only; "
                                "*_marginal_*: the step time minus the step without that kernel "
                                "(events at the ends only), what the kernel adds to the step"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
