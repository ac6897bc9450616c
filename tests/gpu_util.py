"""Helpers shared by the GPU parity tests: move a workload to the device, run
the CUDA path through the binding, run the stand-in expert op, compare with
the oracle.  Nothing here computes an expected value: expected values come
from ``oracle`` only."""
from __future__ import annotations

import numpy as np
import torch

import combine_ep_layout_08_b200 as ep

DEV = "cuda:0"
LAYOUT_VIEWS = ("num_tokens_per_expert", "num_tokens_per_rank", "num_rows_per_rank",
                "expert_off", "rank_off", "is_token_in_rank", "dst_row")


def bits_to_bf16(bits: np.ndarray, device=DEV) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_layout(h: ep.EPHandle) -> dict:
    out = {name: ep.ep_handle_view(h, name).cpu().numpy() for name in LAYOUT_VIEWS}
    P = int(ep.ep_handle_view(h, "total_recv_rows").item())
    out["total_rows"] = P
    out["recv_src"] = ep.ep_handle_view(h, "recv_src")[:P].cpu().numpy()
    return out


def assert_layout_equal(g: dict, lay) -> None:
    for name in LAYOUT_VIEWS:
        exp = getattr(lay, name)
        got = g[name]
        assert got.shape == exp.shape, (name, got.shape, exp.shape)
        if not np.array_equal(got, exp):
            bad = np.argwhere(got != exp)[:5]
            raise AssertionError("%s differs at %s: got %s expected %s" % (
                name, bad.tolist(), got[tuple(bad.T)], exp[tuple(bad.T)]))
    assert g["total_rows"] == lay.total_rows
    assert np.array_equal(g["recv_src"], lay.recv_src)


def expert_op_torch(recv: torch.Tensor, scales, expert_off: torch.Tensor, c: torch.Tensor,
                    P: int) -> torch.Tensor:
    """Stand-in expert op on the device (harness, not the path):
    y = bf16(c[e] * x) or bf16(c[e] * (q * s)), fp32 products in that order."""
    rows = torch.arange(P, device=recv.device)
    e = torch.searchsorted(expert_off[1:].contiguous(), rows, right=True)
    cr = c[e].unsqueeze(1)
    if scales is None:
        yf = recv[:P].float() * cr
    else:
        deq = recv[:P].float() * scales[:P].repeat_interleave(128, dim=1)
        yf = deq * cr
    y = torch.empty((max(P, 1), recv.shape[1]), dtype=torch.bfloat16, device=recv.device)
    y[:P] = yf.to(torch.bfloat16)
    return y


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place (+0 and -0 coincide)."""
    def ordered(b):
        b = b.astype(np.int32)
        mag = b & 0x7FFF
        return np.where(b & 0x8000, -mag, mag)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def nonpad_rows(lay) -> np.ndarray:
    return lay.dst_row[lay.dst_row >= 0].astype(np.int64)


def grad_w_roundings(H):
    """Roundings on the longest path of the combine backward's grad_w
    reduction.  Rows of H % 16 == 0 (32-byte aligned, as torch allocates
    them) take the one-warp-per-token kernel, as the per-rank combine
    backward always does: each lane chains 16 fused multiply-adds per 32-byte
    vector over ceil(H/16/32) vectors, then 5 xor-shuffle levels.  Other H
    take the one-CTA-per-token kernel: each thread chains 8 per 16-byte
    vector over its vectors, 5 shuffle levels, then the sum over the CTA's
    warps in order."""
    if H % 16 == 0:
        vpr = H // 16
        return 16 * -(-vpr // 32) + 5
    vpr = H // 8
    threads = min(256, 32 * -(-vpr // 32))
    return 8 * -(-vpr // threads) + 5 + (threads // 32 - 1)


def grad_w_bound(H, abs_dot, ref):
    """gamma_n * sum|grad_out * y| (the bound of any summation tree whose
    longest path has n roundings) plus half an fp32 ulp of the oracle's own
    rounding of its fp64 dot product."""
    n = grad_w_roundings(H)
    u = 2.0 ** -24
    return n * u / (1.0 - n * u) * abs_dot + u * abs(ref)
