"""Seeded synthetic inputs for the MoE dispatch-layout / dispatch / combine path.

This module only draws inputs: hidden states, router top-k indices and routing
weights, and the per-expert scale table of the stand-in expert op.  It holds
none of the path's arithmetic (no layout, no quantisation, no reduction), so
both the CUDA path and the CPU oracle can take their inputs from it.

The workloads follow the DeepSeek-V3 shape the pages benchmark: 8K tokens per
batch, hidden 7168, FP8 dispatch and BF16 combine ("DeepEP v2 release" notes on
donniechu.com, section "Số liệu kỹ thuật"), with 256 experts and top-8 routing
("DeepEP 编址服务深度对抗分析", section 五.2).  The pages use no dataset; the
router logits here are N(0,1) draws that stand in for a trained router.

Generation order inside one workload (all from ``numpy.random.default_rng(seed)``,
PCG64): hidden states first, then the routing draws, then the weights.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = ["CONFIGS", "Workload", "make_workload", "make_x", "make_x_fp16", "make_x_scale_sweep",
           "route", "expert_scale_table", "random_topk"]

# name -> shape and recipe.  fmt is the dispatch format; combine is BF16 always.
CONFIGS = {
    # 128 tokens, H=256, 16 experts over 4 ranks, top-2 of softmax(N(0,1)),
    # weights renormalised, BF16 dispatch, identity expert.
    "tiny": dict(T=128, H=256, E=16, R=4, k=2, routing="softmax_topk", fmt="bf16",
                 expert="identity"),
    # Decode-style small batch: group-limited top-8 of 256, 16 ranks, FP8.
    "decode": dict(T=128, H=7168, E=256, R=16, k=8, routing="group_limited", fmt="fp8",
                   expert="scale"),
    # DeepSeek-V3 prefill shape: 4096 tokens, 8 ranks, FP8.
    "dsv3": dict(T=4096, H=7168, E=256, R=8, k=8, routing="group_limited", fmt="fp8",
                 expert="scale"),
    # The pages' 8K batch, uniform distinct top-8, Dirichlet(1) weights, BF16.
    "8k": dict(T=8192, H=7168, E=256, R=8, k=8, routing="uniform", fmt="bf16",
               expert="scale"),
    # Skewed: Zipf(1.2) popularity over a seeded permutation, 32 ranks, FP8.
    "skewed": dict(T=8192, H=7168, E=256, R=32, k=8, routing="zipf", fmt="fp8",
                   expert="scale"),
}


@dataclass
class Workload:
    name: str
    T: int
    H: int
    E: int
    R: int
    k: int
    fmt: str                 # "bf16" or "fp8" dispatch
    seed: int
    x_bits: np.ndarray       # uint16 [T, H]: bf16 bit patterns
    topk_idx: np.ndarray     # int64 [T, k]
    topk_weights: np.ndarray  # float32 [T, k]
    expert_c: np.ndarray     # float32 [E]: stand-in expert op y = c[e] * x
    block_m: int = 128
    meta: dict = field(default_factory=dict)


def _bf16_bits_rn(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns with round-to-nearest-even (input drawing only)."""
    import torch  # local: a library cast, used to make inputs

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def make_x(T: int, H: int, rng: np.random.Generator) -> np.ndarray:
    """Hidden states: N(0,1) in fp32, rounded to bf16 (RN-even); returned as bits."""
    return _bf16_bits_rn(rng.standard_normal((T, H), dtype=np.float32))


def make_x_fp16(T: int, H: int, rng: np.random.Generator) -> np.ndarray:
    """Hidden states for FP16 inputs: N(0,1) in fp32, cast to IEEE binary16 by NumPy;
    returned as bits."""
    return rng.standard_normal((T, H), dtype=np.float32).astype(np.float16).view(np.uint16)


def make_x_scale_sweep(T: int, H: int, rng: np.random.Generator, fmt: str = "bf16") -> np.ndarray:
    """Hidden states (bits) whose 128-channel blocks have their largest
    magnitude spread over every binade of the 16-bit format (encodings 1 to
    the largest finite one, plus, for bf16, every encoding from 0x1180 to
    0x1280, magnitudes near 448 * 2^-100); each block's other elements are
    random encodings below its largest, every sign random.  H % 128 == 0."""
    top = 0x7F7F if fmt == "bf16" else 0x7BFF
    nb = T * H // 128
    near = np.arange(0x1180, 0x1281) if fmt == "bf16" else np.zeros(0, np.int64)
    spread = np.linspace(1, top, max(nb - near.size, 1)).astype(np.int64)
    amax = np.concatenate([spread, near])[:nb]
    rng.shuffle(amax)
    blocks = (rng.random((nb, 128)) * (amax[:, None] + 1)).astype(np.int64)
    blocks[np.arange(nb), rng.integers(0, 128, nb)] = amax
    blocks |= rng.integers(0, 2, (nb, 128)) << 15
    return blocks.astype(np.uint16).reshape(T, H)


def expert_scale_table(E: int, identity: bool = False) -> np.ndarray:
    """c[e] = fl32(1 + 0.01 e) for the stand-in expert op (ones for identity)."""
    if identity:
        return np.ones(E, np.float32)
    return (1.0 + 0.01 * np.arange(E, dtype=np.float64)).astype(np.float32)


def _stable_topk_desc(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest per row, descending; ties go to the lower index."""
    order = np.argsort(-scores, axis=1, kind="stable")
    return order[:, :k]


def route(kind: str, T: int, E: int, k: int, rng: np.random.Generator):
    """Router draws -> (topk_idx int64 [T, k], topk_weights float32 [T, k])."""
    if kind == "softmax_topk":
        logits = rng.standard_normal((T, E))
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        idx = _stable_topk_desc(p, k)
        w = np.take_along_axis(p, idx, axis=1)
        w = w / w.sum(axis=1, keepdims=True)
    elif kind == "group_limited":
        # DeepSeek-V3 style: sigmoid scores, 8 groups of E/8 experts, group
        # score = sum of its top-2 scores, keep the top-4 groups, then top-k
        # experts among the kept ones; weights are the chosen scores
        # normalised to sum 1.
        assert E % 8 == 0
        s = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, E))))
        g = s.reshape(T, 8, E // 8)
        top2 = -np.sort(-g, axis=2)[:, :, :2].sum(axis=2)
        keep = _stable_topk_desc(top2, 4)
        mask = np.zeros((T, 8), bool)
        np.put_along_axis(mask, keep, True, axis=1)
        masked = np.where(np.repeat(mask, E // 8, axis=1), s, -np.inf)
        idx = _stable_topk_desc(masked, k)
        w = np.take_along_axis(s, idx, axis=1)
        w = w / w.sum(axis=1, keepdims=True)
    elif kind == "uniform":
        u = rng.random((T, E))
        idx = np.argsort(u, axis=1, kind="stable")[:, :k]
        w = rng.dirichlet(np.ones(k), size=T)
    elif kind == "zipf":
        perm = rng.permutation(E)
        p = np.empty(E)
        p[perm] = (np.arange(E) + 1.0) ** -1.2
        p /= p.sum()
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]) if T else \
            np.zeros((0, k), np.int64)
        z = rng.standard_normal((T, k))
        w = np.exp(z - z.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
    else:
        raise ValueError("unknown routing kind %r" % kind)
    return (np.ascontiguousarray(idx, dtype=np.int64),
            np.ascontiguousarray(w, dtype=np.float32))


def make_workload(name: str, seed: int = 0, T: int | None = None, H: int | None = None) -> Workload:
    """One of the named configs; T and H may be overridden for smaller parity cases."""
    cfg = dict(CONFIGS[name])
    if T is not None:
        cfg["T"] = T
    if H is not None:
        cfg["H"] = H
    rng = np.random.default_rng(seed)
    x = make_x(cfg["T"], cfg["H"], rng)
    idx, w = route(cfg["routing"], cfg["T"], cfg["E"], cfg["k"], rng)
    c = expert_scale_table(cfg["E"], identity=(cfg["expert"] == "identity"))
    return Workload(name=name, T=cfg["T"], H=cfg["H"], E=cfg["E"], R=cfg["R"], k=cfg["k"],
                    fmt=cfg["fmt"], seed=seed, x_bits=x, topk_idx=idx, topk_weights=w,
                    expert_c=c, meta=dict(routing=cfg["routing"], expert=cfg["expert"]))


def random_topk(T: int, E: int, k: int, rng: np.random.Generator, distinct: bool = True,
                p_unused: float = 0.0):
    """Fuzz routing: uniform experts (distinct per token unless told otherwise),
    a fraction p_unused of slots set to -1, weights U(0,1)."""
    if distinct and k <= E:
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    else:
        idx = rng.integers(0, E, size=(T, k))
    idx = idx.astype(np.int64)
    if p_unused > 0:
        idx[rng.random((T, k)) < p_unused] = -1
    w = rng.random((T, k)).astype(np.float32)
    return np.ascontiguousarray(idx), np.ascontiguousarray(w)
