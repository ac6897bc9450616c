"""ep_layout_static_scratch: the dispatch layout for callers that cannot
allocate device memory (a framework or pre-reserved memory pool that forbids
more cudaMalloc calls, plug-ins that receive only input and output pointers).
It keeps its scratch in a fixed array inside the library, so the caller passes
nothing but inputs and outputs.

Checked here through the C ABI, bit-exact (the layout is integer work, as in
the other layout tests): every output field against the oracle, and two calls
in a row (the array keeps the first call's contents when the second runs)
against the workspace entry point ep_layout on the same input.  The cases
cover each kernel path the entry point can take: the three-kernel path (large
batches, and E = 8192), the one-CTA small-batch kernel, and the empty batch.
Sizes beyond the fixed scratch are rejected before anything is enqueued.  This
file runs last so that a failure here leaves every other test already run; it
also passes when run alone in a fresh process (the first call does the
per-device set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from workloads import make_workload, random_topk

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
STATIC_SCRATCH_BYTES = 4 << 20


def _lib():
    import combine_ep_layout_08_b200 as ep
    from combine_ep_layout_08_b200 import _build

    _build.build()
    lib = ep.load_library()
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn = lib.ep_layout_static_scratch
    fn.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, I64, P, P]
    fn.restype = I
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr() if t.numel() else 0)


def static_layout(lib, idx, E, R, B=128):
    import combine_ep_layout_08_b200 as ep

    T, k = idx.shape
    cap = max(ep.ep_recv_rows_upper_bound(T, k, E, B), 1)
    o = dict(
        num_tokens_per_expert=torch.full((E,), -7, dtype=torch.int32, device=DEV),
        num_tokens_per_rank=torch.full((R,), -7, dtype=torch.int32, device=DEV),
        num_rows_per_rank=torch.full((R,), -7, dtype=torch.int32, device=DEV),
        expert_off=torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
        rank_off=torch.full((R + 1,), -7, dtype=torch.int32, device=DEV),
        total=torch.full((1,), -7, dtype=torch.int32, device=DEV),
        is_token_in_rank=torch.full((T, R), 7, dtype=torch.uint8, device=DEV),
        dst_row=torch.full((T, k), -7, dtype=torch.int32, device=DEV),
        recv_src=torch.full((cap,), -7, dtype=torch.int32, device=DEV),
        err=torch.full((1,), 99, dtype=torch.int32, device=DEV),
    )
    d_idx = torch.from_numpy(idx).to(DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.ep_layout_static_scratch(
        _p(d_idx), T, k, E, R, B, _p(o["num_tokens_per_expert"]), _p(o["num_tokens_per_rank"]),
        _p(o["num_rows_per_rank"]), _p(o["expert_off"]), _p(o["rank_off"]), _p(o["total"]),
        _p(o["is_token_in_rank"]), _p(o["dst_row"]), _p(o["recv_src"]), cap, _p(o["err"]),
        stream)
    assert st == 0, "ep_layout_static_scratch returned %d" % st
    torch.cuda.synchronize()
    out = {key: v.cpu().numpy() for key, v in o.items()}
    out["recv_src"] = out["recv_src"][: int(out["total"][0])]
    return out


def workspace_layout(idx, E, R, B=128):
    import combine_ep_layout_08_b200 as ep

    T, k = idx.shape
    h = ep.ep_handle_create(max(T, 1), k, E, R, B, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    P = int(ep.ep_handle_view(h, "total_recv_rows").item())
    out = {name: ep.ep_handle_view(h, name).cpu().numpy() for name in (
        "num_tokens_per_expert", "num_tokens_per_rank", "num_rows_per_rank", "expert_off",
        "rank_off", "is_token_in_rank", "dst_row")}
    out["total"] = np.array([P], np.int32)
    out["recv_src"] = ep.ep_handle_view(h, "recv_src")[:P].cpu().numpy()
    out["err"] = np.array([ep.ep_handle_check(h, raise_on_error=False)], np.int32)
    return out


def _same(a, b):
    for key in ("num_tokens_per_expert", "num_tokens_per_rank", "num_rows_per_rank",
                "expert_off", "rank_off", "is_token_in_rank", "dst_row", "total", "recv_src"):
        assert np.array_equal(a[key], b[key]), key


def _same_as_oracle(a, lay):
    """Every output field against the oracle's layout of the same input."""
    for key in ("num_tokens_per_expert", "num_tokens_per_rank", "num_rows_per_rank",
                "expert_off", "rank_off", "is_token_in_rank", "dst_row", "recv_src"):
        exp = getattr(lay, key)
        assert a[key].shape == exp.shape, (key, a[key].shape, exp.shape)
        assert np.array_equal(a[key], exp), key
    assert int(a["total"][0]) == lay.total_rows


def test_two_calls_in_a_row_match_the_workspace_entry_point(oracle):
    lib = _lib()
    w1 = make_workload("8k", 0, H=128)                      # 8192 tokens, 8 ranks
    w2 = make_workload("skewed", 0, T=3000, H=128)          # fewer tokens, 32 ranks
    a1 = static_layout(lib, w1.topk_idx, w1.E, w1.R)
    a2 = static_layout(lib, w2.topk_idx, w2.E, w2.R)        # reuses the array
    assert a1["err"][0] == 0 and a2["err"][0] == 0
    _same_as_oracle(a1, oracle.layout(w1.topk_idx, w1.E, w1.R))
    _same_as_oracle(a2, oracle.layout(w2.topk_idx, w2.E, w2.R))
    _same(a1, workspace_layout(w1.topk_idx, w1.E, w1.R))
    _same(a2, workspace_layout(w2.topk_idx, w2.E, w2.R))


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_small_batches_match_the_oracle(oracle, name):
    """T k <= 4096: the one-CTA small-batch kernel, no bad index."""
    lib = _lib()
    w = make_workload(name, 0, H=128)
    a = static_layout(lib, w.topk_idx, w.E, w.R)
    assert a["err"][0] == 0
    _same_as_oracle(a, oracle.layout(w.topk_idx, w.E, w.R))
    _same(a, workspace_layout(w.topk_idx, w.E, w.R))


def test_largest_expert_count_matches_the_oracle(oracle):
    """E = 8192: the three-kernel path with a wide count matrix that still fits
    the static array (4 * ceil(2000/32) * (8192 + 8) bytes)."""
    lib = _lib()
    idx, _ = random_topk(2000, 8192, 8, np.random.default_rng(11), p_unused=0.05)
    a = static_layout(lib, idx, 8192, 8)
    assert a["err"][0] == 0
    _same_as_oracle(a, oracle.layout(idx, 8192, 8))


def test_empty_batch_matches_the_oracle(oracle):
    lib = _lib()
    idx = np.zeros((0, 8), np.int64)
    a = static_layout(lib, idx, 256, 8)
    assert a["err"][0] == 0 and int(a["total"][0]) == 0
    _same_as_oracle(a, oracle.layout(idx, 256, 8))


def test_bad_index_sets_the_error_word(oracle):
    lib = _lib()
    idx, _ = random_topk(100, 64, 4, np.random.default_rng(2))
    idx[7, 2] = 64
    a = static_layout(lib, idx, 64, 8)
    assert a["err"][0] == 1  # the bad-index bit
    idx[7, 2] = -1                                          # a bad index counts as unused
    _same_as_oracle(a, oracle.layout(idx, 64, 8))
    _same(a, workspace_layout(idx, 64, 8))


def test_sizes_beyond_the_static_scratch_are_rejected():
    import combine_ep_layout_08_b200 as ep

    lib = _lib()
    # 4 * ceil(T/32) * (E + R) > 4 MiB: T = 131072 tokens, E = 256, R = 8
    T, k, E, R = 131072, 8, 256, 8
    assert 4 * (T // 32) * (E + R) > STATIC_SCRATCH_BYTES
    P = ctypes.c_void_p
    fake = P(0x7f0000000000)
    st = lib.ep_layout_static_scratch(fake, T, k, E, R, 128, fake, fake, fake, fake, fake, fake,
                                      fake, fake, fake, 1 << 30, fake, None)
    assert st == ep.EP_ERR_WORKSPACE_TOO_SMALL
