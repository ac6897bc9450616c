"""Randomised shapes for the small-batch layout kernel and the fused
layout + dispatch launch (T k <= 4096, E <= 1024): the kernel's branches --
rounds of 1024 entries, threads per expert in the count scan, the
tokens-per-rank table (k dividing 32, R <= 128) or shared atomics, shifts or
divisions for k and block_m, empty experts and ranks, unused slots,
duplicate experts -- against the oracle, bit-exact."""
import numpy as np
import pytest
import torch

from workloads import make_x, random_topk

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        E = int(rng.choice([1, 2, 3, 8, 17, 32, 48, 64, 100, 256, 333, 512, 1000, 1024]))
        divs = [r for r in range(1, min(E, 200) + 1) if E % r == 0]
        R = int(rng.choice(divs))
        k = int(rng.choice([1, 2, 3, 4, 5, 6, 8, 9, 16, 20, 32]))
        tmax = max(1, 4096 // k)
        T = int(rng.integers(1, min(tmax, 600) + 1))
        B = int(rng.choice([1, 3, 8, 64, 128, 200]))
        distinct = bool(rng.random() < 0.7) and k <= E
        p_unused = float(rng.choice([0.0, 0.0, 0.1, 0.5]))
        if T * R > 65536:
            continue
        out.append((T, E, R, k, B, distinct, p_unused))
    return out


@pytest.mark.parametrize("T,E,R,k,B,distinct,p_unused", _shapes(40, 2026))
def test_small_layout_random_shapes(oracle, T, E, R, k, B, distinct, p_unused):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import assert_layout_equal, gpu_layout

    rng = np.random.default_rng(T * 7 + E + k)
    idx, _ = random_topk(T, E, k, rng, distinct=distinct, p_unused=p_unused)
    h = ep.ep_handle_create(T, k, E, R, B, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    assert_layout_equal(gpu_layout(h), oracle.layout(idx, E, R, B))


@pytest.mark.parametrize("T,E,R,k,B,distinct,p_unused", _shapes(16, 77))
def test_fused_layout_dispatch_random_shapes(oracle, T, E, R, k, B, distinct, p_unused):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import assert_layout_equal, bits_to_bf16, gpu_layout

    rng = np.random.default_rng(T * 11 + E + k)
    H = int(rng.choice([128, 256, 1024]))
    idx, _ = random_topk(T, E, k, rng, distinct=distinct, p_unused=p_unused)
    x = make_x(T, H, rng)
    lay = oracle.layout(idx, E, R, B)
    h = ep.ep_handle_create(T, k, E, R, B, device=DEV)
    fmt = "fp8" if rng.random() < 0.5 else "bf16"
    recv, sc = ep.ep_layout_dispatch(h, torch.from_numpy(idx).to(DEV), bits_to_bf16(x), fmt)
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    assert_layout_equal(gpu_layout(h), lay)
    rows = lay.dst_row[lay.dst_row >= 0]
    if fmt == "bf16":
        ref = oracle.dispatch_bf16(x, lay.dst_row, lay.total_rows)
        got = recv.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got[rows], ref[rows])
    else:
        q, s = oracle.dispatch_fp8(x, lay.dst_row, lay.total_rows)
        assert np.array_equal(recv.view(torch.uint8).cpu().numpy()[rows], q[rows])
        assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), s[rows].view(np.uint32))
