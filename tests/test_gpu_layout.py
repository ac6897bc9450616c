"""GPU parity of ep_layout against the oracle: bit-exact on every config and
on fuzzed shapes, plus the edge cases (empty batch, ragged chunk tails,
unused slots, duplicates, E = R, k = 1 and k = 32, block_m = 1, large E, bad
indices)."""
import numpy as np
import pytest
import torch

from workloads import make_workload, random_topk

pytestmark = pytest.mark.gpu


def _run(idx_np, E, R, B=128, T_max=None):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, gpu_layout

    T, k = idx_np.shape
    h = ep.ep_handle_create(T_max if T_max is not None else T, k, E, R, B, device=DEV)
    ep.ep_layout(h, torch.from_numpy(idx_np).to(DEV))
    g = gpu_layout(h)
    st = ep.ep_handle_check(h, raise_on_error=False)
    return g, st, h


@pytest.mark.parametrize("name,seeds", [("tiny", range(5)), ("decode", range(5)),
                                        ("dsv3", range(2)), ("8k", [0]), ("skewed", [0, 1])])
def test_layout_configs_bit_exact(oracle, name, seeds):
    from gpu_util import assert_layout_equal

    for seed in seeds:
        w = make_workload(name, seed, H=128)  # layout does not look at H
        g, st, _ = _run(w.topk_idx, w.E, w.R)
        assert st == 0
        assert_layout_equal(g, oracle.layout(w.topk_idx, w.E, w.R))


FUZZ = [
    # T, E, R, k, B, p_unused, distinct
    (1, 4, 2, 2, 4, 0.0, True),
    (31, 16, 4, 2, 128, 0.0, True),
    (33, 16, 4, 2, 128, 0.2, True),
    (1000, 64, 8, 6, 16, 0.1, True),
    (777, 32, 32, 8, 1, 0.0, True),        # E = R, no padding
    (500, 8, 1, 8, 128, 0.0, False),       # duplicates, one rank
    (300, 256, 16, 1, 128, 0.0, True),     # k = 1
    (129, 64, 4, 32, 64, 0.05, True),      # k = 32 (maximum)
    (2000, 2048, 64, 8, 128, 0.0, True),   # large E
    (64, 8192, 8192, 4, 128, 0.0, True),   # maximum E, R = E
    (4096, 256, 256, 8, 128, 0.5, True),   # many unused slots
    (200, 64, 8, 6, 16, 0.1, True),        # small batch, k does not divide 32
    (150, 40, 5, 20, 8, 0.1, True),        # small batch, three rounds of 1024 entries
    (100, 1024, 8, 9, 128, 0.0, False),    # small batch, E = 1024, duplicates
    (20000, 256, 8, 8, 128, 0.0, True),    # many chunks
    (512, 256, 16, 8, 128, 0.1, True),     # 4096 entries: the one-CTA path's limit
    (513, 256, 16, 8, 128, 0.0, True),     # 4104 entries: the tiled path
    (400, 1024, 64, 8, 128, 0.0, True),    # one-CTA path at its largest E
    (300, 1024, 1024, 4, 128, 0.0, True),  # T x R too many bytes for one CTA: tiled
    (1000, 2048, 8, 8, 128, 0.0, True),    # E above the one-CTA limit
    (5000, 8192, 64, 4, 128, 0.0, True),   # tile counts too big for shared memory: 3 kernels
    (3000, 256, 8, 8, 3, 0.1, True),       # block_m = 3: pad ranges not 4-aligned
    (40000, 256, 8, 8, 128, 0.02, True),   # tile layout, 34 tokens per warp (> 32)
    (2000, 20, 4, 4, 16, 0.1, True),       # tile layout, E not a multiple of 8
    (9000, 1024, 16, 6, 128, 0.0, True),   # tile layout at E = 1024, k = 6
    (150000, 64, 8, 2, 128, 0.0, True),    # tile layout, 127 tokens per warp, 13 groups
]


@pytest.mark.parametrize("T,E,R,k,B,p_unused,distinct", FUZZ)
def test_layout_fuzz_bit_exact(oracle, T, E, R, k, B, p_unused, distinct):
    from gpu_util import assert_layout_equal

    rng = np.random.default_rng(T + 7 * E + k)
    idx, _ = random_topk(T, E, k, rng, distinct=distinct, p_unused=p_unused)
    g, st, _ = _run(idx, E, R, B)
    assert st == 0
    assert_layout_equal(g, oracle.layout(idx, E, R, B))


def test_layout_hot_expert_and_round_robin(oracle):
    from gpu_util import assert_layout_equal

    T, k, E, R = 5000, 4, 64, 8
    idx = np.full((T, k), 17, np.int64)
    idx[:, 1:] = (np.arange(T * (k - 1)) % E).reshape(T, k - 1)
    g, st, _ = _run(idx, E, R)
    assert st == 0
    assert_layout_equal(g, oracle.layout(idx, E, R))


def test_layout_empty_batch(oracle):
    from gpu_util import assert_layout_equal

    idx = np.zeros((0, 8), np.int64)
    g, st, _ = _run(idx, 256, 8, T_max=64)
    assert st == 0 and g["total_rows"] == 0
    assert_layout_equal(g, oracle.layout(idx, 256, 8))


def test_layout_reuse_smaller_batch(oracle):
    """A handle sized for many tokens serves a smaller batch; the second
    layout replaces the first."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, assert_layout_equal, gpu_layout

    rng = np.random.default_rng(5)
    h = ep.ep_handle_create(4096, 8, 256, 8, device=DEV)
    for T in (4096, 100, 37):
        idx, _ = random_topk(T, 256, 8, rng)
        ep.ep_layout(h, torch.from_numpy(idx).to(DEV))
        assert_layout_equal(gpu_layout(h), oracle.layout(idx, 256, 8))
        assert ep.ep_handle_check(h, raise_on_error=False) == 0


def test_layout_bad_index_sets_error_and_is_skipped(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import assert_layout_equal

    rng = np.random.default_rng(9)
    idx, _ = random_topk(200, 64, 4, rng)
    bad = idx.copy()
    bad[3, 1] = 64
    bad[150, 0] = -5
    g, st, h = _run(bad, 64, 8)
    assert st == ep.EP_ERR_BAD_INDEX
    clean = bad.copy()
    clean[3, 1] = -1
    clean[150, 0] = -1
    assert_layout_equal(g, oracle.layout(clean, 64, 8))
    # the error word is cleared by the check
    assert ep.ep_handle_check(h, raise_on_error=False) == 0


def test_layout_bad_index_large_batch(oracle):
    import combine_ep_layout_08_b200 as ep
    from gpu_util import assert_layout_equal

    rng = np.random.default_rng(19)
    idx, _ = random_topk(3000, 256, 8, rng)
    bad = idx.copy()
    bad[2999, 7] = 1 << 40
    bad[1234, 0] = -2
    g, st, _ = _run(bad, 256, 8)
    assert st == ep.EP_ERR_BAD_INDEX
    clean = bad.copy()
    clean[2999, 7] = -1
    clean[1234, 0] = -1
    assert_layout_equal(g, oracle.layout(clean, 256, 8))


def test_layout_counts_readback(oracle):
    import combine_ep_layout_08_b200 as ep

    w = make_workload("dsv3", 0, H=128)
    _, _, h = _run(w.topk_idx, w.E, w.R)
    c = ep.ep_handle_read_counts(h)
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    assert np.array_equal(c["num_tokens_per_expert"], lay.num_tokens_per_expert)
    assert np.array_equal(c["num_tokens_per_rank"], lay.num_tokens_per_rank)
    assert np.array_equal(c["num_rows_per_rank"], lay.num_rows_per_rank)
    assert c["total_recv_rows"] == lay.total_rows


def test_layout_deterministic():
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, gpu_layout

    w = make_workload("skewed", 0, H=128)
    h = ep.ep_handle_create(w.T, w.k, w.E, w.R, device=DEV)
    idx = torch.from_numpy(w.topk_idx).to(DEV)
    ep.ep_layout(h, idx)
    a = gpu_layout(h)
    ep.ep_layout(h, idx)
    b = gpu_layout(h)
    for key in a:
        assert np.array_equal(np.asarray(a[key]), np.asarray(b[key])), key


def test_barrier_timeout_is_reported_and_recovered(oracle):
    """The cooperative layout's grid barrier has an iteration limit.  Make it
    run out on purpose (an arrival count that can never complete), check the
    status, then check that the handle works again after ep_handle_check."""
    import combine_ep_layout_08_b200 as ep
    from gpu_util import DEV, assert_layout_equal, gpu_layout

    rng = np.random.default_rng(23)
    idx, _ = random_topk(4096, 256, 8, rng)   # 128 chunks: the cooperative path
    d_idx = torch.from_numpy(idx).to(DEV)
    h = ep.ep_handle_create(4096, 8, 256, 8, device=DEV)
    ep.ep_layout(h, d_idx)
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    words = ep.ep_handle_view(h, "error_words")
    words[1] = -(1 << 30)                     # arrivals never reach the CTA count
    ep.ep_layout(h, d_idx)
    assert ep.ep_handle_check(h, raise_on_error=False) == ep.EP_ERR_TIMEOUT
    assert words.cpu().tolist() == [0, 0, 0]   # error bits and barrier reset
    ep.ep_layout(h, d_idx)                    # the barrier was reset: works again
    assert ep.ep_handle_check(h, raise_on_error=False) == 0
    assert_layout_equal(gpu_layout(h), oracle.layout(idx, 256, 8))
