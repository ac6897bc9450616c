"""The seeded generators reproduce, and draw what the recipes say."""
import numpy as np
import pytest

from workloads import CONFIGS, make_workload, random_topk


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_reproducible(name):
    a = make_workload(name, 3)
    b = make_workload(name, 3)
    c = make_workload(name, 4)
    assert np.array_equal(a.x_bits, b.x_bits) and np.array_equal(a.topk_idx, b.topk_idx)
    assert np.array_equal(a.topk_weights, b.topk_weights)
    assert not np.array_equal(a.topk_idx, c.topk_idx)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_routing_statistics(name):
    T = 256 if CONFIGS[name]["T"] > 256 else None
    w = make_workload(name, 0, T=T, H=256)
    assert w.topk_idx.shape == (w.T, w.k) and w.topk_idx.dtype == np.int64
    assert w.topk_idx.min() >= 0 and w.topk_idx.max() < w.E
    for row in w.topk_idx:
        assert len(set(row.tolist())) == w.k, "experts of a token must be distinct"
    assert np.allclose(w.topk_weights.sum(axis=1), 1.0, atol=1e-6)
    assert np.all(w.topk_weights > 0)
    assert w.E % w.R == 0
    if CONFIGS[name]["routing"] == "group_limited":
        groups = w.topk_idx // (w.E // 8)
        assert max(len(set(g.tolist())) for g in groups) <= 4
        # slots are in descending score order, so weights are non-increasing
        assert np.all(np.diff(w.topk_weights, axis=1) <= 1e-7)


def test_skewed_has_hot_experts():
    w = make_workload("skewed", 0, T=2048, H=128)
    cnt = np.bincount(w.topk_idx.reshape(-1), minlength=w.E)
    assert cnt.max() > 10 * np.median(cnt)


def test_x_is_bf16_normal():
    w = make_workload("tiny", 0)
    xf = (w.x_bits.astype(np.uint32) << 16).view(np.float32)
    assert abs(xf.mean()) < 0.05 and abs(xf.std() - 1) < 0.05


def test_random_topk_unused_fraction():
    idx, wt = random_topk(1000, 32, 4, np.random.default_rng(0), p_unused=0.25)
    frac = (idx == -1).mean()
    assert 0.2 < frac < 0.3 and wt.dtype == np.float32
