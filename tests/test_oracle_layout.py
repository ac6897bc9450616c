"""Pins for the oracle's dispatch layout.

The layout (counts, padded expert-major offsets, is_token_in_rank, the
destination row of every (token, slot) and the source token of every receive
row) is checked against
  * a hand-worked example (tests/golden/layout_hand_example.txt),
  * an independent derivation with Python's stable ``sorted`` (brute force),
  * invariants that hold for any input: counts sum to the used slots, the slot
    map is a bijection onto the non-pad rows, order inside an expert block is
    by source token then slot, rank bookkeeping agrees with is_token_in_rank,
  * closed-form special cases (one hot expert, round robin, T = 0, E = R, k = 1).
"""
import os

import numpy as np
import pytest

from workloads import random_topk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            d[key.strip()] = [int(v) for v in val.split()]
    return d


def pad(c, b):
    return -(-c // b) * b


def brute_force_layout(topk_idx, E, R, B):
    """Independent derivation: stable-sort the used slots by expert."""
    T, k = topk_idx.shape
    slots = [(int(topk_idx[t, j]), t, j) for t in range(T) for j in range(k) if topk_idx[t, j] >= 0]
    slots = sorted(slots, key=lambda s: s[0])  # stable: keeps (t, j) order inside an expert
    cnt = np.bincount([s[0] for s in slots], minlength=E).astype(np.int64)
    off = np.concatenate([[0], np.cumsum([pad(c, B) for c in cnt])])
    dst = -np.ones((T, k), np.int64)
    seen = {}
    for e, t, j in slots:
        i = seen.get(e, 0)
        dst[t, j] = off[e] + i
        seen[e] = i + 1
    return cnt, off, dst


def check_invariants(lay, topk_idx, E, R, B):
    T, k = topk_idx.shape
    epr = E // R
    valid = topk_idx >= 0
    cnt = lay.num_tokens_per_expert.astype(np.int64)
    off = lay.expert_off.astype(np.int64)
    assert cnt.sum() == valid.sum()
    sizes = np.diff(off)
    assert np.all(sizes % B == 0) and np.all(sizes >= cnt) and np.all(sizes - cnt < B)
    assert np.all((cnt == 0) == (sizes == 0))
    assert lay.total_rows == off[-1]
    assert np.array_equal(lay.rank_off, off[::epr])
    # bijection of used slots onto the non-pad rows
    rows = lay.dst_row[valid].astype(np.int64)
    assert np.all(lay.dst_row[~valid] == -1)
    assert len(np.unique(rows)) == rows.size
    nonpad = np.concatenate([np.arange(off[e], off[e] + cnt[e]) for e in range(E)]) if E else []
    assert np.array_equal(np.sort(rows), np.asarray(nonpad, np.int64))
    # each slot lands in its own expert's block
    row_expert = np.searchsorted(off, rows, side="right") - 1
    assert np.array_equal(row_expert, topk_idx[valid])
    # recv_src and order inside a block: by source token, then slot
    t_of = np.repeat(np.arange(T), k).reshape(T, k)
    assert np.array_equal(lay.recv_src[rows], t_of[valid])
    pad_rows = np.setdiff1d(np.arange(lay.total_rows), rows)
    assert np.all(lay.recv_src[pad_rows] == -1)
    j_of = np.tile(np.arange(k), T).reshape(T, k)
    key = np.full(lay.total_rows, -1, np.int64)
    key[rows] = t_of[valid] * k + j_of[valid]
    for e in range(E):
        blk = key[off[e]: off[e] + cnt[e]]
        assert np.all(np.diff(blk) > 0)
    # rank bookkeeping
    itr = np.zeros((T, R), np.uint8)
    for t in range(T):
        for j in range(k):
            if topk_idx[t, j] >= 0:
                itr[t, topk_idx[t, j] // epr] = 1
    assert np.array_equal(lay.is_token_in_rank, itr)
    assert np.array_equal(lay.num_tokens_per_rank, itr.sum(axis=0))
    assert np.array_equal(lay.num_rows_per_rank, cnt.reshape(R, epr).sum(axis=1))


def test_hand_worked_example(oracle):
    g = _read_golden("layout_hand_example.txt")
    T, k, E, R, B = g["T"][0], g["k"][0], g["E"][0], g["R"][0], g["block_m"][0]
    idx = np.array(g["topk_idx"], np.int64).reshape(T, k)
    lay = oracle.layout(idx, E, R, B)
    assert lay.num_tokens_per_expert.tolist() == g["num_tokens_per_expert"]
    assert lay.expert_off.tolist() == g["expert_off"]
    assert lay.rank_off.tolist() == g["rank_off"]
    assert lay.num_rows_per_rank.tolist() == g["num_rows_per_rank"]
    assert lay.num_tokens_per_rank.tolist() == g["num_tokens_per_rank"]
    assert lay.is_token_in_rank.reshape(-1).tolist() == g["is_token_in_rank"]
    assert lay.dst_row.reshape(-1).tolist() == g["dst_row"]
    assert lay.recv_src.tolist() == g["recv_src"]
    assert lay.total_rows == g["total_rows"][0]
    check_invariants(lay, idx, E, R, B)


@pytest.mark.parametrize("T,E,R,k,B,p_unused,distinct", [
    (1, 4, 2, 2, 4, 0.0, True),
    (7, 8, 4, 3, 2, 0.0, True),
    (33, 16, 4, 2, 128, 0.1, True),
    (100, 32, 8, 8, 16, 0.0, True),
    (100, 32, 8, 8, 16, 0.0, False),   # duplicate experts inside a token
    (257, 64, 64, 4, 1, 0.3, True),    # E = R, block_m = 1 (no padding)
    (64, 256, 8, 8, 128, 0.05, True),
    (50, 5, 1, 5, 3, 0.2, True),       # one rank, k = E
])
def test_random_vs_brute_force_and_invariants(oracle, T, E, R, k, B, p_unused, distinct):
    rng = np.random.default_rng(T * 1000 + E)
    idx, _ = random_topk(T, E, k, rng, distinct=distinct, p_unused=p_unused)
    lay = oracle.layout(idx, E, R, B)
    cnt, off, dst = brute_force_layout(idx, E, R, B)
    assert np.array_equal(lay.num_tokens_per_expert, cnt)
    assert np.array_equal(lay.expert_off, off)
    assert np.array_equal(lay.dst_row, dst)
    check_invariants(lay, idx, E, R, B)


def test_all_tokens_to_one_expert(oracle):
    T, k, E, R, B = 300, 1, 16, 4, 128
    idx = np.full((T, k), 5, np.int64)
    lay = oracle.layout(idx, E, R, B)
    assert lay.total_rows == pad(T, B) == 384
    assert lay.dst_row[:, 0].tolist() == list(range(T))
    assert lay.num_tokens_per_rank.tolist() == [0, T, 0, 0]
    assert lay.num_rows_per_rank.tolist() == [0, T, 0, 0]
    assert lay.expert_off[:6].tolist() == [0] * 6 and lay.expert_off[6:].tolist() == [384] * 11


def test_round_robin_equal_counts(oracle):
    T, k, E, R, B = 64, 4, 16, 4, 8
    idx = (np.arange(T * k, dtype=np.int64) % E).reshape(T, k)
    lay = oracle.layout(idx, E, R, B)
    assert np.all(lay.num_tokens_per_expert == T * k // E)
    assert lay.total_rows == E * pad(T * k // E, B)
    # slot (t, j) is the (t*k + j) // E -th arrival of its expert
    f = np.arange(T * k)
    assert np.array_equal(lay.dst_row.reshape(-1), lay.expert_off[f % E] + f // E)


def test_empty_batch(oracle):
    lay = oracle.layout(np.zeros((0, 8), np.int64), 256, 8, 128)
    assert lay.total_rows == 0
    assert np.all(lay.num_tokens_per_expert == 0) and np.all(lay.expert_off == 0)
    assert lay.dst_row.shape == (0, 8) and lay.recv_src.size == 0


def test_all_slots_unused(oracle):
    lay = oracle.layout(np.full((10, 3), -1, np.int64), 8, 2, 4)
    assert lay.total_rows == 0 and np.all(lay.dst_row == -1)
    assert np.all(lay.is_token_in_rank == 0)


def test_bad_index_is_rejected(oracle):
    idx = np.array([[0, 1], [2, 16]], np.int64)
    with pytest.raises(oracle.OracleError) as ei:
        oracle.layout(idx, 16, 4, 128)
    assert ei.value.code == oracle.ERR_BAD_INDEX
    with pytest.raises(oracle.OracleError):
        oracle.layout(np.array([[-2]], np.int64), 16, 4, 128)


def test_recv_rows_bound(oracle):
    rng = np.random.default_rng(3)
    for _ in range(20):
        T = int(rng.integers(0, 200))
        E = int(rng.choice([4, 16, 64, 256]))
        k = int(rng.integers(1, min(E, 8) + 1))
        B = int(rng.choice([1, 16, 128]))
        idx, _ = random_topk(T, E, k, rng)
        lay = oracle.layout(idx, E, 1, B)
        bound = oracle.recv_rows_bound(T, k, E, B)
        assert lay.total_rows <= bound and bound % B == 0
    # the bound is reached when every slot opens its own block
    assert oracle.recv_rows_bound(4, 2, 8, 128) == 8 * 128


def test_tiny_config_sizes(oracle):
    """The named configs give the sizes the design is built around."""
    from workloads import make_workload

    w = make_workload("tiny", 0)
    lay = oracle.layout(w.topk_idx, w.E, w.R)
    assert lay.num_tokens_per_expert.sum() == w.T * w.k == 256
    assert lay.total_rows == 2048  # 16 experts, each one block of 128
    check_invariants(lay, w.topk_idx, w.E, w.R, 128)
