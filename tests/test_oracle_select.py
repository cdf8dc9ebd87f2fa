"""Pins of the oracle's indexer score, Top-K, block pool and Reindex (CPU only)."""
import itertools

import numpy as np
import pytest

from oracle import csa2_ref as R


def brute_topk(scores, k):
    """Rank counting: i is kept iff fewer than k candidates beat it, where j beats i
    when s_j > s_i, or s_j == s_i and j < i."""
    n = len(scores)
    keep = []
    for i in range(n):
        beaten_by = sum(1 for j in range(n)
                        if scores[j] > scores[i] or (scores[j] == scores[i] and j < i))
        if beaten_by < k:
            keep.append(i)
    return keep + [-1] * (k - len(keep))


def test_topk_exhaustive_ties():
    for n in range(0, 7):
        for vals in itertools.product([0.0, 1.0, 2.0], repeat=n):
            for k in range(1, n + 3):
                got = list(R.topk_ascending(np.array(vals), k))
                assert got == brute_topk(list(vals), k), (vals, k)


def test_topk_random_with_ids():
    rng = np.random.default_rng(1)
    for _ in range(300):
        n = int(rng.integers(1, 12))
        s = rng.integers(0, 4, n).astype(np.float64)
        ids = np.sort(rng.choice(100, n, replace=False))
        k = int(rng.integers(1, 14))
        got = R.topk_ascending(s, k, ids)
        ref = [ids[i] if i >= 0 else -1 for i in brute_topk(list(s), k)]
        assert list(got) == ref


def test_index_scores_brute_force_loops():
    rng = np.random.default_rng(2)
    H_I, d_I, n = 3, 5, 7
    qI = rng.integers(-8, 9, (H_I, d_I))
    w = rng.integers(1, 5, H_I)
    kI = rng.integers(-8, 9, (n, d_I))
    got = R.index_scores(qI, w, kI)
    for e in range(n):
        tot = 0
        for h in range(H_I):
            dot = 0
            for d in range(d_I):
                dot += int(qI[h, d]) * int(kI[e, d])
            tot += int(w[h]) * max(0, dot)
        assert got[e] == tot


def test_index_scores_exact_at_full_width():
    """Integer inputs in [-8, 8], weights in [1, 4], 16 heads x 128: every score is an
    integer below 2^24, so fp32 holds it exactly."""
    rng = np.random.default_rng(3)
    qI = np.full((16, 128), 8.0)
    kI = np.concatenate([np.full((1, 128), 8.0), rng.integers(-8, 9, (50, 128))])
    w = np.full(16, 4.0)
    s = R.index_scores(qI, w, kI)
    assert s[0] == 16 * 4 * 128 * 64 == 524288 < 2 ** 24
    assert np.all(s == np.round(s)) and np.all(s.astype(np.float32) == s)


def test_block_scores_brute_force():
    rng = np.random.default_rng(4)
    for n in (1, 7, 8, 9, 23, 64):
        s = rng.integers(0, 5, n).astype(np.float64)
        b = R.block_scores(s, 8)
        assert len(b) == -(-n // 8)
        for j in range(len(b)):
            assert b[j] == max(s[p] for p in range(n) if p // 8 == j)


def test_pool_positions_partial_last_block():
    pool = np.array([0, 2, -1, -1])
    assert list(R.pool_positions(pool, 8, 20)) == list(range(0, 8)) + list(range(16, 20))


def _rand_problem(rng, n, d_I=16, H_I=4):
    kI = rng.integers(-2, 3, (n, d_I)).astype(np.float64)
    qI = rng.integers(-2, 3, (H_I, d_I)).astype(np.float64)
    w = rng.integers(1, 3, H_I).astype(np.float64)
    return qI, w, kI


def test_reindex_pool_covering_everything_equals_full_rescore():
    """A pool holding every block makes Reindex a Full re-score with the Reindex layer's Q."""
    rng = np.random.default_rng(5)
    for n in (5, 64, 203):
        qI1, w1, kI = _rand_problem(rng, n)
        qI2, w2, _ = _rand_problem(rng, n)
        nb = -(-n // 8)
        pool = R.build_pool(R.index_scores(qI1, w1, kI), nb + 3, 8)
        assert set(pool[pool >= 0]) == set(range(nb))
        for k in (1, 17, 64):
            got = R.reindex(qI2, w2, kI, pool, 8, n, k)
            want = R.topk_ascending(R.index_scores(qI2, w2, kI), k)
            np.testing.assert_array_equal(got, want)


def test_reindex_with_full_query_returns_full_topk():
    """With lowest-index tie-breaks, every block ranked above the block of a Top-K
    position p holds a distinct position ranked above p, so that block ranks < K <= P:
    re-scoring the pool with the Full layer's own Q returns exactly the Full Top-K."""
    rng = np.random.default_rng(6)
    for n, P, K in ((500, 16, 16), (1000, 40, 32), (4096, 64, 64), (333, 8, 5)):
        qI, w, kI = _rand_problem(rng, n)
        s = R.index_scores(qI, w, kI)
        pool = R.build_pool(s, P, 8)
        got = R.reindex(qI, w, kI, pool, 8, n, K)
        np.testing.assert_array_equal(got, R.topk_ascending(s, K))


def test_visible_bound_limits_everything():
    rng = np.random.default_rng(7)
    qI, w, kI = _rand_problem(rng, 100)
    s = R.index_scores(qI, w, kI[:37])
    idx = R.topk_ascending(s, 64)
    assert list(idx[:37]) == list(range(37)) and np.all(idx[37:] == -1)
    pool = R.build_pool(s, 2048, 8)
    assert list(pool[:5]) == [0, 1, 2, 3, 4] and np.all(pool[5:] == -1)
    r = R.reindex(qI, w, kI, pool, 8, 37, 64)
    assert list(r[:37]) == list(range(37)) and np.all(r[37:] == -1)
