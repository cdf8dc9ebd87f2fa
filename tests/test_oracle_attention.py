"""Pins of the oracle's sparse attention and mode schedule (CPU only)."""
import numpy as np
import torch

from oracle import csa2_ref as R


def test_dense_case_matches_torch_sdpa():
    """All rows selected and no window: textbook softmax attention with one KV head."""
    rng = np.random.default_rng(1)
    H, D, n = 8, 32, 50
    q = rng.standard_normal((H, D))
    kv = rng.standard_normal((n, D))
    scale = 1.0 / np.sqrt(D)
    out, lse = R.sparse_attention(q, kv, np.zeros((0, D)), scale)
    qt = torch.from_numpy(q)[None, :, None, :]                 # [1, H, 1, D]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, n, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=scale)
    np.testing.assert_allclose(out, ref[0, :, 0].numpy(), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(scale * torch.from_numpy(q) @ torch.from_numpy(kv).T, dim=1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def test_single_row_returns_the_row():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 16))
    row = rng.standard_normal((1, 16))
    out, lse = R.sparse_attention(q, row, np.zeros((0, 16)), 0.25)
    np.testing.assert_allclose(out, np.repeat(row, 4, 0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.25 * (q @ row[0]), atol=1e-15)


def test_uniform_logits_give_the_mean():
    rng = np.random.default_rng(3)
    kv = rng.standard_normal((10, 16))
    win = rng.standard_normal((5, 16))
    out, lse = R.sparse_attention(np.zeros((3, 16)), kv, win, 1.0)
    np.testing.assert_allclose(out, np.repeat(np.concatenate([kv, win]).mean(0)[None], 3, 0),
                               atol=1e-14)
    np.testing.assert_allclose(lse, np.log(15.0), atol=1e-14)


def test_joint_softmax_is_one_softmax_over_the_union():
    """Moving rows between the selected set and the window changes nothing."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal((6, 8))
    rows = rng.standard_normal((20, 8))
    a = R.sparse_attention(q, rows[:12], rows[12:], 0.3)
    b = R.sparse_attention(q, rows[:3], rows[3:], 0.3)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)


def test_window_positions():
    assert list(R.window_positions(5, 128)) == list(range(0, 6))
    assert list(R.window_positions(1000, 128)) == list(range(873, 1001))


def test_reuse_equals_full_with_identical_indices():
    """Reuse runs no indexer: it attends with the latest indices and its own Q / window,
    which is exactly what a Full layer with those indices computes."""
    rng = np.random.default_rng(5)
    n, D, H = 300, 32, 4
    x = rng.standard_normal((n, D)).astype(np.float32)
    codes, scales = R.quantize_rows(x)
    deq = R.dequantize_rows(codes, scales)
    qI, w = rng.integers(-8, 9, (2, 16)), rng.integers(1, 5, 2)
    kI = rng.integers(-8, 9, (n, 16))
    full_idx = R.layer_indices("full", scores_full=R.index_scores(qI, w, kI), k=32)
    reuse_idx = R.layer_indices("reuse", latest=full_idx, k=32)
    q2 = rng.standard_normal((H, D))
    win = rng.standard_normal((7, D))
    a = R.sparse_attention(q2, deq[reuse_idx[reuse_idx >= 0]], win, D ** -0.5)
    b = R.sparse_attention(q2, deq[full_idx[full_idx >= 0]], win, D ** -0.5)
    np.testing.assert_array_equal(a[0], b[0])


def test_reuse_after_reindex_takes_reindex_indices():
    rng = np.random.default_rng(6)
    n = 400
    kI = rng.integers(-8, 9, (n, 16))
    q1, w1 = rng.integers(-8, 9, (2, 16)), rng.integers(1, 5, 2)
    q2, w2 = rng.integers(-8, 9, (2, 16)), rng.integers(1, 5, 2)
    s1 = R.index_scores(q1, w1, kI)
    pool = R.build_pool(s1, 16, 8)
    ri = R.layer_indices("reindex", qI=q2, w=w2, kI_rows=kI, pool=pool, k=20, visible=n)
    ru = R.layer_indices("reuse", latest=ri, k=20)
    assert ru is ri
    assert set(ri[ri >= 0]) <= set(R.pool_positions(pool, 8, n))
