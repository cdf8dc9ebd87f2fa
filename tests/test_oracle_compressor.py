"""The oracle's sequence compressor against closed forms and brute force: identity maps,
sums of token pairs, an explicit triple loop, and exactness of the synthetic inputs'
fp32 rounding (which makes the quantised entries comparable bit for bit)."""
import numpy as np

from fp4_kv_cache_03_b200 import synth
from oracle import csa2_ref as R


def test_identity_map_keeps_the_tokens():
    x = np.random.default_rng(0).standard_normal((6, 16))
    assert np.array_equal(R.compress_rows(x, 1, np.eye(16)), x)


def test_pair_sum_map():
    """m = 2 and w_t = [I | I]: each entry is the sum of its two tokens."""
    x = np.random.default_rng(1).integers(-8, 9, size=(10, 8)).astype(np.float64)
    w_t = np.concatenate([np.eye(8), np.eye(8)], axis=1)
    assert np.array_equal(R.compress_rows(x, 2, w_t), x[0::2] + x[1::2])


def test_brute_force_triple_loop():
    rng = np.random.default_rng(2)
    m, D_in, D, n = 3, 5, 4, 4
    x = rng.integers(-8, 9, size=(n * m, D_in)).astype(np.float64)
    w_t = rng.integers(-4, 5, size=(D, m * D_in)).astype(np.float64) / 64
    want = np.zeros((n, D))
    for j in range(n):
        for c in range(D):
            for i in range(m):
                for d in range(D_in):
                    want[j, c] += x[j * m + i, d] * w_t[c, i * D_in + d]
    assert np.array_equal(R.compress_rows(x, m, w_t), want)


def test_synthetic_entries_are_exact_in_fp32():
    """Integer tokens in [-8, 8] and a map of integers in [-4, 4] / 64: every entry is a
    multiple of 1/64 below 2^10 in magnitude, so fp32 holds it exactly and the GPU's fp32
    accumulation meets the oracle's fp64 sum bit for bit."""
    m, D_in, D = 2, 512, 512
    x = synth.bf16_bits_to_f32(synth.compressor_tokens(5, 64 * m, D_in))
    w_t = synth.bf16_bits_to_f32(synth.compressor_map(5, D, m * D_in))
    e = R.compress_rows(x, m, w_t)
    assert np.array_equal(e.astype(np.float32).astype(np.float64), e)
    assert np.all(np.abs(e) < 2 ** 10) and np.array_equal(e * 64, np.round(e * 64))
    codes, scales = R.compress_quantize(x, m, w_t)
    assert codes.shape == (64, D // 2) and scales.shape == (64, D // 16)
