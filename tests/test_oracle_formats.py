"""Pins of the oracle's FP4 / FP8 formats and of quantise+append (CPU only).

Independent sources: the OCP tables (golden files), ml_dtypes and torch casts
(library routines), closed-form round trips and error bounds.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import csa2_ref as R


def _f(v):
    return float("nan") if v == "nan" else float(v)


def test_e2m1_table_matches_ocp(golden):
    t = R.e2m1_decode_table()
    for code, val in golden("e2m1_ocp_mx_v1.txt"):
        c = int(code)
        assert t[c] == _f(val) and math.copysign(1, t[c]) == math.copysign(1, _f(val))


def test_e2m1_table_matches_ml_dtypes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(R.e2m1_decode_table(), lib)
    assert np.array_equal(np.signbit(R.e2m1_decode_table()), np.signbit(lib))


def test_e4m3_table_matches_ocp_landmarks(golden):
    t = R.e4m3_decode_table()
    for code, val in golden("e4m3_ocp_mx_v1.txt"):
        c, v = int(code, 16), _f(val)
        if math.isnan(v):
            assert math.isnan(t[c])
        else:
            assert t[c] == v and math.copysign(1, t[c]) == math.copysign(1, v)


def test_e4m3_table_matches_torch_all_codes():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = R.e4m3_decode_table()
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2
    np.testing.assert_array_equal(ours[~nan], lib[~nan])


def _dense_e4m3_probe():
    """Every finite E4M3 magnitude, every midpoint, and one fp32 ulp either side."""
    g = R.e4m3_decode_table()[:127].astype(np.float32)
    mids = ((g[:-1].astype(np.float64) + g[1:]) / 2).astype(np.float32)
    pts = np.concatenate([g, mids])
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(0)), np.nextafter(pts, np.float32(1e9))])
    rng = np.random.default_rng(7)
    rand = np.exp(rng.uniform(np.log(1e-5), np.log(448.0), 20000)).astype(np.float32)
    return np.concatenate([pts, rand, [0.0, 2.0**-11, 2.0**-10, 3 * 2.0**-11]]).astype(np.float32)


def test_e4m3_encode_matches_torch_cast_in_range():
    v = _dense_e4m3_probe()
    v = v[v <= 448.0]
    ours = R.e4m3_encode(v)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, lib)
    neg = R.e4m3_encode(-v[v > 0])
    np.testing.assert_array_equal(neg, lib[v > 0] | 0x80)


def test_e4m3_encode_matches_ml_dtypes_in_range():
    v = _dense_e4m3_probe()
    v = v[v <= 448.0]
    lib = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(R.e4m3_encode(v), lib)


def test_e4m3_encode_saturates():
    v = np.array([448.0, 460.0, 464.0, 1000.0, 3.0e38], dtype=np.float32)
    assert list(R.e4m3_encode(v)) == [0x7E] * 5
    assert list(R.e4m3_encode(-v)) == [0xFE] * 5


def test_e2m1_encode_hand_cases(golden):
    for x, val, code in golden("e2m1_rne_cases.txt"):
        c = int(R.e2m1_encode(np.float32(float(x))))
        assert c == int(code), (x, c, code)
        assert R.e2m1_decode_table()[c] == float(val)


def test_e2m1_encode_matches_ml_dtypes():
    g = R.e2m1_decode_table()[:8].astype(np.float32)
    mids = ((g[:-1].astype(np.float64) + g[1:]) / 2).astype(np.float32)
    pts = np.concatenate([g, mids])
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(0)), np.nextafter(pts, np.float32(99))])
    rng = np.random.default_rng(3)
    pts = np.concatenate([pts, rng.uniform(0, 9, 20000).astype(np.float32), [7.0, 50.0, 1e20]])
    pts = np.concatenate([pts, -pts]).astype(np.float32)
    lib = pts.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    np.testing.assert_array_equal(R.e2m1_encode(pts), lib)


def test_quantize_round_trip_exact_on_grid():
    """x = v * s with v on the E2M1 grid and some |v| = 6: amax/6 = s exactly, so the
    stored scale is s and every code is exact."""
    rng = np.random.default_rng(11)
    grid = R.e2m1_decode_table()
    e4 = R.e4m3_decode_table()
    B, D = 64, 512
    x = np.empty((B, D), dtype=np.float32)
    s_used = np.empty((B, D // 16))
    for b in range(B):
        for g in range(D // 16):
            s = e4[rng.integers(1, 127)]                    # a positive finite E4M3 value
            v = grid[rng.integers(0, 16, 16)]
            v[rng.integers(0, 16)] = 6.0 * rng.choice([-1, 1])
            x[b, g * 16:(g + 1) * 16] = (v * s).astype(np.float32)
            s_used[b, g] = s
    codes, scales = R.quantize_rows(x)
    np.testing.assert_array_equal(R.e4m3_decode_table()[scales], s_used)
    np.testing.assert_array_equal(R.dequantize_rows(codes, scales), x.astype(np.float64))


def test_quantize_error_bounds_random():
    """Scale within E4M3 rounding of amax/6; each value within half a grid step
    (times the scale) of x, except where the scale rounded down and x/s passed 6."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((256, 128)).astype(np.float32) * np.float32(3.0)
    codes, scales = R.quantize_rows(x)
    deq = R.dequantize_rows(codes, scales)
    s = R.e4m3_decode_table()[scales]                       # [B, D/16]
    amax = np.abs(x.reshape(256, 8, 16)).max(axis=2)
    assert np.all(np.abs(s - amax / 6.0) <= (amax / 6.0) / 16.0 + 2.0 ** -10)
    err = np.abs(deq - x).reshape(256, 8, 16)
    q = np.abs(x.reshape(256, 8, 16)) / s[:, :, None]
    half_step = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) * s[:, :, None]
    over = np.maximum(q - 6.0, 0.0) * s[:, :, None]          # saturation excess
    assert np.all(err <= half_step + over + 1e-12)


def test_quantize_zero_group_and_signed_zero():
    x = np.zeros((2, 32), dtype=np.float32)
    x[1, :16] = -0.0
    x[1, 16:] = np.linspace(-1, 1, 16, dtype=np.float32)
    codes, scales = R.quantize_rows(x)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert np.all(codes[0] == 0)
    assert np.all(codes[1, :8] == 0x88)                     # -0.0 keeps its sign bit
    assert scales[1, 1] != 0


def test_tiny_group_scale_underflows_to_zero():
    """amax/6 below half the smallest E4M3 subnormal rounds to scale 0: codes are signed zeros."""
    x = np.full((1, 16), 2.0 ** -13, dtype=np.float32)
    x[0, 3] = -(2.0 ** -13)
    codes, scales = R.quantize_rows(x)
    assert scales[0, 0] == 0
    nib = np.stack([codes[0] & 0xF, codes[0] >> 4], 1).reshape(-1)
    assert nib[3] == 0x8 and np.all(np.delete(nib, 3) == 0)


def test_nibble_order_low_is_even_channel():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0], x[0, 1] = 6.0, -3.0                            # scale 1.0
    codes, scales = R.quantize_rows(x)
    assert R.e4m3_decode_table()[scales[0, 0]] == 1.0
    assert codes[0, 0] == (0x7 | (0xD << 4))


def test_bytes_per_entry_from_arrays():
    """Arrays the oracle stores per entry: 4 bits per value plus one byte per 16 values."""
    for D, expect in ((512, 288), (128, 72)):
        codes, scales = R.quantize_rows(np.ones((3, D), dtype=np.float32))
        assert codes.shape[1] + scales.shape[1] == expect == R.bytes_per_entry(D)
        assert expect * 8 == D * 4 + (D // 16) * 8


def test_page_figures_consistent(golden):
    f = {r[0]: int(r[1]) for r in golden("page_figures.txt")}
    assert f["kv_bytes_per_token_v4flash"] == f["kv_bytes_per_token_v41"] * f["ratio_vs_v4flash"]
    assert abs(f["kv_bytes_per_token_v41"] * f["ratio_vs_v1"] - f["kv_bytes_per_token_v1"]) \
        < 0.001 * f["kv_bytes_per_token_v1"]
    assert f["pool_blocks"] * f["pool_block_size"] == f["pool_positions"]


# ---------------------------------------------------------------------------------------
# the compact (E4M3) indexer
# ---------------------------------------------------------------------------------------
def test_small_integers_round_trip_through_e4m3():
    """Integers in [-16, 16] need at most 4 significant bits and lie far inside E4M3's
    normal range, so an E4M3 indexer key holds them exactly."""
    from oracle import csa2_ref as R
    v = np.arange(-16, 17, dtype=np.float32)
    assert np.array_equal(R.e4m3_decode_table()[R.e4m3_encode(v)], v.astype(np.float64))
    # 17 has 5 significant bits: the nearest E4M3 values are 16 and 18, a tie -> even code 16
    assert R.e4m3_decode_table()[R.e4m3_encode(np.float32(17.0))] == 16.0


def test_e4m3_scores_equal_bf16_scores_on_integer_inputs():
    from oracle import csa2_ref as R
    rng = np.random.default_rng(5)
    qI = rng.integers(-8, 9, size=(16, 128)).astype(np.float64)
    kI = rng.integers(-8, 9, size=(500, 128)).astype(np.float64)
    w = rng.integers(1, 5, size=16).astype(np.float64)
    assert np.array_equal(R.index_scores_e4m3(qI, w, kI), R.index_scores(qI, w, kI))


def test_e4m3_scores_round_inputs_first():
    """Closed forms: 1.1 rounds to 1.125 (the E4M3 grid near 1 steps by 1/8), 500 saturates to
    448, and a negative dot product is cut by the ReLU."""
    from oracle import csa2_ref as R
    qI = np.array([[1.1], [500.0], [-1.0]])
    w = np.array([1.0, 0.5, 2.0])
    kI = np.array([[3.0], [1.0]])
    got = R.index_scores_e4m3(qI, w, kI)
    assert np.array_equal(got, np.array([1.125 * 3 + 0.5 * 448 * 3, 1.125 + 0.5 * 448]))
