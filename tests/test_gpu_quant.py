"""a1 quantise + append on the GPU vs the oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

from oracle import csa2_ref as R

pytestmark = pytest.mark.gpu


def gpu_quant(x: np.ndarray, offset=3, d_I=0, kin=None):
    from fp4_kv_cache_03_b200 import csa2
    rows, D = x.shape
    cap = rows + offset + 2
    codes = torch.zeros(cap, D // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(cap, D // 16, dtype=torch.uint8, device="cuda")
    dst = torch.arange(offset, offset + rows, dtype=torch.int64, device="cuda")
    ws = csa2.workspace(csa2.quant_append_workspace())
    idx_k = torch.zeros(cap, d_I, dtype=torch.bfloat16, device="cuda") if kin is not None else None
    kin_t = (torch.from_numpy(kin.view(np.int16)).cuda().view(torch.bfloat16)
             if kin is not None else None)
    csa2.quant_append(torch.from_numpy(x).cuda(), dst, codes, scales, ws, idx_k_in=kin_t,
                      idx_k=idx_k)
    assert csa2.status_fetch(ws) == csa2.OK
    out = (codes[offset:offset + rows].cpu().numpy(), scales[offset:offset + rows].cpu().numpy())
    if kin is not None:
        out = out + (idx_k[offset:offset + rows].view(torch.int16).cpu().numpy().view(np.uint16),)
    assert not codes[:offset].any() and not codes[offset + rows:].any()
    return out


@pytest.mark.parametrize("D", [128, 512])
def test_random_rows_bit_exact(D):
    rng = np.random.default_rng(D)
    x = (rng.standard_normal((2048, D)) * rng.choice([0.01, 1.0, 4.0, 300.0], (2048, 1)))
    x = x.astype(np.float32)
    c, s = gpu_quant(x)
    rc, rs = R.quantize_rows(x)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(c, rc)


def _edge_rows():
    e4 = R.e4m3_decode_table()
    rows = []
    g = lambda vals: np.asarray(vals, dtype=np.float32)
    rows.append(np.zeros(16))
    rows.append(-np.zeros(16))
    rows.append(np.full(16, 2.0 ** -13) * np.tile([1, -1], 8))        # scale underflows to 0
    rows.append(np.full(16, 1e-40))                                    # fp32 subnormals
    rows.append(np.full(16, 3.0e38) * np.tile([1, -1], 8))            # scale saturates at 448
    rows.append(np.linspace(-7000, 7000, 16))
    for s in (e4[1], e4[7], e4[8], 1.0, 1.125, 448.0):                 # grid values x scale
        rows.append(np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6]) * s)
    for s in (1.0, 0.0625, e4[3]):                                     # exact E2M1 midpoints
        rows.append(np.array([6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, -.25, -.75, -1.25, -1.75,
                              -2.5, -3.5, -5, .1]) * s)
    for m in (1.0625, 1.1875, 2.0 ** -10 * 0.5, 3 * 2.0 ** -11):       # amax/6 on E4M3 midpoints
        rows.append(np.concatenate([[6 * m], np.linspace(-m, m, 15)]))
    rng = np.random.default_rng(0)
    for _ in range(16):
        rows.append(rng.standard_normal(16) * np.exp(rng.uniform(-20, 20)))
    x = np.concatenate([g(r) for r in rows]).astype(np.float32)
    pad = (-x.shape[0]) % 128
    x = np.concatenate([x, np.zeros(pad, np.float32)])
    return x.reshape(-1, 128)


def test_edge_values_bit_exact():
    x = _edge_rows()
    c, s = gpu_quant(x)
    rc, rs = R.quantize_rows(x)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(c, rc)


def test_indexer_row_copy():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    kin = rng.integers(0, 1 << 16, (64, 128)).astype(np.uint16)
    c, s, k = gpu_quant(x, d_I=128, kin=kin)
    np.testing.assert_array_equal(k, kin)


def test_row_outside_cache_is_skipped_and_reported():
    from fp4_kv_cache_03_b200 import csa2
    x = torch.ones(4, 64, device="cuda")
    codes = torch.zeros(8, 32, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(8, 4, dtype=torch.uint8, device="cuda")
    dst = torch.tensor([0, 8, -1, 7], dtype=torch.int64, device="cuda")
    ws = csa2.workspace(256)
    csa2.quant_append(x, dst, codes, scales, ws)
    assert csa2.status_fetch(ws) == csa2.ERR_CAPACITY
    rc, rs = R.quantize_rows(np.ones((1, 64), np.float32))
    assert np.array_equal(codes[0].cpu().numpy(), rc[0]) and np.array_equal(codes[7].cpu().numpy(), rc[0])
    assert not codes[1:7].any()
