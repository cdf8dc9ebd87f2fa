"""The fused compressor + quantise + append on the GPU (csa2_compress_append) against the
oracle: codes and scales bit for bit, on a ragged number of entries scattered over the cache,
for every supported output width; rows outside the cache are skipped and reported."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from oracle import csa2_ref as R

pytestmark = pytest.mark.gpu


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("D,m,D_in,n", [(512, 2, 512, 300), (256, 2, 256, 129), (128, 4, 64, 7)])
def test_compress_append_matches_oracle(D, m, D_in, n):
    from fp4_kv_cache_03_b200 import csa2
    xb = synth.compressor_tokens(7, n * m, D_in)
    wb = synth.compressor_map(7, D, m * D_in)
    cap = n + 50
    perm = np.random.default_rng(3).permutation(cap)[:n].astype(np.int64)
    dst = torch.from_numpy(perm).cuda()
    codes = torch.zeros(cap, D // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(cap, D // 16, dtype=torch.uint8, device="cuda")
    ws = csa2.workspace(csa2.quant_append_workspace())
    csa2.compress_append(_bf16(xb), m, _bf16(wb), dst, codes, scales, ws)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws) == csa2.OK
    want_c, want_s = R.compress_quantize(synth.bf16_bits_to_f32(xb), m, synth.bf16_bits_to_f32(wb))
    got_c, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    np.testing.assert_array_equal(got_c[perm], want_c)
    np.testing.assert_array_equal(got_s[perm], want_s)
    untouched = np.setdiff1d(np.arange(cap), perm)
    assert not got_c[untouched].any() and not got_s[untouched].any()


def test_rows_outside_the_cache_are_skipped():
    from fp4_kv_cache_03_b200 import csa2
    n, m, D_in, D = 4, 2, 64, 128
    xb = synth.compressor_tokens(8, n * m, D_in)
    wb = synth.compressor_map(8, D, m * D_in)
    dst = torch.tensor([2, -1, 9, 0], dtype=torch.int64, device="cuda")     # cap = 3
    codes = torch.zeros(3, D // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(3, D // 16, dtype=torch.uint8, device="cuda")
    ws = csa2.workspace(csa2.quant_append_workspace())
    csa2.compress_append(_bf16(xb), m, _bf16(wb), dst, codes, scales, ws)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws) == csa2.ERR_CAPACITY
    want_c, want_s = R.compress_quantize(synth.bf16_bits_to_f32(xb), m, synth.bf16_bits_to_f32(wb))
    np.testing.assert_array_equal(codes.cpu().numpy()[[2, 0]], want_c[[0, 3]])
    assert not codes.cpu().numpy()[1].any()
