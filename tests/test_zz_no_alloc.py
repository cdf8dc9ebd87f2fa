"""csa2_index_full_noalloc: the Full-mode index computed in the library's own fixed device
array instead of a caller workspace.

It exists for callers that cannot call cudaMalloc -- code running inside a host framework
that owns the device allocator, real-time loops that must not allocate, or processes that
may not grow device memory after start-up.  Its results must equal csa2_index_full's, bit
for bit (indices and pool), call after call, since every call shares and reuses the same
array.  This file is collected last on purpose.
"""
import pytest
import torch

from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def _both(dw, L, W):
    from fp4_kv_cache_03_b200 import csa2
    ref_idx = torch.full((W.num_q, W.topk), -7, dtype=torch.int32, device="cuda")
    ref_pool = torch.full((W.num_q, W.pool_blocks), -7, dtype=torch.int32, device="cuda")
    csa2.index_full(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, ref_idx, dw.ws_full, dw.max_visible,
                    q_visible=dw.q_visible, pool_blocks=W.pool_blocks, block=W.block,
                    pool=ref_pool)
    got_idx = torch.full_like(ref_idx, -9)
    got_pool = torch.full_like(ref_pool, -9)
    csa2.index_full_noalloc(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, got_idx, dw.max_visible,
                            q_visible=dw.q_visible, pool_blocks=W.pool_blocks, block=W.block,
                            pool=got_pool)
    torch.cuda.synchronize()
    assert csa2.status_fetch(dw.ws_full) == csa2.OK
    assert csa2.index_full_noalloc_status() == csa2.OK     # the array's own status word
    return ref_idx, ref_pool, got_idx, got_pool


def test_noalloc_equals_workspace_entry_point_two_calls_in_a_row():
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(131072,), D=512, H=64, H_I=16, d_I=128, topk=512,
                       pool_blocks=2048, modes=("full", "reindex"), seed=21)
    dw = DeviceWorkload(W)
    results = []
    for li in (0, 1):              # two calls in a row, each with different indexer inputs
        ref_idx, ref_pool, got_idx, got_pool = _both(dw, dw.layers[li], W)
        assert torch.equal(got_idx, ref_idx), f"call {li}: indices differ"
        assert torch.equal(got_pool, ref_pool), f"call {li}: pools differ"
        results.append(got_idx.clone())
    assert not torch.equal(results[0], results[1])   # the second call did not reuse stale output


def test_noalloc_ragged_batch_matches():
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(5, 900, 4097, 20000), topk=64, pool_blocks=64,
                       modes=("full",), seed=22)
    dw = DeviceWorkload(W)
    for _ in range(2):
        ref_idx, ref_pool, got_idx, got_pool = _both(dw, dw.layers[0], W)
        assert torch.equal(got_idx, ref_idx) and torch.equal(got_pool, ref_pool)


def test_noalloc_rejects_sizes_beyond_its_array():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(4096,), modes=("full",), seed=23)
    dw = DeviceWorkload(W)
    L = dw.layers[0]
    idx = torch.zeros(1, W.topk, dtype=torch.int32, device="cuda")
    with pytest.raises(csa2.CSA2Error) as e:
        csa2.index_full_noalloc(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, idx, 4_000_000)
    assert e.value.status == csa2.ERR_CAPACITY
    assert csa2.index_full_workspace(1, 4_000_000, W.topk) > csa2.NOALLOC_SCRATCH_BYTES


def test_noalloc_argument_errors_match_the_workspace_entry_point():
    """Bad arguments give the same status as csa2_index_full, before the size check."""
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(4096,), modes=("full",), seed=24)
    dw = DeviceWorkload(W)
    L = dw.layers[0]
    idx = torch.zeros(1, 64, dtype=torch.int32, device="cuda")
    for topk, pool_blocks, block in ((0, 0, 8), (5000, 0, 8), (64, 16, 3), (64, 9000, 8)):
        codes = []
        for fn in (lambda: csa2.index_full(L.qI, L.w, dw.idx_k, dw.seqs, topk, idx, dw.ws_full,
                                           4_000_000, pool_blocks=pool_blocks, block=block,
                                           pool=idx if pool_blocks else None),
                   lambda: csa2.index_full_noalloc(L.qI, L.w, dw.idx_k, dw.seqs, topk, idx,
                                                   4_000_000, pool_blocks=pool_blocks,
                                                   block=block, pool=idx if pool_blocks else None)):
            with pytest.raises(csa2.CSA2Error) as e:
                fn()
            codes.append(e.value.status)
        assert codes[0] == codes[1] == csa2.ERR_UNSUPPORTED, (topk, pool_blocks, block, codes)
