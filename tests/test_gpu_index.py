"""a2-a5 on the GPU vs the oracle: Top-K indices and pools bit-exact."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from oracle import csa2_ref as R
from tests import oracle_harness as OH
from tests.gpu_common import gpu_indices, small_workload

pytestmark = pytest.mark.gpu


def run(W, queries=None, attention=False):
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    dw = DeviceWorkload(W)
    used = dw.run_step(attention=attention)
    torch.cuda.synchronize()
    assert dw.status() == csa2.OK
    idx = gpu_indices(dw, used)
    pool = dw.pool.cpu().numpy().astype(np.int64)
    qs = range(W.num_q) if queries is None else queries
    for q in qs:
        ref = OH.query_layers(W, q, with_attention=False)
        for li, r in enumerate(ref):
            np.testing.assert_array_equal(idx[li][q], r["indices"], err_msg=f"q={q} layer={li}")
            if "pool" in r:
                np.testing.assert_array_equal(pool[q], r["pool"], err_msg=f"pool q={q}")
    return dw, idx, pool


def test_tiny_config():
    run(synth.workload("tiny"))


def test_ragged_lengths_and_pool():
    W = small_workload(lengths=(1, 7, 100, 129, 4095, 9001), topk=64, pool_blocks=16,
                       modes=("full", "reindex", "reuse"))
    run(W)


def test_fewer_visible_than_topk():
    W = small_workload(lengths=(37, 64, 65), topk=64, pool_blocks=8,
                       modes=("full", "reindex"))
    run(W)


def test_all_equal_scores_take_lowest_positions():
    """qI = 0 makes every score 0: ties everywhere, the lowest positions win."""
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(20000,), topk=512, pool_blocks=2048, modes=("full",),
                       H_I=16, d_I=128)
    dw = DeviceWorkload(W)
    dw.layers[0].qI.zero_()
    dw.run_step(attention=False)
    assert dw.status() == csa2.OK
    assert np.array_equal(dw.indices[0][0].cpu().numpy(), np.arange(512))
    assert np.array_equal(dw.pool[0].cpu().numpy(), np.arange(2048))


def test_causal_visibility_chunk():
    """Several queries of one sequence, each seeing floor((t+1)/2) entries."""
    W = small_workload(lengths=(3000,), q_per_seq=40, ratio=2, q_token0=(5900,), topk=64,
                       modes=("full", "reuse"), H_I=16, d_I=128)
    run(W)


def test_repeat_runs_identical():
    W = small_workload(lengths=(50000,), topk=512, pool_blocks=256, H_I=16, d_I=128,
                       modes=("full", "reindex"))
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    dw = DeviceWorkload(W)
    a = [t.clone() for t in dw.run_step(attention=False)] + [dw.pool.clone()]
    b = [t.clone() for t in dw.run_step(attention=False)] + [dw.pool.clone()]
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_decoder_group_128k_index():
    run(synth.workload("decoder_group_128k"))


def test_hier_decoder_1m_index_and_reindex():
    W = synth.workload("hier_decoder_1m")
    dw, idx, pool = run(W)
    assert (pool[0] >= 0).sum() == 2048


def test_reindex_with_full_query_reproduces_full_topk_1m():
    """Theorem (lowest-index tie-breaks): re-scoring the pool with the Full layer's own
    indexer Q returns exactly the Full Top-K.  Checked on the GPU at 1M entries."""
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = synth.workload("hier_decoder_1m")
    dw = DeviceWorkload(W)
    L0, L1 = dw.layers[0], dw.layers[1]
    L1.qI.copy_(L0.qI)
    L1.w.copy_(L0.w)
    used = dw.run_step(attention=False)
    assert dw.status() == csa2.OK
    assert torch.equal(used[0], used[1])
