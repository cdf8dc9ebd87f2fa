"""The compact indexer path (E4M3 indexer K and Q) on the GPU: with integer-valued indexer
inputs every index and pool must equal the oracle's (E4M3 scores are then exact) and the bf16
path's, bit for bit -- Full with the 2048 x 8 pool, Reindex over it, a ragged batch, and the
whole decoder schedule (append into the E4M3 cache included) through csa2_layer_step."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from tests import oracle_harness as OH
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def _both(W, queries, via_layer_step=False):
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    runs = []
    for e4m3 in (False, True):
        dw = DeviceWorkload(W, indexer_e4m3=e4m3)
        used = dw.run_step(attention=True, via_layer_step=via_layer_step)
        torch.cuda.synchronize()
        assert dw.status() == csa2.OK
        runs.append((dw, [u.cpu().numpy() for u in used], dw.pool.cpu().numpy()))
    (d16, i16, p16), (d8, i8, p8) = runs
    assert d8.idx_k.dtype == torch.uint8 and d8.idx_k.element_size() == 1
    for li in range(len(W.modes)):
        np.testing.assert_array_equal(i8[li], i16[li], err_msg=f"layer {li}")
        assert torch.equal(d8.out[li], d16.out[li])
    np.testing.assert_array_equal(p8, p16)
    for q in queries:
        ref = OH.query_layers(W, q, with_attention=False)
        for li, r in enumerate(ref):
            np.testing.assert_array_equal(i8[li][q], r["indices"], err_msg=f"q={q} layer={li}")
            if "pool" in r:
                np.testing.assert_array_equal(p8[q], r["pool"])


def test_e4m3_full_with_pool_and_reindex_131072():
    W = small_workload(lengths=(131072,), D=128, H=16, H_I=16, d_I=128, topk=512,
                       pool_blocks=2048, modes=("full", "reuse", "reindex", "reuse"), seed=41)
    _both(W, [0])


def test_e4m3_ragged_batch():
    W = small_workload(lengths=(3, 700, 4099, 9000, 20000), D=128, H=16, H_I=16, d_I=128,
                       topk=256, modes=("full",), seed=42)
    _both(W, range(W.num_q))


def test_e4m3_decoder_step_via_layer_step():
    """The 20-layer decoder schedule on the compact path, every layer one csa2_layer_step call;
    the step's append writes its indexer key into the E4M3 cache."""
    _both(synth.workload("decoder_step_128k"), [0], via_layer_step=True)
