"""The five CSA2 workloads end to end through the C ABI (append, Full / Reindex / Reuse
schedule, attention) vs the oracle: indices and pools bit-exact, attention within
max-abs 2e-2 and rel-L2 1e-2.  The large workloads are compared on sampled queries,
including the first and last of each batch."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from tests import oracle_harness as OH

pytestmark = pytest.mark.gpu


def check(W, queries, via_layer_step=False):
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    dw = DeviceWorkload(W)
    used = dw.run_step(attention=True, via_layer_step=via_layer_step)
    torch.cuda.synchronize()
    assert dw.status() == csa2.OK
    idx = [u.cpu().numpy() for u in used]
    pool = dw.pool.cpu().numpy()
    for q in queries:
        ref = OH.query_layers(W, q, with_attention=True)
        for li, r in enumerate(ref):
            np.testing.assert_array_equal(idx[li][q], r["indices"], err_msg=f"q={q} layer={li}")
            if "pool" in r:
                np.testing.assert_array_equal(pool[q], r["pool"])
            ok, mx, rl2 = OH.attn_close(dw.out[li][q].cpu().numpy(), r["out"])
            assert ok, f"q={q} layer={li} max-abs={mx:.3e} rel-L2={rl2:.3e}"
    return dw


def test_tiny():
    check(synth.workload("tiny"), [0])


def test_decoder_group_128k():
    check(synth.workload("decoder_group_128k"), [0])


def test_hier_decoder_1m():
    check(synth.workload("hier_decoder_1m"), [0])


def test_encoder_chunk_sampled():
    W = synth.workload("encoder_chunk")
    check(W, [0, 1, 777, 2048, 4094, 4095])


def test_ragged_decode_sampled():
    W = synth.workload("ragged_decode")
    lens = np.asarray(W.lengths)
    qs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 31, 63})
    check(W, qs)


def test_decoder_step_128k_sampled():
    """The 20-layer decoder schedule (Full + pool, 3 Reuse, then 4 x (Reindex + 3 Reuse)),
    every layer one csa2_layer_step call."""
    check(synth.workload("decoder_step_128k"), [0], via_layer_step=True)


def test_encoder_stack_via_layer_step():
    """The 18-layer encoder stack: 3 groups (each its own 32,768-entry cache at ratio 2) of
    Full + 5 Reuse over a 4,096-query causal chunk, every layer one csa2_layer_step call;
    sampled queries of every layer of every group against the oracle."""
    for name in synth.ENCODER_STACK:
        check(synth.workload(name), [0, 2047, 4095], via_layer_step=True)
