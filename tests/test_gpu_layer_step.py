"""csa2_layer_step drives a layer by its mode: the Full (+pool) / Reuse / Reindex / Reuse
schedule through it gives the same bits as the separate index and attention calls."""
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def test_layer_step_equals_separate_calls():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(4096, 2000), D=128, H=16, topk=64, window=128,
                       modes=("full", "reuse", "reindex", "reuse"), pool_blocks=64)
    a = DeviceWorkload(W)
    used = a.run_step()
    b = DeviceWorkload(W)
    latest, n_idx = None, 0
    for li, L in enumerate(b.layers):
        attn = dict(q=L.q, swa_kv=L.swa, swa_start=L.swa_start, q_pos=b.q_pos, window=W.window,
                    softmax_scale=b.scale, out=b.out[li], lse=b.lse[li], ws=b.ws_attn,
                    stash=b.stash)
        if L.mode == synth.REUSE:
            csa2.layer_step(csa2.MODE_REUSE, b.kv_codes, b.kv_scales, b.seqs, W.topk, latest, attn)
            continue
        idx = b.indices[n_idx]
        n_idx += 1
        ix = dict(qI=L.qI, w=L.w, idx_k=b.idx_k, q_visible=b.q_visible, block=W.block,
                  pool_blocks=W.pool_blocks, pool=b.pool)
        if L.mode == synth.FULL:
            ix.update(ws=b.ws_full, max_visible=b.max_visible)
            csa2.layer_step(csa2.MODE_FULL, b.kv_codes, b.kv_scales, b.seqs, W.topk, idx, attn, ix)
        else:
            ix.update(ws=b.ws_pool)
            csa2.layer_step(csa2.MODE_REINDEX, b.kv_codes, b.kv_scales, b.seqs, W.topk, idx, attn, ix)
        latest = idx
    torch.cuda.synchronize()
    assert a.status() == csa2.OK and b.status() == csa2.OK
    assert torch.equal(a.pool, b.pool)
    for li in range(len(W.modes)):
        assert torch.equal(used[li], b.indices[min(li // 2, 1)]), li
        assert torch.equal(a.out[li], b.out[li]), li
        assert torch.equal(a.lse[li], b.lse[li]), li
