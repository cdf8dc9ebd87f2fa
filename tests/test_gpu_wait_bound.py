"""The bounded-wait failure path on the GPU, made to run out on purpose and safely.

Every wait inside the library's kernels gives up after a bound (2 s by default).  Here the
bound is set to 1 ns for two small calls, so the first wait that is not satisfied at once
runs out while the kernel's own TMA loads and MMAs are still in flight: the kernel must stop
every role, wait for those copies and MMAs, free its tensor memory, return, and report
CSA2_ERR_TIMEOUT in the call's status word.  Afterwards, with the default bound back, the
same GPU context must still produce bit-exact indices and in-tolerance attention.
No memory fault, trap or unbounded wait is involved: the waits that run out are on work
that completes by itself a few microseconds later.
"""
import math

import numpy as np
import pytest
import torch

from tests import oracle_harness as OH
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def test_wait_bound_runs_out_then_the_context_still_works():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(20000,), D=512, H=64, H_I=16, d_I=128, topk=256,
                       modes=("full",), pool_blocks=64, seed=31)
    dw = DeviceWorkload(W)
    L = dw.layers[0]
    # indices from a normal call, for the attention call below
    idx = torch.full((W.num_q, W.topk), -1, dtype=torch.int32, device="cuda")
    csa2.index_full(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, idx, dw.ws_full, dw.max_visible)
    torch.cuda.synchronize()
    assert csa2.status_fetch(dw.ws_full) == csa2.OK

    ws_i = csa2.workspace(csa2.index_full_workspace(W.num_q, dw.max_visible, W.topk, 64, 8))
    ws_a = csa2.workspace(csa2.sparse_attn_workspace(W.num_q, W.H, W.D, W.topk, W.window))
    got_idx = torch.full_like(idx, -1)
    pool = torch.full((W.num_q, 64), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros(W.num_q, W.H, W.D, device="cuda")
    prev = csa2.set_wait_limit_ns(1)
    try:
        csa2.index_full(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, got_idx, ws_i, dw.max_visible,
                        pool_blocks=64, block=8, pool=pool)
        csa2.sparse_attn(L.q, dw.kv_codes, dw.kv_scales, dw.seqs, idx, L.swa, L.swa_start,
                         dw.q_pos, W.window, 1.0 / math.sqrt(W.D), out, ws_a)
        torch.cuda.synchronize()
    finally:
        assert csa2.set_wait_limit_ns(prev) == 1
    assert csa2.status_fetch(ws_i) == csa2.ERR_TIMEOUT
    assert csa2.status_fetch(ws_a) == csa2.ERR_TIMEOUT

    # the same context, default bound: a whole step is exact again
    used = dw.run_step(attention=True)
    torch.cuda.synchronize()
    assert dw.status() == csa2.OK
    ref = OH.query_layers(W, 0, with_attention=True)
    np.testing.assert_array_equal(used[0][0].cpu().numpy(), ref[0]["indices"])
    np.testing.assert_array_equal(idx[0].cpu().numpy(), ref[0]["indices"])
    ok, mx, rl2 = OH.attn_close(dw.out[0][0].cpu().numpy(), ref[0]["out"])
    assert ok, (mx, rl2)
