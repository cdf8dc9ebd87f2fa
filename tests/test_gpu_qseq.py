"""A batch that mixes decode queries with chunks of several queries per sequence, described
by the per-query sequence map of csa2_seqs_t (q_seq): 1, 5 and 2 queries of three sequences.
Indices are compared bit for bit and attention within max-abs 2e-2 / rel-L2 1e-2 against the
oracle, query by query (each query is one of the equal-split workload's, picked out)."""
import math

import numpy as np
import pytest
import torch

from tests import oracle_harness as OH
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def test_unequal_queries_per_sequence():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(3000, 9000, 5000), q_per_seq=5, D=256, H=32, H_I=8, d_I=128,
                       topk=256, window=128, modes=("full",), ratio=2,
                       q_token0=(5990, 17990, 9990), seed=43)
    dw = DeviceWorkload(W)
    picked = [4, 5, 6, 7, 8, 9, 12, 13]               # seq 0: 1 query, seq 1: 5, seq 2: 2
    sel = torch.tensor(picked, device="cuda")
    q_seq = torch.tensor([p // W.q_per_seq for p in picked], dtype=torch.int32, device="cuda")
    seqs = csa2.make_seqs(dw.seq_start, dw.seq_len, q_per_seq=0, q_seq=q_seq)
    L = dw.layers[0]
    nq = len(picked)
    qI = L.qI[sel].contiguous()
    w = L.w[sel].contiguous()
    q = L.q[sel].contiguous()
    q_pos = dw.q_pos[sel].contiguous()
    q_vis = torch.from_numpy(W.q_visible()).cuda()[sel].contiguous()
    idx = torch.full((nq, W.topk), -7, dtype=torch.int32, device="cuda")
    ws_i = csa2.workspace(csa2.index_full_workspace(nq, dw.max_visible, W.topk))
    csa2.index_full(qI, w, dw.idx_k, seqs, W.topk, idx, ws_i, dw.max_visible, q_visible=q_vis)
    out = torch.zeros(nq, W.H, W.D, device="cuda")
    lse = torch.zeros(nq, W.H, device="cuda")
    ws_a = csa2.workspace(csa2.sparse_attn_workspace(nq, W.H, W.D, W.topk, W.window))
    csa2.sparse_attn(q, dw.kv_codes, dw.kv_scales, seqs, idx, L.swa, L.swa_start, q_pos, W.window,
                     1.0 / math.sqrt(W.D), out, ws_a, lse=lse)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws_i) == csa2.OK and csa2.status_fetch(ws_a) == csa2.OK
    for j, p in enumerate(picked):
        ref = OH.query_layers(W, p, with_attention=True)[0]
        np.testing.assert_array_equal(idx[j].cpu().numpy(), ref["indices"], err_msg=f"query {p}")
        ok, mx, rl2 = OH.attn_close(out[j].cpu().numpy(), ref["out"])
        assert ok, (p, mx, rl2)


def test_out_of_range_sequence_is_skipped_and_reported():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(2000, 2000), topk=64, modes=("full",), seed=44)
    dw = DeviceWorkload(W)
    L = dw.layers[0]
    q_seq = torch.tensor([1, 5], dtype=torch.int32, device="cuda")     # 5: no such sequence
    seqs = csa2.make_seqs(dw.seq_start, dw.seq_len, q_per_seq=0, q_seq=q_seq)
    idx = torch.zeros(2, W.topk, dtype=torch.int32, device="cuda")
    ws = csa2.workspace(csa2.index_full_workspace(2, dw.max_visible, W.topk))
    order = torch.tensor([1, 0], device="cuda")      # row 0 carries query 1's indexer Q
    csa2.index_full(L.qI[order].contiguous(), L.w[order].contiguous(), dw.idx_k, seqs, W.topk,
                    idx, ws, dw.max_visible)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws) == csa2.ERR_INVALID_ARG
    assert torch.all(idx[1] == -1)                    # the bad query sees nothing
    ref = OH.query_layers(W, 1, with_attention=False)[0]
    np.testing.assert_array_equal(idx[0].cpu().numpy(), ref["indices"])
