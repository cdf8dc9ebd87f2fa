"""a7 sparse attention on the GPU vs the fp64 oracle (max-abs 2e-2, rel-L2 1e-2)."""
import math

import numpy as np
import pytest
import torch

from fp4_kv_cache_03_b200 import synth
from tests import oracle_harness as OH
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def run_attn(W, queries=None):
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    dw = DeviceWorkload(W)
    dw.run_step(attention=True)
    torch.cuda.synchronize()
    assert dw.status() == csa2.OK
    qs = range(W.num_q) if queries is None else queries
    worst = 0.0
    for q in qs:
        ref = OH.query_layers(W, q, with_attention=True)
        for li, r in enumerate(ref):
            got = dw.out[li][q].cpu().numpy()
            ok, mx, rl2 = OH.attn_close(got, r["out"])
            assert ok, f"q={q} layer={li} max-abs={mx:.3e} rel-L2={rl2:.3e}"
            lse = dw.lse[li][q].cpu().numpy()
            np.testing.assert_allclose(lse, r["lse"], atol=2e-3, rtol=1e-4)
            worst = max(worst, mx)
    return dw, worst


def test_tiny_config_attention():
    run_attn(synth.workload("tiny"))


def test_short_context_window_and_padding():
    """t < 127: the window holds only t+1 rows; fewer than topk entries: -1 slots skipped."""
    W = small_workload(lengths=(1, 50, 200), topk=64, window=128, modes=("full", "reuse"))
    run_attn(W)


@pytest.mark.parametrize("D,H", [(256, 40), (512, 12), (128, 64), (256, 1)])
def test_head_groups_and_dims(D, H):
    """Every supported D, and head counts that leave a partial 16-head group (the heads past
    H read as zero); Full then Reuse with the stash, 2 queries of a ragged batch."""
    W = small_workload(lengths=(700, 3000), D=D, H=H, topk=256, window=128,
                       modes=("full", "reuse"), outlier_frac=0.01)
    run_attn(W)


def test_many_tiles_per_cta():
    """More tiles than splits: a CTA loops over several tiles (rescaled running max, the
    stash stored and loaded per tile) -- 128 queries of one sequence at topk 512."""
    W = small_workload(lengths=(8192,), q_per_seq=128, D=128, H=16, topk=512, window=128,
                       modes=("full", "reuse"), q_token0=(8192 - 128,))
    run_attn(W, queries=[0, 63, 127])


def test_window_only_and_empty():
    from fp4_kv_cache_03_b200 import csa2
    dev = "cuda"
    H, D = 16, 128
    q = torch.randn(2, H, D, device=dev).to(torch.bfloat16)
    codes = torch.zeros(4, D // 2, dtype=torch.uint8, device=dev)
    scales = torch.zeros(4, D // 16, dtype=torch.uint8, device=dev)
    seq_start = torch.zeros(2, dtype=torch.int64, device=dev)
    seq_len = torch.tensor([2, 2], dtype=torch.int32, device=dev)
    seqs = csa2.make_seqs(seq_start, seq_len)
    idx = torch.full((2, 16), -1, dtype=torch.int32, device=dev)
    swa = torch.randn(8, D, device=dev).to(torch.bfloat16)
    swa_start = torch.tensor([0, 4], dtype=torch.int64, device=dev)
    q_pos = torch.tensor([3, 0], dtype=torch.int64, device=dev)
    out = torch.full((2, H, D), 7.0, device=dev)
    lse = torch.zeros(2, H, device=dev)
    ws = csa2.workspace(csa2.sparse_attn_workspace(2, H, D, 16, 4))
    csa2.sparse_attn(q, codes, scales, seqs, idx, swa, swa_start, q_pos, 4, 1 / math.sqrt(D), out,
                     ws, lse=lse)
    assert csa2.status_fetch(ws) == csa2.OK
    from oracle import csa2_ref as R
    qf = q.float().cpu().numpy()
    sf = swa.float().cpu().numpy()
    o0, l0 = R.sparse_attention(qf[0], np.zeros((0, D)), sf[0:4], 1 / math.sqrt(D))
    o1, l1 = R.sparse_attention(qf[1], np.zeros((0, D)), sf[4:5], 1 / math.sqrt(D))
    assert OH.attn_close(out[0].cpu().numpy(), o0)[0] and OH.attn_close(out[1].cpu().numpy(), o1)[0]
    # no rows at all: window 0 and every index -1
    ws2 = csa2.workspace(csa2.sparse_attn_workspace(2, H, D, 16, 0))
    csa2.sparse_attn(q, codes, scales, seqs, idx, swa, swa_start, q_pos, 0, 0.1, out, ws2, lse=lse)
    assert csa2.status_fetch(ws2) == csa2.OK
    assert not out.any() and torch.all(lse == -math.inf)


def test_bad_index_is_skipped_and_reported():
    from fp4_kv_cache_03_b200 import csa2
    dev = "cuda"
    H, D = 16, 128
    q = torch.randn(1, H, D, device=dev).to(torch.bfloat16)
    codes = torch.zeros(8, D // 2, dtype=torch.uint8, device=dev)
    scales = torch.zeros(8, D // 16, dtype=torch.uint8, device=dev)
    seqs = csa2.make_seqs(torch.zeros(1, dtype=torch.int64, device=dev),
                          torch.tensor([4], dtype=torch.int32, device=dev))
    idx = torch.tensor([[0, 9, -5, 3]], dtype=torch.int32, device=dev)
    swa = torch.zeros(1, D, device=dev).to(torch.bfloat16)
    out = torch.zeros(1, H, D, device=dev)
    ws = csa2.workspace(csa2.sparse_attn_workspace(1, H, D, 4, 0))
    csa2.sparse_attn(q, codes, scales, seqs, idx, swa, torch.zeros(1, dtype=torch.int64, device=dev),
                     torch.zeros(1, dtype=torch.int64, device=dev), 0, 0.1, out, ws)
    assert csa2.status_fetch(ws) == csa2.ERR_INVALID_ARG


def test_decoder_group_128k_attention():
    run_attn(synth.workload("decoder_group_128k"))


def test_reuse_stash_equals_stateless():
    """Reuse layers reading the stashed FP4 rows give bit-identical results to Reuse
    layers that gather and dequantise the FP4 rows again; Reindex layers refresh it."""
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(3000, 9000), D=512, H=64, H_I=16, d_I=128, topk=256,
                       pool_blocks=64, modes=("full", "reuse", "reuse", "reindex", "reuse"))
    a = DeviceWorkload(W, use_stash=True)
    b = DeviceWorkload(W, use_stash=False)
    assert a.stash is not None and b.stash is None
    a.run_step()
    b.run_step()
    torch.cuda.synchronize()
    for li in range(len(W.modes)):
        assert torch.equal(a.out[li], b.out[li]), li
        assert torch.equal(a.lse[li], b.lse[li]), li


def test_all_heads_in_one_cta():
    """A batch large enough that one CTA takes all 64 heads of a query (N = 64 in the MMAs),
    with the stash in the staging order of that path."""
    W = small_workload(lengths=(6000,), q_per_seq=80, D=512, H=64, H_I=16, d_I=128, topk=256,
                       window=128, modes=("full", "reuse"), q_token0=(6000 - 80,),
                       outlier_frac=0.01)
    run_attn(W, queries=[0, 41, 79])
