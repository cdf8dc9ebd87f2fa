"""The paged global cache and the window ring on the GPU.

Paged: the same logical cache stored as 128-row pages in a shuffled pool (with unused pages)
and a block table must give bit-identical indices, pools and attention to the linear layout,
through a Full + Reuse + Reindex + Reuse schedule.  Moving a sequence's entries out
(export: csa2_cache_rows + csa2_gather_rows) and back into a fresh pool (import:
csa2_scatter_rows) must round-trip byte for byte.  Ring: window rows stored in a per-sequence
ring of 128 rows (the latest 128 tokens, slot = position mod 128) give the attention of the
linear window within the oracle tolerance, including a ring not yet full.
"""
import math

import numpy as np
import pytest
import torch

from tests import oracle_harness as OH
from tests.gpu_common import small_workload

pytestmark = pytest.mark.gpu


def _paged_copy(dw, extra_pages=13, seed=0):
    """Pages of dw's linear cache scattered over a shuffled pool; returns (seqs, tables)."""
    from fp4_kv_cache_03_b200 import csa2
    W = dw.W
    lens = [int(v) for v in W.lengths]
    n_pages = [-(-n // 128) for n in lens]
    total = sum(n_pages) + extra_pages
    perm = np.random.default_rng(seed).permutation(total)
    bt = np.full((W.num_seqs, max(n_pages) + 2), -1, dtype=np.int32)
    k = 0
    for s, npg in enumerate(n_pages):
        bt[s, :npg] = perm[k:k + npg]
        k += npg
    block_table = torch.from_numpy(bt).cuda()
    seqs_p = csa2.make_seqs(None, dw.seq_len, W.q_per_seq, block_table=block_table)
    seq = torch.from_numpy(np.repeat(np.arange(W.num_seqs), lens).astype(np.int32)).cuda()
    pos = torch.from_numpy(np.concatenate([np.arange(n) for n in lens]).astype(np.int32)).cuda()
    rows_p = csa2.cache_rows(seqs_p, seq, pos)
    rows_l = csa2.cache_rows(dw.seqs, seq, pos)
    tables = {}
    for name in ("kv_codes", "kv_scales", "idx_k"):
        lin = getattr(dw, name)
        paged = torch.zeros((total * 128,) + tuple(lin.shape[1:]), dtype=lin.dtype, device="cuda")
        csa2.scatter_rows(csa2.gather_rows(lin, rows_l), rows_p, paged)
        tables[name] = paged
    torch.cuda.synchronize()
    return seqs_p, tables, rows_p, rows_l


def test_paged_equals_linear_and_export_import_round_trip():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(3000, 700, 9000), D=256, H=32, H_I=16, d_I=128, topk=256,
                       pool_blocks=64, modes=("full", "reuse", "reindex", "reuse"), seed=51)
    lin = DeviceWorkload(W)
    used_l = [u.clone() for u in lin.run_step()]
    out_l = [o.clone() for o in lin.out]
    pool_l = lin.pool.clone()
    torch.cuda.synchronize()
    assert lin.status() == csa2.OK

    pg = DeviceWorkload(W)
    seqs_p, tables, rows_p, rows_l = _paged_copy(pg)
    pg.seqs, pg.kv_codes, pg.kv_scales, pg.idx_k = seqs_p, tables["kv_codes"], tables["kv_scales"], tables["idx_k"]
    used_p = pg.run_step()
    torch.cuda.synchronize()
    assert pg.status() == csa2.OK
    for li in range(len(W.modes)):
        assert torch.equal(used_p[li], used_l[li]), li
        assert torch.equal(pg.out[li], out_l[li]), li
    assert torch.equal(pg.pool, pool_l)
    ref = OH.query_layers(W, 2, with_attention=False)
    for li, r in enumerate(ref):
        np.testing.assert_array_equal(used_p[li][2].cpu().numpy(), r["indices"])

    # export the longest sequence from the pages, compare with the linear rows, import it
    # into a fresh pool and compare the pages
    s, n = 2, W.lengths[2]
    sel = slice(int(sum(W.lengths[:s])), int(sum(W.lengths[:s + 1])))
    for name in ("kv_codes", "kv_scales", "idx_k"):
        exported = csa2.gather_rows(tables[name], rows_p[sel])
        assert torch.equal(exported, getattr(lin, name)[rows_l[sel]])
        fresh = torch.zeros_like(tables[name])
        csa2.scatter_rows(exported, rows_p[sel], fresh)
        assert torch.equal(fresh[rows_p[sel]], tables[name][rows_p[sel]])
        assert not fresh[rows_p[:sel.start]].any()


def test_missing_page_is_skipped_and_reported():
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=(1000,), topk=64, modes=("full",), seed=52)
    dw = DeviceWorkload(W)
    seqs_p, tables, _, _ = _paged_copy(dw)
    bt = seqs_p._keep[3]
    bt[0, 3] = -1                                        # positions 384 .. 511 have no page
    L = dw.layers[0]
    idx = torch.zeros(1, W.topk, dtype=torch.int32, device="cuda")
    ws = csa2.workspace(csa2.index_full_workspace(1, dw.max_visible, W.topk))
    csa2.index_full(L.qI, L.w, tables["idx_k"], seqs_p, W.topk, idx, ws, dw.max_visible)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws) == csa2.ERR_CAPACITY
    got = idx[0].cpu().numpy()
    assert not np.any((got >= 384) & (got < 512))
    # the others are the Top-K of the remaining positions
    from oracle import csa2_ref as R
    kI = OH._kI_seq(W, 0)[:1000]
    qI, w = OH._iq(W, 0)
    sc = R.index_scores(qI[0], w[0], kI)
    keep = np.r_[0:384, 512:1000]
    np.testing.assert_array_equal(got, R.topk_ascending(sc[keep], W.topk, ids=keep))


@pytest.mark.parametrize("lengths", [(5000,), (40, 3000)])
def test_window_ring_matches_the_linear_window(lengths):
    """A 128-row ring per sequence; with lengths 40 the ring is not full yet (t = 39)."""
    from fp4_kv_cache_03_b200 import csa2
    from fp4_kv_cache_03_b200.workload import DeviceWorkload
    W = small_workload(lengths=lengths, D=256, H=32, H_I=16, d_I=128, topk=128, modes=("full",),
                       seed=53)
    dw = DeviceWorkload(W)
    dw.run_step()
    torch.cuda.synchronize()
    L = dw.layers[0]
    ring_rows = torch.zeros(W.num_seqs * 128, W.D, dtype=torch.bfloat16, device="cuda")
    t = W.q_pos()
    for s in range(W.num_seqs):
        lo = max(0, int(t[s]) - W.window + 1)
        for u in range(lo, int(t[s]) + 1):
            ring_rows[s * 128 + u % 128] = L.swa[int(L.swa_start[s]) + u]
    ring_start = torch.arange(W.num_seqs, dtype=torch.int64, device="cuda") * 128
    out = torch.zeros_like(dw.out[0])
    ws = csa2.workspace(csa2.sparse_attn_workspace(W.num_q, W.H, W.D, W.topk, W.window))
    csa2.sparse_attn(L.q, dw.kv_codes, dw.kv_scales, dw.seqs, dw.indices[0], ring_rows, ring_start,
                     dw.q_pos, W.window, 1.0 / math.sqrt(W.D), out, ws, swa_ring=128)
    torch.cuda.synchronize()
    assert csa2.status_fetch(ws) == csa2.OK
    # same keys, but small batches use 64-key tiles, and the two layouts split the window
    # into different tiles (by age / by ring slot): the key splits then sum in another order
    assert torch.allclose(out, dw.out[0], atol=1e-3, rtol=1e-3)
    for q in range(W.num_q):
        ref = OH.query_layers(W, q, with_attention=True)[0]
        ok, mx, rl2 = OH.attn_close(out[q].cpu().numpy(), ref["out"])
        assert ok, (q, mx, rl2)
