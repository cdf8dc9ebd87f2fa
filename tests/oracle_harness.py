"""Oracle results for a synthetic workload, query by query (test infrastructure).

Uses only ``oracle`` and the seeded generators in ``synth``; nothing here reads
anything the CUDA path produced.
"""
from __future__ import annotations

import functools
import math

import numpy as np

from fp4_kv_cache_03_b200 import synth
from oracle import csa2_ref as R


def f32(bits):
    return synth.bf16_bits_to_f32(bits)


@functools.lru_cache(maxsize=8)
def _queries(W, li):
    return f32(synth.queries(W.seed, li, W.num_q, W.H, W.D))


@functools.lru_cache(maxsize=8)
def _iq(W, li):
    return (f32(synth.index_queries(W.seed, li, W.num_q, W.H_I, W.d_I)),
            synth.index_weights(W.seed, li, W.num_q, W.H_I))


@functools.lru_cache(maxsize=4)
def _kI_seq(W, s):
    base, n = int(W.seq_start[s]), int(W.lengths[s])
    k = f32(synth.index_k_rows(W.seed, base, n, W.d_I)).astype(np.float64)
    if W.append:
        k[n - 1] = f32(synth.append_index_k(W.seed, 0, W.num_seqs, W.d_I))[s]
    return k


def kv_rows_for(W, s, positions):
    """fp32 main-KV rows of sequence s at the given positions (append applied)."""
    base, n = int(W.seq_start[s]), int(W.lengths[s])
    rows = base + np.asarray(positions, dtype=np.int64)
    out = np.empty((rows.shape[0], W.D), dtype=np.float32)
    blocks = rows // synth.ROW_BLOCK
    for b in np.unique(blocks):
        blk = synth.kv_rows(W.seed, int(b) * synth.ROW_BLOCK, synth.ROW_BLOCK, W.D,
                            W.outlier_frac)
        m = blocks == b
        out[m] = blk[rows[m] - int(b) * synth.ROW_BLOCK]
    if W.append:
        last = np.asarray(positions) == n - 1
        if last.any():
            out[last] = synth.append_rows(W.seed, 0, W.num_seqs, W.D)[s]
    return out


def window_rows(W, li, q):
    """bf16 window rows (as fp32) a query reads: token positions max(0, t-W+1)..t."""
    s = q // W.q_per_seq
    t = int(W.q_pos()[q])
    pos = R.window_positions(t, W.window)
    if pos.shape[0] == 0:
        return np.zeros((0, W.D))
    return f32(synth.swa_rows(W.seed, li, s, int(pos[0]), pos.shape[0], W.D))


def query_layers(W, q, with_attention=True):
    """Per layer of the schedule: dict(indices, pool (Full layers that build it),
    out, lse) for query q, computed by the oracle."""
    s = q // W.q_per_seq
    vis = int(W.q_visible()[q])
    kI = _kI_seq(W, s)[:vis]
    res, latest, pool, pool_built = [], None, None, False
    for li, mode in enumerate(W.modes):
        r = {"mode": mode}
        if mode == synth.FULL:
            qI, w = _iq(W, li)
            sc = R.index_scores(qI[q], w[q], kI)
            latest = R.topk_ascending(sc, W.topk)
            if W.pool_blocks and not pool_built:
                pool = R.build_pool(sc, W.pool_blocks, W.block)
                pool_built = True
                r["pool"] = pool
        elif mode == synth.REINDEX:
            qI, w = _iq(W, li)
            latest = R.reindex(qI[q], w[q], kI, pool, W.block, vis, W.topk)
        r["indices"] = latest
        if with_attention:
            sel = latest[latest >= 0]
            codes, scales = R.quantize_rows(kv_rows_for(W, s, sel))
            deq = R.dequantize_rows(codes, scales)
            out, lse = R.sparse_attention(_queries(W, li)[q], deq, window_rows(W, li, q),
                                          1.0 / math.sqrt(W.D))
            r["out"], r["lse"] = out, lse
        res.append(r)
    return res


def attn_close(got, want, atol=2e-2, rel_l2=1e-2):
    """The attention tolerance: max-abs <= atol and relative L2 <= rel_l2."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    rl2 = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    return float(err.max()) <= atol and rl2 <= rel_l2, float(err.max()), float(rl2)
