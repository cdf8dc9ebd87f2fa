"""Device-side set-up and layer schedule of a CSA2 workload (plumbing around libcsa2).

``DeviceWorkload`` puts one synthetic workload (shapes from ``synth``) into HBM:
the FP4 main-KV cache, written through ``csa2_quant_append`` from the seeded fp32
rows; the bf16 indexer keys; per-layer queries, indexer queries/weights and
sliding-window rows.  ``run_step`` drives one pass of the layer schedule through
the C ABI: the optional append, then per layer Full (index + pool), Reindex (pool
re-score) or Reuse (no indexer: the latest indices), each followed by sparse
attention.  No arithmetic of the method happens here.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import csa2, synth


def _bf16(a: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 patterns -> torch.bfloat16 tensor on ``device``."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


@dataclass
class LayerInputs:
    mode: str
    q: torch.Tensor                # [num_q, H, D] bf16
    qI: torch.Tensor | None        # [num_q, H_I, d_I] bf16 (Full / Reindex)
    w: torch.Tensor | None         # [num_q, H_I] fp32
    swa: torch.Tensor              # [swa_rows, D] bf16
    swa_start: torch.Tensor        # [num_seqs] int64: row of token position 0


class DeviceWorkload:
    FILL_ROWS = 65536

    STASH_LIMIT = 256 << 20   # keep Reuse stashes for batches whose stash stays this small

    def __init__(self, W: synth.Workload, device="cuda", fill=True, use_stash=True,
                 indexer_e4m3=False):
        self.W = W
        self.device = device
        dev = device
        cap = W.total_rows
        self.cap = cap
        self.kv_codes = torch.zeros(cap, W.D // 2, dtype=torch.uint8, device=dev)
        self.kv_scales = torch.zeros(cap, W.D // 16, dtype=torch.uint8, device=dev)
        self.idx_k = torch.zeros(cap, W.d_I, dtype=torch.bfloat16, device=dev)
        self.seq_start = torch.from_numpy(W.seq_start).to(dev)
        self.seq_len = torch.tensor(W.lengths, dtype=torch.int32, device=dev)
        self.seqs = csa2.make_seqs(self.seq_start, self.seq_len, W.q_per_seq)
        self.q_pos = torch.from_numpy(W.q_pos()).to(dev)
        vis = W.q_visible()
        self.max_visible = int(vis.max())
        self.q_visible = torch.from_numpy(vis).to(dev) if W.ratio != 1 or W.q_per_seq > 1 else None
        self.ws_append = csa2.workspace(csa2.quant_append_workspace(), dev)
        if fill:
            self._fill_cache()
        self.layers = [self._layer_inputs(i, m) for i, m in enumerate(W.modes)]
        # compact indexer path: E4M3 indexer K (converted from the bf16 cache) and queries
        self.indexer_e4m3 = indexer_e4m3
        if indexer_e4m3:
            self.idx_k = csa2.e4m3_from_bf16(self.idx_k)
            for L in self.layers:
                if L.qI is not None:
                    L.qI = csa2.e4m3_from_bf16(L.qI)
            torch.cuda.synchronize(dev)
        # outputs / workspaces
        nq = W.num_q
        self.has_pool = W.pool_blocks > 0
        self.ws_full = csa2.workspace(csa2.index_full_workspace(
            nq, self.max_visible, W.topk, W.pool_blocks, W.block), dev)
        self.ws_pool = csa2.workspace(csa2.index_pool_workspace(
            nq, max(W.pool_blocks, 1), W.block, W.topk), dev) if self.has_pool else None
        self.ws_attn = csa2.workspace(csa2.sparse_attn_workspace(nq, W.H, W.D, W.topk, W.window), dev)
        # staged FP4 rows (codes, scales, validity) of the latest Full/Reindex layer, for
        # its Reuse layers
        sb = csa2.sparse_attn_stash_bytes(nq, W.D, W.topk)
        self.stash = (torch.empty(sb, dtype=torch.uint8, device=dev)
                      if use_stash and 0 < sb <= self.STASH_LIMIT else None)
        self.pool = torch.full((nq, max(W.pool_blocks, 1)), -1, dtype=torch.int32, device=dev)
        n_idx = sum(1 for m in W.modes if m != synth.REUSE)
        self.indices = [torch.full((nq, W.topk), -1, dtype=torch.int32, device=dev)
                        for _ in range(n_idx)]
        self.out = [torch.zeros(nq, W.H, W.D, dtype=torch.float32, device=dev) for _ in W.modes]
        self.lse = [torch.zeros(nq, W.H, dtype=torch.float32, device=dev) for _ in W.modes]
        self.scale = 1.0 / math.sqrt(W.D)
        # append inputs (one new entry per sequence), fixed for step 0
        if W.append:
            self.append_x = torch.from_numpy(synth.append_rows(W.seed, 0, W.num_seqs, W.D)).to(dev)
            self.append_k = _bf16(synth.append_index_k(W.seed, 0, W.num_seqs, W.d_I), dev)
            self.append_dst = (self.seq_start + self.seq_len.to(torch.int64) - 1).contiguous()

    # -------------------------------------------------------------------------------
    def _fill_cache(self):
        W, dev = self.W, self.device
        for s in range(W.num_seqs):
            base, n = int(W.seq_start[s]), int(W.lengths[s])
            for r0 in range(0, n, self.FILL_ROWS):
                c = min(self.FILL_ROWS, n - r0)
                # every sequence draws from its own row range of the seeded streams
                x = torch.from_numpy(synth.kv_rows(W.seed, base + r0, c, W.D, W.outlier_frac)).to(dev)
                dst = torch.arange(base + r0, base + r0 + c, dtype=torch.int64, device=dev)
                k = _bf16(synth.index_k_rows(W.seed, base + r0, c, W.d_I), dev)
                csa2.quant_append(x, dst, self.kv_codes, self.kv_scales, self.ws_append,
                                  idx_k_in=k, idx_k=self.idx_k)
        torch.cuda.synchronize(dev)
        st = csa2.status_fetch(self.ws_append)
        if st != csa2.OK:
            raise csa2.CSA2Error(st, "cache fill")

    def window_span(self, s: int):
        """Token positions [lo, hi] of sequence s whose window rows a query may read."""
        W = self.W
        t = W.q_pos()[s * W.q_per_seq:(s + 1) * W.q_per_seq]
        return max(0, int(t.min()) - W.window + 1), int(t.max())

    def _layer_inputs(self, li: int, mode: str) -> LayerInputs:
        W, dev = self.W, self.device
        q = _bf16(synth.queries(W.seed, li, W.num_q, W.H, W.D), dev)
        qI = w = None
        if mode != synth.REUSE:
            qI = _bf16(synth.index_queries(W.seed, li, W.num_q, W.H_I, W.d_I), dev)
            w = torch.from_numpy(synth.index_weights(W.seed, li, W.num_q, W.H_I)).to(dev)
        rows, starts, r = [], [], 0
        for s in range(W.num_seqs):
            lo, hi = self.window_span(s)
            rows.append(synth.swa_rows(W.seed, li, s, lo, hi - lo + 1, W.D))
            starts.append(r - lo)
            r += hi - lo + 1
        swa = _bf16(np.concatenate(rows, 0), dev)
        return LayerInputs(mode, q, qI, w, swa, torch.tensor(starts, dtype=torch.int64, device=dev))

    # -------------------------------------------------------------------------------
    def append(self, stream=None):
        if self.idx_k.dtype == torch.uint8:
            csa2.quant_append_e4m3k(self.append_x, self.append_dst, self.kv_codes, self.kv_scales,
                                    self.ws_append, self.append_k, self.idx_k, stream=stream)
        else:
            csa2.quant_append(self.append_x, self.append_dst, self.kv_codes, self.kv_scales,
                              self.ws_append, idx_k_in=self.append_k, idx_k=self.idx_k, stream=stream)

    def run_step(self, stream=None, attention=True, via_layer_step=False, append=True):
        """One pass of the layer schedule; returns the index tensor each layer used.
        With ``via_layer_step`` every layer is one csa2_layer_step call (index + attention
        by the layer's mode).  ``append=False`` leaves out the step's append."""
        W = self.W
        if W.append and append:
            self.append(stream)
        latest, used, n_idx, pool_built = None, [], 0, False
        for li, L in enumerate(self.layers):
            if L.mode == synth.FULL:
                idx = self.indices[n_idx]
                n_idx += 1
                build = self.has_pool and not pool_built
                if via_layer_step and attention:
                    self.layer_step(li, idx, build_pool=build, stream=stream)
                else:
                    csa2.index_full(L.qI, L.w, self.idx_k, self.seqs, W.topk, idx, self.ws_full,
                                    self.max_visible, q_visible=self.q_visible,
                                    pool_blocks=W.pool_blocks if build else 0, block=W.block,
                                    pool=self.pool if build else None, stream=stream)
                pool_built = pool_built or build
                latest = idx
            elif L.mode == synth.REINDEX:
                idx = self.indices[n_idx]
                n_idx += 1
                if via_layer_step and attention:
                    self.layer_step(li, idx, stream=stream)
                else:
                    csa2.index_pool(L.qI, L.w, self.idx_k, self.seqs, self.pool, W.pool_blocks,
                                    W.block, W.topk, idx, self.ws_pool, q_visible=self.q_visible,
                                    stream=stream)
                latest = idx
            else:  # Reuse: no indexer, the latest indices
                assert latest is not None, "a Reuse layer needs an earlier Full/Reindex layer"
                if via_layer_step and attention:
                    self.layer_step(li, latest, stream=stream)
            used.append(latest)
            if attention and not via_layer_step:
                self.attend(li, latest, stream)
        return used

    def layer_step(self, li: int, indices, build_pool=False, stream=None):
        """Layer li through csa2_layer_step: its mode's indexer (into ``indices``) and
        attention; a Reuse layer attends with ``indices`` as given."""
        L, W = self.layers[li], self.W
        attn = dict(q=L.q, swa_kv=L.swa, swa_start=L.swa_start, q_pos=self.q_pos,
                    window=W.window, softmax_scale=self.scale, out=self.out[li], lse=self.lse[li],
                    ws=self.ws_attn, stash=self.stash)
        ix = None
        if L.mode == synth.FULL:
            ix = dict(qI=L.qI, w=L.w, idx_k=self.idx_k, ws=self.ws_full, q_visible=self.q_visible,
                      max_visible=self.max_visible, pool_blocks=W.pool_blocks if build_pool else 0,
                      block=W.block, pool=self.pool if build_pool else None)
        elif L.mode == synth.REINDEX:
            ix = dict(qI=L.qI, w=L.w, idx_k=self.idx_k, ws=self.ws_pool, q_visible=self.q_visible,
                      pool_blocks=W.pool_blocks, block=W.block, pool=self.pool)
        csa2.layer_step(self.MODES[L.mode], self.kv_codes, self.kv_scales, self.seqs, W.topk,
                        indices, attn, ix, stream=stream)

    MODES = {synth.FULL: csa2.MODE_FULL, synth.REINDEX: csa2.MODE_REINDEX, synth.REUSE: csa2.MODE_REUSE}

    def attend(self, li: int, indices, stream=None):
        """Attention of layer li with the given indices; Reuse layers read the stash the
        latest Full/Reindex layer filled."""
        L, W = self.layers[li], self.W
        csa2.sparse_attn(L.q, self.kv_codes, self.kv_scales, self.seqs, indices, L.swa,
                         L.swa_start, self.q_pos, W.window, self.scale, self.out[li],
                         self.ws_attn, lse=self.lse[li], mode=self.MODES[L.mode],
                         stash=self.stash, stream=stream)

    def status(self) -> int:
        """First device-side error recorded by any call (0 = none)."""
        for ws in (self.ws_append, self.ws_full, self.ws_pool, self.ws_attn):
            if ws is not None:
                st = csa2.status_fetch(ws)
                if st != csa2.OK:
                    return st
        return csa2.OK
