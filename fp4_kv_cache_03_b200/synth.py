"""Seeded synthetic inputs shaped like the CSA2 workloads on the V4.1-Flash pages.

This module holds random-number generation, data-type packing (fp32 -> bf16 bit
patterns) and workload shapes only.  It contains none of the method's
arithmetic: no quantisation, no indexer score, no selection, no attention.
The CUDA path (tests, bench) and the CPU oracle both take their inputs from
here; neither imports the other.

Every array is a pure function of (seed, stream, block): rows are generated in
blocks of ``ROW_BLOCK`` so that any row range can be regenerated on its own,
e.g. by the oracle when it checks a sample of a 1M-entry cache.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

ROW_BLOCK = 4096

# independent random streams, one per kind of input
(S_KV, S_IDXK, S_Q, S_QI, S_W, S_SWA, S_APPEND_X, S_APPEND_K, S_LEN, S_OUTLIER, S_COMP_X,
 S_COMP_W) = range(12)


def _rng(seed: int, stream: int, *more: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), *[int(m) for m in more]])


# ----------------------------------------------------------------------------
# bf16 bit patterns (data packing, round-to-nearest-even)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); return uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _int_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    # small integers are exact in bf16
    return f32_to_bf16_bits(v.astype(np.float32))


# ----------------------------------------------------------------------------
# row generators (block-seeded)
# ----------------------------------------------------------------------------
def _blocked(fn, start: int, count: int, width: int, dtype) -> np.ndarray:
    out = np.empty((count, width), dtype=dtype)
    if count == 0:
        return out
    b0, b1 = start // ROW_BLOCK, (start + count - 1) // ROW_BLOCK
    for b in range(b0, b1 + 1):
        blk = fn(b)
        lo = max(start, b * ROW_BLOCK)
        hi = min(start + count, (b + 1) * ROW_BLOCK)
        out[lo - start:hi - start] = blk[lo - b * ROW_BLOCK:hi - b * ROW_BLOCK]
    return out


def kv_rows(seed: int, start: int, count: int, D: int,
            outlier_frac: float = 0.0, outlier_scale: float = 4.0) -> np.ndarray:
    """Main-KV rows before quantisation: fp32 N(0,1); a fraction of rows x scale."""
    def blk(b):
        r = _rng(seed, S_KV, D, b)
        v = r.standard_normal((ROW_BLOCK, D), dtype=np.float32)
        if outlier_frac > 0.0:
            m = _rng(seed, S_OUTLIER, b).random(ROW_BLOCK) < outlier_frac
            v[m] *= np.float32(outlier_scale)
        return v
    return _blocked(blk, start, count, D, np.float32)


def index_k_rows(seed: int, start: int, count: int, d_I: int,
                 lo: int = -8, hi: int = 8) -> np.ndarray:
    """Indexer-K rows: integers uniform in [lo, hi], stored as bf16 bits."""
    def blk(b):
        r = _rng(seed, S_IDXK, d_I, b)
        return _int_to_bf16_bits(r.integers(lo, hi + 1, size=(ROW_BLOCK, d_I)))
    return _blocked(blk, start, count, d_I, np.uint16)


def queries(seed: int, layer: int, num_q: int, H: int, D: int) -> np.ndarray:
    """Attention queries [num_q, H, D], bf16 N(0,1)."""
    r = _rng(seed, S_Q, layer)
    return f32_to_bf16_bits(r.standard_normal((num_q, H, D), dtype=np.float32))


def index_queries(seed: int, layer: int, num_q: int, H_I: int, d_I: int,
                  lo: int = -8, hi: int = 8) -> np.ndarray:
    """Indexer queries [num_q, H_I, d_I]: integers in [lo, hi] as bf16 bits."""
    r = _rng(seed, S_QI, layer)
    return _int_to_bf16_bits(r.integers(lo, hi + 1, size=(num_q, H_I, d_I)))


def index_weights(seed: int, layer: int, num_q: int, H_I: int,
                  lo: int = 1, hi: int = 4) -> np.ndarray:
    """Per-query per-head indexer weights [num_q, H_I]: integers in [lo, hi], fp32."""
    r = _rng(seed, S_W, layer)
    return r.integers(lo, hi + 1, size=(num_q, H_I)).astype(np.float32)


def swa_rows(seed: int, layer: int, seq: int, start: int, count: int, D: int) -> np.ndarray:
    """Sliding-window KV rows of one layer and sequence, bf16 N(0,1) bits; row r of the
    result is token position start + r."""
    def blk(b):
        r = _rng(seed, S_SWA, layer, seq, D, b)
        return f32_to_bf16_bits(r.standard_normal((ROW_BLOCK, D), dtype=np.float32))
    return _blocked(blk, start, count, D, np.uint16)


def append_rows(seed: int, step: int, count: int, D: int) -> np.ndarray:
    """New main-KV rows appended by one decode step: fp32 N(0,1)."""
    return _rng(seed, S_APPEND_X, step, D).standard_normal((count, D), dtype=np.float32)


def append_index_k(seed: int, step: int, count: int, d_I: int) -> np.ndarray:
    r = _rng(seed, S_APPEND_K, step, d_I)
    return _int_to_bf16_bits(r.integers(-8, 9, size=(count, d_I)))


def compressor_tokens(seed: int, count: int, D_in: int, lo: int = -8, hi: int = 8) -> np.ndarray:
    """Token rows entering the sequence compressor: integers in [lo, hi] as bf16 bits."""
    r = _rng(seed, S_COMP_X, D_in)
    return _int_to_bf16_bits(r.integers(lo, hi + 1, size=(count, D_in)))


def compressor_map(seed: int, D: int, K: int, lo: int = -4, hi: int = 4, shift: int = 6) -> np.ndarray:
    """The compressor's synthetic linear map, transposed ([D][K]): integers in [lo, hi]
    times 2^-shift, as bf16 bits (exact).  With integer token rows every fp32 accumulation of
    the map is exact, so the quantised entries can be compared bit for bit."""
    r = _rng(seed, S_COMP_W, D, K)
    v = r.integers(lo, hi + 1, size=(D, K)).astype(np.float32) * np.float32(2.0 ** -shift)
    return f32_to_bf16_bits(v)


def ragged_lengths(seed: int, num_seqs: int, lo: int, hi: int) -> np.ndarray:
    """Context lengths drawn log-uniform in [lo, hi]."""
    u = _rng(seed, S_LEN).uniform(math.log(lo), math.log(hi), size=num_seqs)
    return np.minimum(np.floor(np.exp(u)).astype(np.int64), hi).astype(np.int32)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
FULL, REINDEX, REUSE = "full", "reindex", "reuse"


@dataclass(frozen=True)
class Workload:
    """Shapes of one CSA2 workload.  Sizes follow the pages' decoder/encoder
    description (window 128, Top-512, a pool of 2048 blocks x 8)."""
    name: str
    seed: int
    num_seqs: int
    lengths: tuple            # stored compressed entries per sequence
    q_per_seq: int            # queries per sequence (decode: 1)
    D: int                    # main-KV dim
    H: int                    # query heads
    H_I: int                  # indexer heads
    d_I: int                  # indexer dim
    topk: int
    window: int
    modes: tuple              # per-layer static mode
    pool_blocks: int = 0      # 0: no hierarchical pool
    block: int = 8
    ratio: int = 1            # compression ratio m of the sequence axis
    outlier_frac: float = 0.0
    append: bool = False      # one new entry per sequence per step
    q_token0: tuple = field(default=())  # token position of each sequence's first query

    @property
    def num_q(self) -> int:
        return self.num_seqs * self.q_per_seq

    @property
    def seq_start(self) -> np.ndarray:
        s = np.zeros(self.num_seqs, dtype=np.int64)
        s[1:] = np.cumsum(np.asarray(self.lengths, dtype=np.int64))[:-1]
        return s

    @property
    def total_rows(self) -> int:
        return int(np.sum(np.asarray(self.lengths, dtype=np.int64)))

    def q_pos(self) -> np.ndarray:
        """Token position t of every query (int64)."""
        out = np.empty(self.num_q, dtype=np.int64)
        for s in range(self.num_seqs):
            t0 = self.q_token0[s] if self.q_token0 else self.lengths[s] * self.ratio - 1
            out[s * self.q_per_seq:(s + 1) * self.q_per_seq] = t0 + np.arange(self.q_per_seq)
        return out

    def q_visible(self) -> np.ndarray:
        """Entries a query at token t sees: an entry becomes visible once all m of
        its tokens are <= t, i.e. floor((t+1)/m); never more than are stored."""
        t = self.q_pos()
        vis = (t + 1) // self.ratio
        lens = np.repeat(np.asarray(self.lengths, dtype=np.int64), self.q_per_seq)
        return np.minimum(vis, lens).astype(np.int32)

    def max_visible(self) -> int:
        return int(self.q_visible().max()) if self.num_q else 0


def _decoder_modes(groups: int, first_full: bool = True) -> tuple:
    modes = []
    for g in range(groups):
        modes.append(FULL if (g == 0 and first_full) else REINDEX)
        modes += [REUSE] * 3
    return tuple(modes)


def workload(name: str) -> Workload:
    if name == "tiny":
        return Workload("tiny", 0, 1, (4096,), 1, 128, 16, 4, 64, 64, 128, (FULL,))
    if name == "decoder_group_128k":
        return Workload("decoder_group_128k", 1, 1, (131072,), 1, 512, 64, 16, 128, 512, 128,
                        (FULL, REUSE, REUSE, REUSE), outlier_frac=0.01)
    if name == "hier_decoder_1m":
        return Workload("hier_decoder_1m", 2, 1, (1048576,), 1, 512, 64, 16, 128, 512, 128,
                        (FULL,) + (REINDEX,) * 4, pool_blocks=2048, block=8)
    if name == "encoder_chunk":
        return Workload("encoder_chunk", 3, 1, (32768,), 4096, 512, 64, 16, 128, 512, 128,
                        (FULL,) + (REUSE,) * 5, ratio=2, q_token0=(61440,))
    if name == "ragged_decode":
        lens = tuple(int(v) for v in ragged_lengths(4, 64, 4096, 262144))
        return Workload("ragged_decode", 4, 64, lens, 1, 512, 64, 16, 128, 512, 128, (FULL,),
                        append=True)
    if name == "decoder_step_128k":
        return Workload("decoder_step_128k", 1, 1, (131072,), 1, 512, 64, 16, 128, 512, 128,
                        _decoder_modes(5), pool_blocks=2048, block=8, outlier_frac=0.01,
                        append=True)
    if name.startswith("encoder_group"):
        # the encoder stack: 3 groups of 6 layers at ratio 2, each group with its own cache
        # (its Full layer computes its own main KV and indexer K); group g draws its own
        # streams (seed 3 + 10 g)
        g = int(name[len("encoder_group"):])
        return Workload(name, 3 + 10 * g, 1, (32768,), 4096, 512, 64, 16, 128, 512, 128,
                        (FULL,) + (REUSE,) * 5, ratio=2, q_token0=(61440,))
    if name == "decoder_step_1m":
        return Workload("decoder_step_1m", 2, 1, (1048576,), 1, 512, 64, 16, 128, 512, 128,
                        _decoder_modes(5), pool_blocks=2048, block=8, outlier_frac=0.01,
                        append=True)
    raise KeyError(name)


WORKLOADS = ("tiny", "decoder_group_128k", "hier_decoder_1m", "encoder_chunk", "ragged_decode",
             "decoder_step_128k", "decoder_step_1m")
# the 18-layer encoder stack: 3 groups x (Full + 5 Reuse) at ratio 2
ENCODER_STACK = ("encoder_group0", "encoder_group1", "encoder_group2")
