"""CPU oracle for the CSA2 attention step over an FP4 global KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module; only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` do.  It shares no code with the CUDA path: its inputs come
from ``fp4_kv_cache_03_b200.synth`` (random numbers and shapes only) and are
passed in as arrays.

Plain, slow and meant to be read against the pages.  Floating-point work is in
float64, except where a float decides an integer code (the FP4 encoder): there
both sides decide in fp32, the kernel's precision, because the pages fix none.

Sources (pages on DeepSeek-V4.1-Flash; cited by title and section):
  [OVR]   "DeepSeek-V4.1-Flash：推动 KV 缓存压缩极限" (course overview page), 摘要 (abstract)
  [SURV]  "DeepSeek-V4.1-Flash 技术调研报告" (gkm0120.cn), §2.2.1 三个压缩维度,
          §2.2.2 Full / Reindex / Reuse 三档模式 (modes table), §2.2.3 分层稀疏索引器,
          §五 KV Cache 效率对比 (KV table)
  [MTP]   "DeepSeek V4.1 Flash 发布：KV cache 降到 890 字节/token…" (aprilzz.com,
          relaying MarkTechPost), sections "CSA2：在层的维度上共享缓存",
          "FP4 KV 与部署层的几个改动", "把 prefill 砍掉一半"
  [NEWS]  aimodeling.com news, section "第二层:CSA2 三模式加 FP4"
  [OCP]   the OCP Microscaling Formats spec v1.0 (FP4 E2M1, FP8 E4M3 element
          formats), which the pages name by format only

Readings where the pages are silent (each also listed in the design notes):
  * indexer score s[e] = sum_h w_h * ReLU(q_h . k_e)
  * Top-K order (score desc, position asc); output ascending; pad with -1
  * block score = max over the block's visible members; blocks aligned [8j, 8j+8)
  * scale = E4M3_RNE_satfinite(fp32(amax / 6)); code = E2M1_RNE_satfinite(fp32(x / scale));
    a zero scale gives signed-zero codes; low nibble = even channel
  * attention: one joint softmax over [selected compressed rows ; window rows],
    K = V = the single dequantised row, scale 1/sqrt(D), no dedup, no sink
"""
from __future__ import annotations

import numpy as np

# ============================================================================
# element formats  [OCP]; named by [MTP] "FP4 KV 与部署层的几个改动" and [SURV] §2.2.1
# ============================================================================

def e2m1_decode_table() -> np.ndarray:
    """Value of each 4-bit E2M1 code: sign in bit 3, 2 exponent bits (bias 1),
    1 mantissa bit; exponent field 0 is subnormal (m * 0.5)."""
    out = np.empty(16, dtype=np.float64)
    for code in range(16):
        s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
        mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
        out[code] = -mag if s else mag
    return out


def e4m3_decode_table() -> np.ndarray:
    """Value of each 8-bit E4M3 code: sign bit 7, 4 exponent bits (bias 7),
    3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN;
    there is no infinity, so the largest finite magnitude is S.1111.110 = 448."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            out[code] = np.nan
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out[code] = -mag if s else mag
    return out


def _encode_nearest_even(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each magnitude; on an exact tie the
    even index (even code) wins; beyond the last value the last index (satfinite).
    ``grid`` holds the non-negative finite values in code order (ascending)."""
    mag = np.asarray(mag, dtype=np.float64).reshape(-1)
    out = np.empty(mag.shape[0], dtype=np.int64)
    CH = 1 << 15
    for i in range(0, mag.shape[0], CH):
        m = mag[i:i + CH, None]
        d = np.abs(m - grid[None, :])                      # distance to every value
        best = d.min(axis=1, keepdims=True)
        cand = d == best                                   # one or two nearest values
        idx = np.arange(grid.shape[0])[None, :]
        even = cand & (idx % 2 == 0)
        pick = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
        # satfinite: at or beyond the largest value the largest code is taken (this is
        # also what nearest gives, but for huge inputs every distance rounds alike)
        pick = np.where(m[:, 0] >= grid[-1], grid.shape[0] - 1, pick)
        out[i:i + CH] = pick
    return out


def e4m3_encode(v) -> np.ndarray:
    """fp32 -> E4M3 code, round to nearest (ties to even code), saturating to
    +-448.  Input must be finite."""
    v = np.asarray(v, dtype=np.float32)
    grid = e4m3_decode_table()[:127]                       # codes 0x00..0x7E, ascending
    code = _encode_nearest_even(np.abs(v.astype(np.float64)), grid)
    sign = np.signbit(v).reshape(-1).astype(np.int64)
    return ((sign << 7) | code).astype(np.uint8).reshape(v.shape)


def e2m1_encode(v) -> np.ndarray:
    """fp32 -> E2M1 code, round to nearest (ties to even code), saturating to
    +-6; the sign bit follows the input's sign bit (so -0.1 -> code 0x8)."""
    v = np.asarray(v, dtype=np.float32)
    grid = e2m1_decode_table()[:8]                         # 0, .5, 1, 1.5, 2, 3, 4, 6
    code = _encode_nearest_even(np.abs(v.astype(np.float64)), grid)
    sign = np.signbit(v).reshape(-1).astype(np.int64)
    return ((sign << 3) | code).astype(np.uint8).reshape(v.shape)


# ============================================================================
# a1  quantise + append   [MTP] "FP4 KV 与部署层的几个改动"; [OVR] 摘要; [SURV] §2.2.1
#     E2M1 values, one E4M3 scale per 16 channels, NVFP4-like but no global scale
# ============================================================================
GROUP = 16


def quantize_rows(x: np.ndarray):
    """x: fp32 [B, D] -> (codes uint8 [B, D/2], scales uint8 [B, D/16]).

    Per group g of 16 channels: amax = max |x|; scale byte s = E4M3(fp32(amax / 6));
    each value's code is E2M1(fp32(x / dec(s))) (or a signed zero if dec(s) = 0).
    Byte k of a row holds code[2k] in its low nibble and code[2k+1] in its high nibble.
    """
    x = np.asarray(x, dtype=np.float32)
    B, D = x.shape
    assert D % GROUP == 0
    g = x.reshape(B, D // GROUP, GROUP)
    amax = np.max(np.abs(g), axis=2)                                   # fp32, exact
    s_code = e4m3_encode(amax / np.float32(6.0))                       # fp32 divide
    s_val = e4m3_decode_table()[s_code].astype(np.float32)             # exact in fp32
    with np.errstate(divide="ignore", invalid="ignore"):
        q = g / s_val[:, :, None]                                      # fp32 divide
    q = np.where(s_val[:, :, None] == 0, np.where(np.signbit(g), np.float32(-0.0),
                                                   np.float32(0.0)), q)
    codes = e2m1_encode(q).reshape(B, D)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, s_code.astype(np.uint8)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(codes [B, D/2], scales [B, D/16]) -> float64 [B, D]: e2m1(code) * e4m3(scale)."""
    codes = np.asarray(codes, dtype=np.uint8)
    B, half = codes.shape
    D = half * 2
    nib = np.empty((B, D), dtype=np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    vals = e2m1_decode_table()[nib]
    sc = e4m3_decode_table()[np.asarray(scales, dtype=np.uint8)]
    return vals * np.repeat(sc, GROUP, axis=1)


def bytes_per_entry(D: int) -> int:
    """Stored bytes of one main-KV entry: D/2 code bytes + D/16 scale bytes."""
    return D // 2 + D // GROUP


# ============================================================================
# sequence-axis compressor  [SURV] §2.2.1 三个压缩维度 (sequence dimension: every m tokens
#     become one entry; the compressor is inherited from V4); [MTP] "CSA2：…" (encoder groups
#     at ratio 2).  The pages give no formula: here a linear map of the m token rows.
# ============================================================================

def compress_rows(x_tokens: np.ndarray, m: int, w_t: np.ndarray) -> np.ndarray:
    """x_tokens [n*m, D_in] -> entries float64 [n, D]: entry j = concat(x_{jm}, ...,
    x_{jm+m-1}) @ w_t^T, w_t being the map's transpose [D, m*D_in]."""
    x = np.asarray(x_tokens, np.float64)
    n = x.shape[0] // m
    xcat = x[:n * m].reshape(n, m * x.shape[1])
    return xcat @ np.asarray(w_t, np.float64).T


def compress_quantize(x_tokens: np.ndarray, m: int, w_t: np.ndarray):
    """The compressor followed by a1: the entries rounded to fp32, then quantize_rows."""
    return quantize_rows(compress_rows(x_tokens, m, w_t).astype(np.float32))


# ============================================================================
# a2  indexer score     [SURV] §2.2.2 modes table, §2.2.3; [MTP] "CSA2：在层的维度上共享缓存"
#     (the pages name the indexer; the score formula is a stated reading)
# ============================================================================

def index_scores(qI: np.ndarray, w: np.ndarray, kI: np.ndarray) -> np.ndarray:
    """qI [H_I, d_I], w [H_I], kI [n, d_I] -> float64 [n]:
    s[e] = sum_h w[h] * max(0, sum_d qI[h, d] * kI[e, d])."""
    dots = np.asarray(kI, np.float64) @ np.asarray(qI, np.float64).T   # [n, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w, np.float64)


def index_scores_e4m3(qI: np.ndarray, w: np.ndarray, kI: np.ndarray) -> np.ndarray:
    """The compact indexer (indexer K and Q stored as E4M3 bytes): each value of qI and kI is
    first rounded to E4M3 (nearest, ties to even, saturating to +-448), then scored exactly
    as index_scores does.  [OVR] 摘要 puts the whole global cache at 890 bytes per token, which
    leaves little room for a 2-byte indexer key."""
    dec = e4m3_decode_table()
    q8 = dec[e4m3_encode(np.asarray(qI, np.float32))]
    k8 = dec[e4m3_encode(np.asarray(kI, np.float32))]
    return index_scores(q8, w, k8)


# ============================================================================
# a3  Top-K selection   [MTP] "CSA2：…" (Full selects a new Top-512)
# ============================================================================

def topk_ascending(scores: np.ndarray, k: int, ids: np.ndarray | None = None) -> np.ndarray:
    """The k candidates ranked first by (score descending, id ascending), listed
    by ascending id and padded with -1 to length k.  ``ids`` defaults to 0..n-1."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    ids = np.arange(n, dtype=np.int64) if ids is None else np.asarray(ids, dtype=np.int64)
    order = np.lexsort((ids, -scores))          # primary: -score, secondary: id
    chosen = np.sort(ids[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.shape[0]] = chosen
    return out


# ============================================================================
# a4  hierarchical pool  [SURV] §2.2.3 分层稀疏索引器; [MTP] "CSA2：…" (at most 16,384
#     positions = 2048 blocks x 8, built by the decoder's first Full layer)
# ============================================================================

def block_scores(scores: np.ndarray, block: int) -> np.ndarray:
    """Block j covers positions [block*j, block*j + block) that exist; its score is
    the maximum score of those positions."""
    n = scores.shape[0]
    nb = -(-n // block)
    out = np.empty(nb, dtype=np.float64)
    for j in range(nb):
        out[j] = np.max(scores[j * block:min(n, (j + 1) * block)])
    return out


def build_pool(scores: np.ndarray, pool_blocks: int, block: int) -> np.ndarray:
    """Top ``pool_blocks`` blocks by (block score desc, block id asc), ascending, -1 padded."""
    return topk_ascending(block_scores(scores, block), pool_blocks)


def pool_positions(pool: np.ndarray, block: int, visible: int) -> np.ndarray:
    """Positions covered by the pool's blocks that are visible, ascending."""
    pos = [j * block + i for j in pool if j >= 0 for i in range(block) if j * block + i < visible]
    return np.asarray(sorted(pos), dtype=np.int64)


# ============================================================================
# a5  Reindex over the pool  [SURV] §2.2.2 (Reindex: own indexer Q, re-select) and
#     §2.2.3; [MTP] "CSA2：…" (Reindex scores only inside the bounded pool)
# ============================================================================

def reindex(qI, w, kI_rows: np.ndarray, pool: np.ndarray, block: int, visible: int,
            k: int) -> np.ndarray:
    """kI_rows: the sequence's indexer-K rows (at least ``visible`` of them).
    Score only the pool's visible positions with this layer's qI/w; Top-k."""
    pos = pool_positions(pool, block, visible)
    s = index_scores(qI, w, kI_rows[pos]) if pos.shape[0] else np.zeros(0)
    return topk_ascending(s, k, ids=pos)


# ============================================================================
# a7  sparse attention + sliding window  [MTP] "把 prefill 砍掉一半" (every layer keeps a
#     128-token SWA) and "CSA2：…" (each layer keeps its own main Q and SWA KV)
# ============================================================================

def sparse_attention(q: np.ndarray, kv_sel: np.ndarray, kv_win: np.ndarray, scale: float):
    """q [H, D]; kv_sel [n1, D] dequantised selected rows; kv_win [n2, D] window rows.
    Logits l[h, j] = scale * q[h] . kv[j] over the concatenation kv = [kv_sel; kv_win];
    one softmax per head; out[h] = sum_j p[h, j] kv[j]; lse[h] = log sum_j exp(l[h, j]).
    Returns (out float64 [H, D], lse float64 [H]); with no rows at all, out = 0, lse = -inf."""
    q = np.asarray(q, np.float64)
    kv = np.concatenate([np.asarray(kv_sel, np.float64).reshape(-1, q.shape[1]),
                         np.asarray(kv_win, np.float64).reshape(-1, q.shape[1])], axis=0)
    if kv.shape[0] == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    logits = scale * (q @ kv.T)                                        # [H, n]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    l = e.sum(axis=1, keepdims=True)
    return (e / l) @ kv, (m + np.log(l))[:, 0]


def window_positions(t: int, window: int) -> np.ndarray:
    """Token positions of the sliding window of a query at token t: max(0, t-W+1) .. t."""
    return np.arange(max(0, t - window + 1), t + 1, dtype=np.int64)


# ============================================================================
# a6 + mode schedule   [SURV] §2.2.2 modes table (Full / Reindex / Reuse);
#     [MTP] "CSA2：…" (Reuse runs no indexer and takes the latest Top-K; decoder groups
#     are Full + 3 Reuse, then Reindex + 3 Reuse)
# ============================================================================

def layer_indices(mode: str, *, scores_full=None, qI=None, w=None, kI_rows=None, pool=None,
                  latest=None, k: int, block: int = 8, visible: int = 0):
    """Indices a layer attends with.  Full: Top-k of the full scores.  Reindex:
    Top-k of its own scores over the pool.  Reuse: the latest Full/Reindex indices."""
    if mode == "full":
        return topk_ascending(scores_full, k)
    if mode == "reindex":
        return reindex(qI, w, kI_rows, pool, block, visible, k)
    if mode == "reuse":
        assert latest is not None
        return latest
    raise ValueError(mode)
