"""ctypes binding of libcsa2.so (the C ABI in include/csa2.h).

Argument marshalling only: every step of the CSA2 path runs in the library's CUDA
kernels.  Tensors are PyTorch tensors (device memory and streams are PyTorch's);
each function passes their pointers to the C entry point of the same name and
raises ``CSA2Error`` on a non-OK status.  If the library is not built, importing
anything that needs it raises -- there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int32, c_int64, c_size_t, c_void_p

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcsa2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_TIMEOUT = range(6)
MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
STATUS_BYTES = 256


class CSA2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = f" [{lib().csa2_last_cuda_error().decode()}]" if status == ERR_CUDA else ""
        super().__init__(f"{what}: {status_string(status)} (status {status}){detail}")
        self.status = status


class Seqs(ctypes.Structure):
    """csa2_seqs_t: ragged batch description (device arrays)."""
    _fields_ = [("num_seqs", c_int32), ("q_per_seq", c_int32),
                ("seq_start", c_void_p), ("seq_len", c_void_p), ("q_seq", c_void_p),
                ("block_table", c_void_p), ("max_pages", c_int32)]


class Indexer(ctypes.Structure):
    """csa2_indexer_t: a layer's indexer inputs (FULL / REINDEX)."""
    _fields_ = [("qI", c_void_p), ("w", c_void_p), ("H_I", c_int32), ("d_I", c_int32),
                ("idx_k", c_void_p), ("q_visible", c_void_p), ("max_visible", c_int32),
                ("pool_blocks", c_int32), ("block", c_int32), ("pool", c_void_p),
                ("workspace", c_void_p), ("ws_bytes", c_size_t), ("e4m3", c_int32)]


class Attention(ctypes.Structure):
    """csa2_attention_t: a layer's attention inputs and outputs."""
    _fields_ = [("q", c_void_p), ("H", c_int32), ("D", c_int32), ("swa_kv", c_void_p),
                ("swa_rows", c_int64), ("swa_start", c_void_p), ("q_pos", c_void_p),
                ("window", c_int32), ("swa_ring", c_int32), ("softmax_scale", c_float), ("out", c_void_p),
                ("lse", c_void_p), ("kv_stash", c_void_p), ("stash_bytes", c_size_t),
                ("workspace", c_void_p), ("ws_bytes", c_size_t)]


_lib = None

_SIGS = {
    "csa2_quant_append_workspace": (c_size_t, []),
    "csa2_quant_append": (c_int32, [c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                    c_int64, c_void_p, c_void_p, c_int32, c_void_p, c_size_t,
                                    c_void_p]),
    "csa2_quant_append_e4m3k": (c_int32, [c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                          c_int64, c_void_p, c_void_p, c_int32, c_void_p, c_size_t,
                                          c_void_p]),
    "csa2_e4m3_from_bf16": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p]),
    "csa2_compress_append": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_int32,
                                       c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_size_t,
                                       c_void_p]),
    "csa2_index_full_e4m3": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                       c_int64, Seqs, c_void_p, c_int32, c_int32, c_void_p,
                                       c_int32, c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa2_index_pool_e4m3": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                       c_int64, Seqs, c_void_p, c_void_p, c_int32, c_int32,
                                       c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa2_index_full_workspace": (c_size_t, [c_int32, c_int32, c_int32, c_int32, c_int32]),
    "csa2_index_full": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                  c_int64, Seqs, c_void_p, c_int32, c_int32, c_void_p, c_int32,
                                  c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa2_index_full_noalloc": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                          c_int64, Seqs, c_void_p, c_int32, c_int32, c_void_p,
                                          c_int32, c_int32, c_void_p, c_void_p]),
    "csa2_index_full_noalloc_status": (c_int32, [c_void_p]),
    "csa2_index_pool_workspace": (c_size_t, [c_int32, c_int32, c_int32, c_int32]),
    "csa2_index_pool": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                  c_int64, Seqs, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                  c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa2_sparse_attn_workspace": (c_size_t, [c_int32, c_int32, c_int32, c_int32, c_int32]),
    "csa2_sparse_attn_stash_bytes": (c_size_t, [c_int32, c_int32, c_int32]),
    "csa2_sparse_attn": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                   c_int64, Seqs, c_void_p, c_int32, c_void_p, c_int64, c_void_p,
                                   c_void_p, c_int32, c_int32, c_float, c_void_p, c_void_p, c_int32,
                                   c_void_p, c_size_t, c_void_p, c_size_t, c_void_p]),
    "csa2_layer_step": (c_int32, [c_int32, c_int32, c_void_p, c_void_p, c_int64, Seqs, c_int32,
                                  c_void_p, ctypes.POINTER(Indexer), ctypes.POINTER(Attention),
                                  c_void_p]),
    "csa2_cache_rows": (c_int32, [Seqs, c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    "csa2_gather_rows": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_int32, c_void_p,
                                   c_void_p]),
    "csa2_scatter_rows": (c_int32, [c_void_p, c_int32, c_void_p, c_int32, c_void_p, c_int64,
                                    c_void_p]),
    "csa2_status_reset": (c_int32, [c_void_p, c_void_p]),
    "csa2_status_fetch": (c_int32, [c_void_p, c_void_p]),
    "csa2_status_string": (ctypes.c_char_p, [c_int32]),
    "csa2_last_cuda_error": (ctypes.c_char_p, []),
    "csa2_device_sms": (c_int32, []),
    "csa2_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
}


def lib() -> ctypes.CDLL:
    """Load libcsa2.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m fp4_kv_cache_03_b200.build_lib`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().csa2_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise CSA2Error(status, what)


def _p(t) -> c_void_p | None:
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to libcsa2 must be contiguous"
    return c_void_p(t.data_ptr())


def _s(stream) -> c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def _u16(t):
    """bf16 tensors travel as their 16-bit patterns."""
    if t is None:
        return None
    assert t.dtype in (torch.bfloat16, torch.uint16, torch.int16), t.dtype
    return _p(t)


def make_seqs(seq_start: torch.Tensor | None, seq_len: torch.Tensor, q_per_seq: int = 1,
              q_seq: torch.Tensor | None = None, block_table: torch.Tensor | None = None) -> Seqs:
    """csa2_seqs_t; with ``q_seq`` (int32 [num_q]) each query names its own sequence; with
    ``block_table`` (int32 [num_seqs, max_pages]) the cache is paged (128-row pages)."""
    assert seq_start is None or seq_start.dtype == torch.int64
    assert seq_len.dtype == torch.int32
    assert q_seq is None or q_seq.dtype == torch.int32
    assert block_table is None or (block_table.dtype == torch.int32 and block_table.dim() == 2)
    s = Seqs(int(seq_len.numel()), int(q_per_seq), _p(seq_start), _p(seq_len), _p(q_seq),
             _p(block_table), int(block_table.shape[1]) if block_table is not None else 0)
    s._keep = (seq_start, seq_len, q_seq, block_table)  # keep the tensors alive with the struct
    return s


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed byte workspace (its status word starts clear)."""
    return torch.zeros(max(int(nbytes), STATUS_BYTES), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------------------------
# entry points
# ------------------------------------------------------------------------------------
def quant_append_workspace() -> int:
    return int(lib().csa2_quant_append_workspace())


def quant_append(x, dst_row, kv_codes, kv_scales, ws, idx_k_in=None, idx_k=None, stream=None):
    assert x.dtype == torch.float32 and dst_row.dtype == torch.int64
    rows, D = x.shape
    d_I = idx_k.shape[1] if idx_k is not None else 0
    _check(lib().csa2_quant_append(_p(x), rows, D, _p(dst_row), _p(kv_codes), _p(kv_scales),
                                   kv_codes.shape[0], _u16(idx_k_in), _u16(idx_k), d_I, _p(ws),
                                   ws.numel(), _s(stream)), "csa2_quant_append")


def quant_append_e4m3k(x, dst_row, kv_codes, kv_scales, ws, idx_k_in, idx_k, stream=None):
    """csa2_quant_append with an E4M3 indexer-K cache (``idx_k`` uint8 [cap, d_I])."""
    assert x.dtype == torch.float32 and dst_row.dtype == torch.int64 and idx_k.dtype == torch.uint8
    rows, D = x.shape
    _check(lib().csa2_quant_append_e4m3k(_p(x), rows, D, _p(dst_row), _p(kv_codes), _p(kv_scales),
                                         kv_codes.shape[0], _u16(idx_k_in), _p(idx_k), idx_k.shape[1],
                                         _p(ws), ws.numel(), _s(stream)), "csa2_quant_append_e4m3k")


def compress_append(x, m, w_t, dst_row, kv_codes, kv_scales, ws, stream=None):
    """csa2_compress_append: x bf16 [n_entries * m, D_in] token rows, w_t bf16 [D, m * D_in];
    entry j goes to cache row dst_row[j]."""
    assert dst_row.dtype == torch.int64
    rows, D_in = x.shape
    D = w_t.shape[0]
    assert rows % m == 0 and w_t.shape[1] == m * D_in
    _check(lib().csa2_compress_append(_u16(x), rows // m, m, D_in, _u16(w_t), D, _p(dst_row),
                                      _p(kv_codes), _p(kv_scales), kv_codes.shape[0], _p(ws),
                                      ws.numel(), _s(stream)), "csa2_compress_append")


def e4m3_from_bf16(x, out=None, stream=None):
    """bf16 tensor -> E4M3 bytes (uint8, same shape), on the device."""
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    assert out.dtype == torch.uint8 and out.numel() == x.numel()
    _check(lib().csa2_e4m3_from_bf16(_u16(x), _p(out), x.numel(), _s(stream)), "csa2_e4m3_from_bf16")
    return out


def index_full_workspace(num_q, max_visible, topk, pool_blocks=0, block=8) -> int:
    return int(lib().csa2_index_full_workspace(num_q, max_visible, topk, pool_blocks, block))


def index_full(qI, w, idx_k, seqs: Seqs, topk, indices, ws, max_visible, q_visible=None,
               pool_blocks=0, block=8, pool=None, stream=None):
    """csa2_index_full; with uint8 (E4M3) ``qI`` and ``idx_k``, csa2_index_full_e4m3."""
    num_q, H_I, d_I = qI.shape
    assert w.dtype == torch.float32 and indices.dtype == torch.int32
    assert pool is None or pool.dtype == torch.int32
    if qI.dtype == torch.uint8:
        assert idx_k.dtype == torch.uint8
        _check(lib().csa2_index_full_e4m3(_p(qI), _p(w), num_q, H_I, d_I, _p(idx_k), idx_k.shape[0],
                                          seqs, _p(q_visible), int(max_visible), topk, _p(indices),
                                          pool_blocks, block, _p(pool), _p(ws), ws.numel(),
                                          _s(stream)), "csa2_index_full_e4m3")
        return
    _check(lib().csa2_index_full(_u16(qI), _p(w), num_q, H_I, d_I, _u16(idx_k), idx_k.shape[0],
                                 seqs, _p(q_visible), int(max_visible), topk, _p(indices),
                                 pool_blocks, block, _p(pool), _p(ws), ws.numel(), _s(stream)),
           "csa2_index_full")


NOALLOC_SCRATCH_BYTES = 8 << 20


def index_full_noalloc(qI, w, idx_k, seqs: Seqs, topk, indices, max_visible, q_visible=None,
                       pool_blocks=0, block=8, pool=None, stream=None):
    """csa2_index_full with the library's own fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory); see include/csa2.h."""
    num_q, H_I, d_I = qI.shape
    assert w.dtype == torch.float32 and indices.dtype == torch.int32
    assert pool is None or pool.dtype == torch.int32
    _check(lib().csa2_index_full_noalloc(_u16(qI), _p(w), num_q, H_I, d_I, _u16(idx_k),
                                         idx_k.shape[0], seqs, _p(q_visible), int(max_visible),
                                         topk, _p(indices), pool_blocks, block, _p(pool),
                                         _s(stream)), "csa2_index_full_noalloc")


def index_full_noalloc_status(stream=None) -> int:
    """Wait for the stream; return the status word of the latest index_full_noalloc call on
    the current device (0 = OK)."""
    return int(lib().csa2_index_full_noalloc_status(_s(stream)))


def index_pool_workspace(num_q, pool_blocks, block, topk) -> int:
    return int(lib().csa2_index_pool_workspace(num_q, pool_blocks, block, topk))


def index_pool(qI, w, idx_k, seqs: Seqs, pool, pool_blocks, block, topk, indices, ws,
               q_visible=None, stream=None):
    """csa2_index_pool; with uint8 (E4M3) ``qI`` and ``idx_k``, csa2_index_pool_e4m3."""
    num_q, H_I, d_I = qI.shape
    assert w.dtype == torch.float32 and indices.dtype == torch.int32 and pool.dtype == torch.int32
    if qI.dtype == torch.uint8:
        assert idx_k.dtype == torch.uint8
        _check(lib().csa2_index_pool_e4m3(_p(qI), _p(w), num_q, H_I, d_I, _p(idx_k), idx_k.shape[0],
                                          seqs, _p(q_visible), _p(pool), pool_blocks, block, topk,
                                          _p(indices), _p(ws), ws.numel(), _s(stream)),
               "csa2_index_pool_e4m3")
        return
    _check(lib().csa2_index_pool(_u16(qI), _p(w), num_q, H_I, d_I, _u16(idx_k), idx_k.shape[0],
                                 seqs, _p(q_visible), _p(pool), pool_blocks, block, topk,
                                 _p(indices), _p(ws), ws.numel(), _s(stream)),
           "csa2_index_pool")


def sparse_attn_workspace(num_q, H, D, topk, window) -> int:
    return int(lib().csa2_sparse_attn_workspace(num_q, H, D, topk, window))


def sparse_attn_stash_bytes(num_q, D, topk) -> int:
    return int(lib().csa2_sparse_attn_stash_bytes(num_q, D, topk))


def sparse_attn(q, kv_codes, kv_scales, seqs: Seqs, indices, swa_kv, swa_start, q_pos, window,
                softmax_scale, out, ws, lse=None, mode=MODE_FULL, stash=None, stream=None,
                swa_ring=0):
    num_q, H, D = q.shape
    topk = indices.shape[1] if indices is not None else 0
    assert out.dtype == torch.float32 and q_pos.dtype == torch.int64
    _check(lib().csa2_sparse_attn(_u16(q), num_q, H, D, _p(kv_codes), _p(kv_scales),
                                  kv_codes.shape[0], seqs, _p(indices), topk, _u16(swa_kv),
                                  swa_kv.shape[0] if swa_kv is not None else 0, _p(swa_start),
                                  _p(q_pos), window, int(swa_ring), float(softmax_scale), _p(out), _p(lse),
                                  int(mode), _p(stash), stash.numel() if stash is not None else 0,
                                  _p(ws), ws.numel(), _s(stream)), "csa2_sparse_attn")


def layer_step(mode, kv_codes, kv_scales, seqs: Seqs, topk, indices, attn: dict,
               indexer: dict | None = None, stream=None):
    """csa2_layer_step: one layer of the schedule.  ``indexer`` (FULL / REINDEX) holds qI, w,
    idx_k, ws and optionally q_visible, max_visible, pool_blocks, block, pool; ``attn`` holds
    q, swa_kv, swa_start, q_pos, window, softmax_scale, out, ws and optionally lse, stash."""
    q = attn["q"]
    num_q, H, D = q.shape
    at = Attention(_u16(q), H, D, _u16(attn["swa_kv"]), attn["swa_kv"].shape[0], _p(attn["swa_start"]),
                   _p(attn["q_pos"]), int(attn["window"]), int(attn.get("swa_ring", 0)),
                   float(attn["softmax_scale"]),
                   _p(attn["out"]), _p(attn.get("lse")), _p(attn.get("stash")),
                   attn["stash"].numel() if attn.get("stash") is not None else 0,
                   _p(attn["ws"]), attn["ws"].numel())
    ix = None
    if indexer is not None:
        qI = indexer["qI"]
        e4m3 = qI.dtype == torch.uint8
        assert e4m3 == (indexer["idx_k"].dtype == torch.uint8)
        qp, kp = (_p(qI), _p(indexer["idx_k"])) if e4m3 else (_u16(qI), _u16(indexer["idx_k"]))
        ix = Indexer(qp, _p(indexer["w"]), qI.shape[1], qI.shape[2], kp,
                     _p(indexer.get("q_visible")), int(indexer.get("max_visible", 0)),
                     int(indexer.get("pool_blocks", 0)), int(indexer.get("block", 8)),
                     _p(indexer.get("pool")), _p(indexer["ws"]), indexer["ws"].numel(), int(e4m3))
    _check(lib().csa2_layer_step(int(mode), num_q, _p(kv_codes), _p(kv_scales), kv_codes.shape[0],
                                 seqs, topk, _p(indices), ctypes.byref(ix) if ix is not None else None,
                                 ctypes.byref(at), _s(stream)), "csa2_layer_step")


def cache_rows(seqs: Seqs, seq, pos, rows=None, stream=None):
    """Cache rows (int64) of (seq[i], pos[i]) under the layout of ``seqs``; -1 if missing."""
    assert seq.dtype == torch.int32 and pos.dtype == torch.int32 and seq.numel() == pos.numel()
    if rows is None:
        rows = torch.empty(seq.numel(), dtype=torch.int64, device=seq.device)
    _check(lib().csa2_cache_rows(seqs, _p(seq), _p(pos), seq.numel(), _p(rows), _s(stream)),
           "csa2_cache_rows")
    return rows


def gather_rows(table, rows, dst=None, stream=None):
    """dst[i] = table[rows[i]] (a zero row for rows outside the table)."""
    row_bytes = table.shape[1] * table.element_size()
    if dst is None:
        dst = torch.empty((rows.numel(),) + tuple(table.shape[1:]), dtype=table.dtype, device=table.device)
    _check(lib().csa2_gather_rows(_p(table), table.shape[0], row_bytes, _p(rows), rows.numel(),
                                  _p(dst), _s(stream)), "csa2_gather_rows")
    return dst


def scatter_rows(src, rows, table, stream=None):
    """table[rows[i]] = src[i] (rows outside the table are skipped)."""
    row_bytes = table.shape[1] * table.element_size()
    _check(lib().csa2_scatter_rows(_p(src), row_bytes, _p(rows), rows.numel(), _p(table),
                                   table.shape[0], _s(stream)), "csa2_scatter_rows")


def status_reset(ws, stream=None) -> None:
    _check(lib().csa2_status_reset(_p(ws), _s(stream)), "csa2_status_reset")


def status_fetch(ws, stream=None) -> int:
    """Wait for the stream; return the status word recorded in ``ws`` (0 = OK)."""
    return int(lib().csa2_status_fetch(_p(ws), _s(stream)))


def set_wait_limit_ns(ns: int) -> int:
    """Bound of the kernels' waits for later launches (0 = the default 2 s); returns the
    previous bound."""
    return int(lib().csa2_set_wait_limit_ns(int(ns)))


def device_sms() -> int:
    return int(lib().csa2_device_sms())
