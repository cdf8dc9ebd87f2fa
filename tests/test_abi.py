"""The C-ABI library loads and exports every entry point of include/csa2.h; host-side
argument checks return their status codes without touching a GPU."""
import ctypes
import os
import re

import pytest

from fp4_kv_cache_03_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_lib.build()
    from fp4_kv_cache_03_b200 import csa2
    return csa2.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "csa2.h"), encoding="utf-8").read()
    return sorted(set(re.findall(r"^CSA2_API[^;(]*?\b(csa2_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    from fp4_kv_cache_03_b200 import csa2
    assert csa2.status_string(0) == "ok"
    assert "timed out" in csa2.status_string(csa2.ERR_TIMEOUT)


def test_workspace_sizes(L):
    from fp4_kv_cache_03_b200 import csa2
    assert csa2.quant_append_workspace() == 256
    a = csa2.index_full_workspace(1, 131072, 512, 0, 8)
    b = csa2.index_full_workspace(1, 131072, 512, 2048, 8)
    assert a >= 256 + 131072 * 4 and b > a
    assert csa2.index_pool_workspace(1, 2048, 8, 512) >= 256 + 16384 * 4
    assert csa2.sparse_attn_workspace(1, 64, 512, 512, 128) >= 256


def test_attention_split_policy_through_workspace_sizes(L):
    """The attention workspace holds the key splits' partials ([q][split][H][D] fp32 and
    (m, l) [q][split][H]), so its size shows the host's tile and split choice (148 SMs
    without a GPU).  A decode query: 64-key tiles, 8 + 2 = 10 splits; 64 queries: 128-key
    tiles, 2 splits (SMs per query); 4,096 queries: one split, no partials."""
    from fp4_kv_cache_03_b200 import csa2
    sms = L.csa2_device_sms()
    if sms > 0 and sms != 148:
        pytest.skip(f"the expectations below are for 148 SMs, this device has {sms}")
    a256 = lambda x: (x + 255) // 256 * 256
    def expect(nq, ns, H=64, D=512):
        return 256 + a256(nq * ns * H * D * 4) + a256(nq * ns * H * 2 * 4) if ns > 1 else 256
    assert csa2.sparse_attn_workspace(1, 64, 512, 512, 128) == expect(1, 10)
    assert csa2.sparse_attn_workspace(64, 64, 512, 512, 128) == expect(64, 2)
    assert csa2.sparse_attn_workspace(4096, 64, 512, 512, 128) == expect(4096, 1)


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: the checks below return first


def test_host_checks_quant_append(L):
    from fp4_kv_cache_03_b200 import csa2
    st = L.csa2_quant_append(FAKE, 4, 24, FAKE, FAKE, FAKE, 100, None, None, 0, FAKE, 256, None)
    assert st == csa2.ERR_INVALID_ARG                        # D not a multiple of 32
    st = L.csa2_quant_append(FAKE, 4, 64, FAKE, FAKE, FAKE, 100, None, None, 0, FAKE, 16, None)
    assert st == csa2.ERR_CAPACITY                           # workspace too small
    st = L.csa2_quant_append(FAKE, 0, 64, FAKE, FAKE, FAKE, 100, None, None, 0, FAKE, 256, None)
    assert st == csa2.OK                                     # nothing to do


def _seqs(n=1, qps=1):
    from fp4_kv_cache_03_b200 import csa2
    return csa2.Seqs(n, qps, FAKE, FAKE)


def test_host_checks_index(L):
    from fp4_kv_cache_03_b200 import csa2
    args = lambda H_I=4, d_I=64, topk=64, ws=1 << 30, pool_blocks=0, block=8: (
        FAKE, FAKE, 1, H_I, d_I, FAKE, 4096, _seqs(), None, 4096, topk, FAKE, pool_blocks, block,
        FAKE, ctypes.c_void_p(0x100000), ws, None)
    assert L.csa2_index_full(*args(H_I=0)) == csa2.ERR_UNSUPPORTED
    assert L.csa2_index_full(*args(H_I=33)) == csa2.ERR_UNSUPPORTED
    assert L.csa2_index_full(*args(d_I=96)) == csa2.ERR_UNSUPPORTED
    assert L.csa2_index_full(*args(topk=0)) == csa2.ERR_UNSUPPORTED
    assert L.csa2_index_full(*args(pool_blocks=16, block=3)) == csa2.ERR_UNSUPPORTED
    assert L.csa2_index_full(*args(ws=1024)) == csa2.ERR_CAPACITY
    a = list(args())
    a[7] = _seqs(2, 1)                                       # 2 sequences x 1 != num_q
    assert L.csa2_index_full(*a) == csa2.ERR_INVALID_ARG
    pa = (FAKE, FAKE, 1, 4, 64, FAKE, 4096, _seqs(), None, FAKE, 16, 4, 64, FAKE,
          ctypes.c_void_p(0x100000), 1 << 30, None)
    assert L.csa2_index_pool(*pa) == csa2.ERR_UNSUPPORTED    # block must be 8


def test_host_checks_attention(L):
    from fp4_kv_cache_03_b200 import csa2
    def call(H=16, D=128, topk=64, window=128, ws=1 << 30, mode=0, stash=None, stash_bytes=0, ring=0):
        return L.csa2_sparse_attn(FAKE, 1, H, D, FAKE, FAKE, 100, _seqs(), FAKE, topk, FAKE, 100,
                                  FAKE, FAKE, window, ring, 0.1, FAKE, None, mode, stash, stash_bytes,
                                  ctypes.c_void_p(0x100000), ws, None)
    assert call(H=65) == csa2.ERR_UNSUPPORTED
    assert call(H=0) == csa2.ERR_UNSUPPORTED
    assert call(D=96) == csa2.ERR_UNSUPPORTED
    assert call(D=64) == csa2.ERR_UNSUPPORTED
    assert call(topk=4096) == csa2.ERR_INVALID_ARG
    assert call(ws=300) == csa2.ERR_CAPACITY
    assert call(mode=7) == csa2.ERR_INVALID_ARG
    assert call(ring=100) == csa2.ERR_INVALID_ARG            # a ring is whole 128-row tiles
    assert call(ring=128, window=200) == csa2.ERR_INVALID_ARG  # ... at least the window
    assert call(stash=ctypes.c_void_p(0x200000), stash_bytes=16) == csa2.ERR_CAPACITY
    assert call(stash=ctypes.c_void_p(0x200008), stash_bytes=1 << 30) == csa2.ERR_INVALID_ARG
    # 4 tiles of 128 rows: codes (256 B), scales (32 B) and a validity byte per row
    assert L.csa2_sparse_attn_stash_bytes(1, 512, 512) == 4 * 128 * (256 + 32 + 1)
    # a per-query sequence map lifts the num_seqs x q_per_seq = num_q rule
    bad = csa2.Seqs(2, 1, FAKE, FAKE)                       # 2 x 1 != 1 query
    mapped = csa2.Seqs(2, 0, FAKE, FAKE, FAKE)             # q_seq given: q_per_seq unused
    args = lambda seqs: (FAKE, 1, 16, 128, FAKE, FAKE, 100, seqs, FAKE, 64, FAKE, 100, FAKE, FAKE,
                         128, 0, 0.1, FAKE, None, 0, None, 0, ctypes.c_void_p(0x100000), 300, None)
    assert L.csa2_sparse_attn(*args(bad)) == csa2.ERR_INVALID_ARG
    assert L.csa2_sparse_attn(*args(mapped)) == csa2.ERR_CAPACITY   # passes the map check


def test_device_query_without_gpu_is_harmless(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.csa2_device_sms() == 0


def test_host_checks_layer_step(L):
    """csa2_layer_step rejects a bad mode or missing argument blocks, and passes the
    first call's host-side status through (nothing is launched on these paths)."""
    import ctypes as C
    from fp4_kv_cache_03_b200 import csa2
    seqs = csa2.Seqs(1, 1, FAKE, FAKE)
    at = csa2.Attention(FAKE, 16, 128, FAKE, 8, FAKE, FAKE, 4, 0, 0.1, FAKE, None, None, 0, FAKE, 16)
    ix = csa2.Indexer(FAKE, FAKE, 4, 64, FAKE, None, 4096, 0, 8, None, FAKE, 1 << 30)

    def call(mode, ix_, at_, topk=64):
        return L.csa2_layer_step(mode, 1, FAKE, FAKE, 100, seqs, topk, FAKE,
                                 C.byref(ix_) if ix_ is not None else None,
                                 C.byref(at_) if at_ is not None else None, None)
    assert call(7, ix, at) == csa2.ERR_INVALID_ARG                    # no such mode
    assert call(csa2.MODE_REUSE, None, None) == csa2.ERR_INVALID_ARG   # attention args needed
    assert call(csa2.MODE_FULL, None, at) == csa2.ERR_INVALID_ARG      # Full needs its indexer
    assert call(csa2.MODE_REINDEX, None, at) == csa2.ERR_INVALID_ARG
    # Reuse: straight to attention, whose workspace (16 B) is below the status word
    assert call(csa2.MODE_REUSE, None, at) == csa2.ERR_CAPACITY
    # Full: the index call's own check comes first (33 indexer heads are unsupported)
    bad = csa2.Indexer(FAKE, FAKE, 33, 64, FAKE, None, 4096, 0, 8, None, FAKE, 1 << 30)
    assert call(csa2.MODE_FULL, bad, at) == csa2.ERR_UNSUPPORTED


def test_binding_matches_header():
    """Every entry point of include/csa2.h is bound in csa2.py with as many argument types
    as the C declaration has parameters (guards the ABI against drift)."""
    from fp4_kv_cache_03_b200 import csa2
    text = open(os.path.join(ROOT, "include", "csa2.h"), encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)          # drop comments
    decls = re.findall(r"CSA2_API[^;(]*?\b(csa2_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S)
    assert len(decls) >= 12
    for name, params in decls:
        assert name in csa2._SIGS, name
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        assert len(csa2._SIGS[name][1]) == n, (name, n, len(csa2._SIGS[name][1]))


def test_binding_rejects_wrong_dtypes_before_any_call(L):
    """The binding checks tensor dtypes before it calls into the library (a wrong dtype would
    otherwise reach a kernel as a mis-sized buffer); CPU tensors suffice: nothing runs."""
    import torch
    from fp4_kv_cache_03_b200 import csa2
    qI = torch.zeros(1, 16, 128, dtype=torch.bfloat16)
    idx_k = torch.zeros(256, 128, dtype=torch.bfloat16)
    seqs = csa2.Seqs(1, 1, FAKE, FAKE)
    good_w = torch.zeros(1, 16, dtype=torch.float32)
    good_i = torch.zeros(1, 64, dtype=torch.int32)
    for w, ind, pool in [(good_w.double(), good_i, None), (good_w, good_i.long(), None),
                         (good_w, good_i, torch.zeros(1, 8, dtype=torch.int64))]:
        with pytest.raises(AssertionError):
            csa2.index_full_noalloc(qI, w, idx_k, seqs, 64, ind, 256, pool_blocks=8 if pool is not None else 0,
                                    pool=pool)
