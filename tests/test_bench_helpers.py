"""Host-side helpers of bench.py (CPU only): the attention traffic taken from the committed ncu
capture is reported only while the kernel's sources still hash to the captured value, and
the step's inputs and outputs are re-homed into one tensor per kind without changing them."""
import hashlib
import json
import os
import sys
from dataclasses import dataclass

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _tree(tmp_path, sources, workload="decoder_step_128k", sha=None, nbytes=4096):
    (tmp_path / "profiles").mkdir()
    h = hashlib.sha256()
    for rel, text in sources.items():
        f = tmp_path / rel
        f.parent.mkdir(parents=True, exist_ok=True)
        f.write_bytes(text)
        h.update(text)
    rec = {"workload": workload, "dram_bytes_per_launch": nbytes,
           "source_files": list(sources), "source_sha256": sha or h.hexdigest()}
    (tmp_path / "profiles" / "attn_tc_traffic.json").write_text(json.dumps(rec))


def test_traffic_reported_while_the_sources_match(tmp_path):
    _tree(tmp_path, {"k/a.cu": b"kernel a", "k/b.cuh": b"header b"}, nbytes=1234)
    assert bench.captured_attn_traffic("decoder_step_128k", str(tmp_path)) == 1234
    assert bench.captured_attn_traffic("ragged_decode", str(tmp_path)) is None


def test_traffic_dropped_once_a_source_changes(tmp_path):
    _tree(tmp_path, {"k/a.cu": b"kernel a"})
    (tmp_path / "k" / "a.cu").write_bytes(b"kernel a, edited")
    assert bench.captured_attn_traffic("decoder_step_128k", str(tmp_path)) is None


def test_traffic_missing_record_or_source_is_none(tmp_path):
    assert bench.captured_attn_traffic("decoder_step_128k", str(tmp_path)) is None
    _tree(tmp_path, {"k/a.cu": b"x"})
    (tmp_path / "k" / "a.cu").unlink()
    assert bench.captured_attn_traffic("decoder_step_128k", str(tmp_path)) is None


def test_committed_record_matches_the_committed_sources():
    # the committed capture belongs to the committed kernel (else the bench reports null)
    assert bench.captured_attn_traffic("decoder_step_128k") is not None


@dataclass
class _Layer:
    q: torch.Tensor
    qI: torch.Tensor | None
    w: torch.Tensor | None
    swa: torch.Tensor


class _DW:
    pass


def test_coalesce_io_keeps_values_and_shares_storage():
    g = torch.Generator().manual_seed(0)
    modes = ["full", "reuse", "reindex", "reuse"]
    layers = [_Layer(torch.randn(2, 4, 8, generator=g),
                     torch.randn(2, 3, 8, generator=g) if m != "reuse" else None,
                     torch.rand(2, 3, generator=g) if m != "reuse" else None,
                     torch.randn(5, 8, generator=g)) for m in modes]
    dw = _DW()
    dw.layers = layers
    dw.out = [torch.randn(2, 4, 8, generator=g) for _ in modes]
    before = [(L.q.clone(), None if L.qI is None else L.qI.clone(), None if L.w is None else L.w.clone(),
               L.swa.clone()) for L in layers]
    out_before = [o.clone() for o in dw.out]
    io = bench.coalesce_io(dw)
    assert io["q"].shape == (4, 2, 4, 8) and io["qI"].shape == (2, 2, 3, 8) and io["swa"].shape == (4, 5, 8)
    for i, (L, b) in enumerate(zip(dw.layers, before)):
        assert torch.equal(L.q, b[0]) and torch.equal(L.swa, b[3])
        assert L.q.data_ptr() == io["q"][i].data_ptr() and L.swa.data_ptr() == io["swa"][i].data_ptr()
        if L.qI is not None:
            assert torch.equal(L.qI, b[1]) and torch.equal(L.w, b[2])
    for i, o in enumerate(dw.out):
        assert torch.equal(o, out_before[i]) and o.data_ptr() == io["out"][i].data_ptr()
    # a write through the step's tensor reaches the layer's view (one transfer serves all)
    io["q"][2].fill_(7.0)
    assert torch.all(dw.layers[2].q == 7.0)
    new_rows = io["swa"][:, -1]
    new_rows.copy_(torch.zeros_like(new_rows))
    assert all(torch.all(L.swa[-1] == 0) for L in dw.layers)
