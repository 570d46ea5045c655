"""bench.py's `traffic` key: DRAM bytes per launch come from a committed ncu
capture only while the kernel sources it was taken on are unchanged (a sha256
over them); otherwise the key is null rather than a stale figure."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path, sources, sha=None, kernels=None):
    csrc = tmp_path / "mixture_experts_layer_22_b200" / "csrc"
    csrc.mkdir(parents=True)
    h = hashlib.sha256()
    for name, text in sources.items():
        (csrc / name).write_bytes(text)
        h.update(text)
    (tmp_path / "profiles").mkdir()
    cap = {"sources": list(sources), "source_sha256": sha or h.hexdigest(),
           "kernels": kernels or {"wl T=8 gemm1": 1234}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"captures": [cap]}))
    return csrc


def test_fresh_capture_is_reported(tmp_path, monkeypatch):
    _tree(tmp_path, {"a.cu": b"kernel a", "b.cuh": b"header"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("wl T=8 gemm1") == 1234


def test_changed_source_makes_the_capture_stale(tmp_path, monkeypatch):
    csrc = _tree(tmp_path, {"a.cu": b"kernel a", "b.cuh": b"header"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "b.cuh").write_bytes(b"header, edited")
    assert bench.captured_traffic("wl T=8 gemm1") is None


def test_source_order_is_part_of_the_hash(tmp_path, monkeypatch):
    h = hashlib.sha256()
    h.update(b"header")
    h.update(b"kernel a")                       # the reverse of the listed order
    _tree(tmp_path, {"a.cu": b"kernel a", "b.cuh": b"header"}, sha=h.hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("wl T=8 gemm1") is None


def test_unknown_key_missing_file_or_source(tmp_path, monkeypatch):
    csrc = _tree(tmp_path, {"a.cu": b"kernel a"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("wl T=16 gemm1") is None
    os.remove(csrc / "a.cu")
    assert bench.captured_traffic("wl T=8 gemm1") is None
    os.remove(tmp_path / "profiles" / "traffic.json")
    assert bench.captured_traffic("wl T=8 gemm1") is None


def test_committed_captures_name_existing_sources():
    """Every capture in the committed file lists kernel sources that exist."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert t["captures"]
    for cap in t["captures"]:
        for name in cap["sources"]:
            assert os.path.exists(os.path.join(ROOT, "mixture_experts_layer_22_b200", "csrc", name)), name
        assert all(isinstance(v, int) and v > 0 for v in cap["kernels"].values())
