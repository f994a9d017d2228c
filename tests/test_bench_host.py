"""Host logic of bench.py on CPU: the roofline's `traffic` comes from a
committed ncu summary only while that summary's kernel sources are the ones
being measured (the recorded source hash equals the current one), else it is
null; and the source hash follows the bytes of the files it names."""
import json
import os

import bench


def _profile(tmp_path, name, payload):
    d = tmp_path / "profiles"
    d.mkdir(exist_ok=True)
    (d / name).write_text(json.dumps(payload))


def test_traffic_only_from_a_current_capture(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _profile(tmp_path, "k.json", {"kernel_source_hash": "abc", "dram_bytes_per_launch": 1000.0, "x": 7})
    assert bench.traffic_from_profile("k.json", "abc") == 1000.0
    assert bench.traffic_from_profile("k.json", "abc", units_scale=2.5) == 2500.0
    assert bench.traffic_from_profile("k.json", "abd") is None      # the kernel changed since the capture
    assert bench.traffic_from_profile("missing.json", "abc") is None
    assert bench.profile_field("k.json", "abc", "x") == 7
    assert bench.profile_field("k.json", "abc", "absent") is None


def test_kernel_hash_follows_the_source_bytes(tmp_path, monkeypatch):
    src = tmp_path / "local_linear_attention_streamed_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "a.cu").write_bytes(b"kernel one")
    (src / "b.cuh").write_bytes(b"header")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_hash("a.cu", "b.cuh")
    assert h1 == bench.kernel_hash("a.cu", "b.cuh") and len(h1) == 16
    (src / "a.cu").write_bytes(b"kernel one ")                       # one byte more
    assert bench.kernel_hash("a.cu", "b.cuh") != h1
    (src / "a.cu").write_bytes(b"kernel one")
    assert bench.kernel_hash("b.cuh", "a.cu") != h1                  # the order of the files counts


def test_committed_captures_name_their_sources_and_command():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pdir = os.path.join(root, "profiles")
    found = 0
    for name in sorted(os.listdir(pdir)):
        if not name.endswith(".json"):
            continue
        with open(os.path.join(pdir, name)) as f:
            p = json.load(f)
        found += 1
        assert len(p["kernel_source_hash"]) == 16, name
        assert "--clock-control none" in p["command"], name
        assert p["dram_bytes_per_launch"] > 0, name
    assert found >= 6
