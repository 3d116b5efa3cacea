"""Host-side logic of bench.py that the roofline entry depends on (CPU only).

The line's `traffic` is the DRAM bytes of one decode launch, taken from a
committed ncu summary only while that summary was captured on the current
kernel source. The source is identified by a hash of the decode sources with
comments and whitespace removed, so an edited comment keeps the recorded
counters, and any change to the code drops them.
"""

import os

import bench


def _write_sources(root, body):
    for rel in bench.DECODE_SOURCES:
        path = os.path.join(root, rel)
        os.makedirs(os.path.dirname(path), exist_ok=True)
        with open(path, "w", encoding="utf-8") as f:
            f.write(body)


def _hash_of(tmp_path, monkeypatch, body):
    _write_sources(str(tmp_path), body)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench.decode_source_hash()


def test_hash_ignores_comments_and_whitespace(tmp_path, monkeypatch):
    code = "int f(int x) {\n  return x + 1;\n}\n"
    h0 = _hash_of(tmp_path, monkeypatch, code)
    commented = ("// header line\n/* a block\n   comment */\nint f(int x)   {\n"
                 "  return x + 1;  // trailing\n}\n\n")
    assert _hash_of(tmp_path, monkeypatch, commented) == h0
    assert _hash_of(tmp_path, monkeypatch, code.replace("+ 1", "+ 2")) != h0
    assert len(h0) == 16 and int(h0, 16) >= 0


def test_traffic_is_read_only_for_the_current_source(tmp_path, monkeypatch):
    h = _hash_of(tmp_path, monkeypatch, "int g() { return 3; }\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "decode_tc_w.md").write_text(
        f"# summary\n\nsource_sha256: `{h}`\n\ntraffic_bytes_per_launch: `123456`\n")
    assert bench.recorded_traffic("w") == 123456
    (prof / "decode_tc_w.md").write_text(
        "source_sha256: `0000000000000000`\ntraffic_bytes_per_launch: `123456`\n")
    assert bench.recorded_traffic("w") is None      # taken on another kernel
    (prof / "decode_tc_w.md").write_text(f"source_sha256: `{h}`\n")
    assert bench.recorded_traffic("w") is None      # no figure recorded
    assert bench.recorded_traffic("missing") is None


def test_committed_headline_summary_has_a_traffic_figure():
    """The headline summary carries both keys the bench reads; its figure is
    a plausible per-launch byte count (the call moves ~0.92 GB)."""
    path = os.path.join(bench.ROOT, "profiles", "decode_tc_llama8b_gqa_b256.md")
    keys = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            for k in ("source_sha256", "traffic_bytes_per_launch"):
                if line.strip().startswith(k + ":"):
                    keys[k] = line.split(":", 1)[1].strip().strip("`")
    assert len(keys["source_sha256"]) == 16
    assert 0.9e9 < int(keys["traffic_bytes_per_launch"]) < 1.0e9
