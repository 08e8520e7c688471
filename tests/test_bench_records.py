"""bench.py's recorded-traffic lookup: the source hash that keys a committed ncu
capture ignores comments and blank lines but not code, and a record is used only
for the workload and hash it names."""
import os

import bench


def test_code_only_strips_comments_keeps_code_and_strings():
    a = 'int x = 1;  // one\n\n// a whole-line comment\nconst char *s = "a // b";\n'
    b = 'int   x = 1;\nconst char *s = "a // b";   // other words\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert 'a // b' in bench._code_only(a)
    assert bench._code_only("int x = 1;") != bench._code_only("int x = 2;")


def test_record_needs_matching_workload_and_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "paged_kv_cache_396_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("int f() { return 1; }  // v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(["k.cu"])
    (tmp_path / "profiles" / "t.txt").write_text(
        f"# header\nworkload=w1 sources={h} bytes_per_launch=123\n")
    assert bench.recorded_traffic("w1", "t.txt", ["k.cu"]) == 123.0
    assert bench.recorded_traffic("w2", "t.txt", ["k.cu"]) is None
    (csrc / "k.cu").write_text("int f() { return 1; }  // comment edited\n")
    assert bench.recorded_traffic("w1", "t.txt", ["k.cu"]) == 123.0
    (csrc / "k.cu").write_text("int f() { return 2; }\n")
    assert bench.recorded_traffic("w1", "t.txt", ["k.cu"]) is None
