"""Host logic of bench.py that needs no GPU: the source hash that decides
whether a committed DRAM-traffic capture still describes the kernels."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_are_removed_and_literals_kept():
    src = 'int a = 1; // note\n/* block\n */ const char* s = "x // y /* z */"; char c = \'"\'; int d;'
    out = bench.strip_c_comments(src)
    assert "note" not in out and "block" not in out
    assert '"x // y /* z */"' in out and "'\"'" in out and "int d;" in out


def test_comment_edits_keep_the_hash_and_code_edits_change_it():
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "int f(int x) {\n  return x + 1;  // increment\n}\n"
    c = "int f(int x) {\n  return x + 2;  // add one\n}\n"
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)
    assert bench.strip_c_comments(a) != bench.strip_c_comments(c)


def test_comment_and_layout_edits_keep_the_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_query_attention_sqa_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("// one line\nint f(int x) { return x + 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha256()
    (csrc / "k.cuh").write_text("// a comment\n// of two lines\nint f(int x) {\n  return x + 1;\n}\n")
    assert bench.kernel_source_sha256() == h0
    (csrc / "k.cuh").write_text("int f(int x) { return x - 1; }\n")
    assert bench.kernel_source_sha256() != h0


def test_traffic_table_names_a_capture_command_per_entry():
    import json

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for e in table["entries"]:
        assert e["command"].startswith("ncu ") and "--clock-control none" in e["command"]
        assert e["dram_bytes_per_launch"] > 0 and len(e["source_sha256"]) == 64
