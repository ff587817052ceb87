"""Host-side helpers of bench.py on CPU: the kernel-code hash that keys the
recorded ncu traffic ignores comments and blank lines but no code, and the
recorded traffic is only reported while that hash matches."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = 'a = "//x";  // c\n/* b\n c */ int k = \'/\';\n\n  \nq("/*", 1); /**/ r;\n'
    assert bench.strip_comments(src) == 'a = "//x";\n int k = \'/\';\nq("/*", 1);  r;'
    assert bench.strip_comments('s = "a\\"//b"; // t\n') == 's = "a\\"//b";'
    assert bench.strip_comments("x; /* never closed") == "x;"


def test_code_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "mla_decode_attention_13_b200" / "csrc"
    csrc.mkdir(parents=True)
    files = {name: f"int f_{i}() {{ return {i}; }}\n" for i, name in enumerate(bench.KERNEL_SOURCES)}
    for name, text in files.items():
        (csrc / name).write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha()
    first = bench.KERNEL_SOURCES[0]
    (csrc / first).write_text("// a comment\n" + files[first] + "\n/* another */\n")
    assert bench.kernel_source_sha() == h0
    (csrc / first).write_text(files[first].replace("return 0", "return 1"))
    assert bench.kernel_source_sha() != h0


def test_recorded_traffic_only_for_the_recorded_code(tmp_path, monkeypatch):
    csrc = tmp_path / "mla_decode_attention_13_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        (csrc / name).write_text("int x;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    rec.write_text(json.dumps({"source_sha": bench.kernel_source_sha(), "workloads": {"w": 1234}}))
    assert bench.committed_traffic("w") == 1234
    assert bench.committed_traffic("other") is None
    rec.write_text(json.dumps({"source_sha": "0" * 16, "workloads": {"w": 1234}}))
    assert bench.committed_traffic("w") is None
