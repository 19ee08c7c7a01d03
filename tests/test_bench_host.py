"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
ties the committed DRAM-traffic record to the code it was measured on."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_code_hash_ignores_comments_and_blank_lines():
    b = _bench()
    src = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    assert b.code_sha1(src) == b.code_sha1("// header\n\nint f(int x) {\n  return x + 1;\n}\n")
    assert b.code_sha1(src) == b.code_sha1("/* block\n comment */int f(int x) {\n  return x + 1;\n}\n")


def test_code_hash_sees_code_changes():
    b = _bench()
    assert b.code_sha1("int f(int x) { return x + 1; }") != b.code_sha1("int f(int x) { return x + 2; }")


def test_traffic_record_is_dropped_when_the_code_differs(tmp_path, monkeypatch):
    b = _bench()
    ent = {"source_file": "k.cuh", "source_code_sha1": b.code_sha1("int a;"), "bytes_per_entry": 2.0}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text('{"k": %s}' % __import__("json").dumps(ent))
    (tmp_path / "k.cuh").write_text("int a;  // the measured code\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.load_traffic("k", 10) == 20.0
    (tmp_path / "k.cuh").write_text("int b;\n")
    assert b.load_traffic("k", 10) is None
