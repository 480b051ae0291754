"""Host logic of bench.py that needs no GPU: the source hash that ties recorded
ncu traffic to a build covers the code only, and the traffic table is read
back only for the matching hash."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_blank_lines():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */\n'
           '\n'
           'const char *s = "// not a comment /* nor this */";\n'
           "char c = '/';  /* inline */ int b = 2;\n")
    out = bench._code_only(src)
    assert out.splitlines() == ['int a = 1;',
                                'const char *s = "// not a comment /* nor this */";',
                                "char c = '/';   int b = 2;"]


def test_code_only_keeps_escaped_quotes_in_literals():
    src = 'const char *s = "a \\" // b";  // c\n'
    assert bench._code_only(src) == 'const char *s = "a \\" // b";'


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "gated_delta_rule_99_b200" / "csrc"
    inc = tmp_path / "include"
    csrc.mkdir(parents=True)
    inc.mkdir()
    (inc / "x.h").write_text("int f(void);\n")
    (csrc / "k.cu").write_text("// kernel\n__global__ void k() { int x = 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.csrc_hash()
    (csrc / "k.cu").write_text("// the kernel, reworded\n\n__global__ void k() { int x = 1; }  // x\n")
    assert bench.csrc_hash() == h0
    (csrc / "k.cu").write_text("__global__ void k() { int x = 2; }\n")
    assert bench.csrc_hash() != h0


def test_recorded_traffic_needs_the_matching_hash(tmp_path, monkeypatch):
    (tmp_path / "gated_delta_rule_99_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "include").mkdir()
    (tmp_path / "gated_delta_rule_99_b200" / "csrc" / "k.cu").write_text("int k;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.csrc_hash()
    (tmp_path / "profiles" / "traffic.md").write_text(
        "| kernel | read bytes | write bytes | csrc hash | workload |\n|---|---|---|---|---|\n"
        "| tc_grads | 100 | 20 | %s | w1 |\n| tc_out | 5 | 5 | 0000000000000000 | w1 |\n" % h)
    assert bench.recorded_traffic("tc_grads", "w1") == 120
    assert bench.recorded_traffic("tc_grads", "w2") is None
    assert bench.recorded_traffic("tc_out", "w1") is None  # recorded for other sources
