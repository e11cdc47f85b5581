"""Host-side helpers of bench.py that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_keeps_strings():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ asm volatile("mbarrier.try_wait // not a comment");\n'
           "char q = '\"'; char r = '/';\n"
           '\n'
           'int b = a / 2; /* inline */ int c = b;\n')
    got = bench.code_only(src)
    assert got == ('int a = 1;\n'
                   ' asm volatile("mbarrier.try_wait // not a comment");\n'
                   "char q = '\"'; char r = '/';\n"
                   'int b = a / 2;  int c = b;')


def test_source_hash_ignores_comment_edits(tmp_path, monkeypatch):
    csrc = tmp_path / "gated_delta_rule_fg_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in bench.TC_SOURCES:
        (csrc / n).write_text("// header\n__global__ void k() { int x = 1; }  // note\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_hash()
    for n in bench.TC_SOURCES:
        (csrc / n).write_text("// another header\n\n__global__ void k() { int x = 1; }\n")
    assert bench.source_hash() == h0
    (csrc / bench.TC_SOURCES[0]).write_text("__global__ void k() { int x = 2; }\n")
    assert bench.source_hash() != h0
