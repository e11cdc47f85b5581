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


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with the
    reference arm's keys; a tiny sample keeps this to seconds."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-seconds", "0.5"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
