"""CPU test of bench.py's reference arm: it runs the oracle on the host and
prints one JSON line with the fields the benchmark contract names."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def test_kernel_source_digest_ignores_comments_only():
    """The digest that ties the committed ncu traffic to the decode sources: a comment or whitespace edit keeps it, a
    code edit (also inside a string literal, such as an inline-PTX instruction) changes it."""
    sys.path.insert(0, ROOT)
    import bench

    src = 'int f(int x) { // the count\n  /* a block\n comment */ asm("add.s32 %0, %1, 1; // not a comment");\n  return x + 1;\n}\n'
    same = 'int f(int x) {   // another remark\n  asm("add.s32 %0, %1, 1; // not a comment");\n\n  return x + 1;   }\n'
    code_changed = src.replace("x + 1", "x + 2")
    string_changed = src.replace("add.s32", "sub.s32")
    t = bench._code_tokens
    assert t(src) == t(same)
    assert t(src) != t(code_changed) and t(src) != t(string_changed)
    assert "// not a comment" in t(src) and "the count" not in t(src)
    assert len(bench.kernel_sources_digest()) == 64
