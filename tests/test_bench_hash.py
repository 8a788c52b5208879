"""The bench reports an ncu capture's DRAM traffic only while the kernel's
sources, comments removed, hash to the value stored with the capture."""
import importlib.util
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]


def load_bench():
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("bench_module", ROOT / "bench.py")
        m = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(m)
        return m
    finally:
        sys.argv = argv


def test_comments_do_not_count_but_code_does():
    b = load_bench()
    src = "int f(int a) {  // add one\n    /* the\n       increment */\n    return a + 1;\n}\n"
    reworded = "int f(int a) {  // plus one\n    return a + 1;   /* done */\n}\n"
    changed = "int f(int a) {  // add one\n    return a + 2;\n}\n"
    assert b.strip_comments(src) == b.strip_comments(reworded)
    assert b.strip_comments(src) != b.strip_comments(changed)

