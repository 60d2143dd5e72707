"""The source hash that ties a recorded ncu traffic figure to the kernel it
was measured on ignores comments and layout, and nothing else."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
spec = importlib.util.spec_from_file_location("_moe_build", os.path.join(ROOT, "expert_ffn_router_b200", "build.py"))
B = importlib.util.module_from_spec(spec)
spec.loader.exec_module(B)


def test_comments_and_layout_are_ignored():
    a = 'int f(int x) {  // the sum\n    return x + 1; /* one */ }\n'
    b = '/* header */\nint f(int x) {\n  return x + 1;\n}\n'
    assert B._code_only(a) == B._code_only(b)


def test_code_and_literals_count():
    assert B._code_only("return x + 1;") != B._code_only("return x + 2;")
    # comment markers inside string and character literals are code
    s = 'asm("ld.global // not a comment"); char c = \'/\'; // gone'
    assert B._code_only(s) == 'asm("ld.global // not a comment"); char c = \'/\';'
    assert B._code_only('s = "a\\"/* x */";') == 's = "a\\"/* x */";'


def test_hash_is_stable_and_short():
    h = B.source_hash()
    assert h == B.source_hash() and len(h) == 16
