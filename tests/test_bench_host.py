"""Host logic of bench.py that needs no GPU: the GEMM traffic figure is tied
to the kernel code (not its comments) it was captured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_keeps_strings():
    a = 'asm("cvt.rn // not a comment"); // a comment\n/* block\n comment */ int   x = 1;\n'
    assert bench._code_only(a) == 'asm("cvt.rn // not a comment"); int x = 1; '


def test_comment_edits_keep_the_hash_code_edits_change_it():
    base = "int f(int a) { // sum\n  return a + 1; /* one */\n}\n"
    comment_edit = "int f(int a) { // add one\n  return a + 1;   /* 1 */\n}\n"
    code_edit = "int f(int a) { // sum\n  return a + 2; /* one */\n}\n"
    assert bench._code_only(base) == bench._code_only(comment_edit)
    assert bench._code_only(base) != bench._code_only(code_edit)
    # tokens stay separated: "int x" and "intx" differ
    assert bench._code_only("int x;") != bench._code_only("intx;")


def test_traffic_is_null_once_the_kernel_code_differs(monkeypatch):
    # either the stored figure (kernel code unchanged since the capture) or
    # None; a stored hash of other code always gives None
    assert bench.gemm_traffic() in (bench.GEMM_TRAFFIC["bytes_per_launch"], None)
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "sources_sha256", "0" * 64)
    assert bench.gemm_traffic() is None
