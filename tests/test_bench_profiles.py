"""The bench's link to the committed ncu summaries (CPU): `roofline.traffic` is taken from a
profile only while the profile's kernel-source hash matches the CUDA sources' code, and that
hash ignores comments and layout but not code."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_tokens_drop_comments_and_layout():
    src = 'int a = 1; // one\n/* block\n comment */ int  b =\n 2;\n'
    assert bench._code_tokens(src) == "int a = 1; int b = 2;"


def test_code_tokens_keep_string_literals():
    # a comment marker inside a string or a character literal is code
    src = 'asm("mov.u32 %0, 1; // not a comment");  // a comment\nchar c = \'/\'; char d = \'"\';\n'
    toks = bench._code_tokens(src)
    assert '"mov.u32 %0, 1; // not a comment"' in toks
    assert "a comment\n" not in toks and toks.endswith("char c = '/'; char d = '\"';")


def test_code_edits_change_the_tokens():
    a = "x = y + 1; // note"
    assert bench._code_tokens(a) == bench._code_tokens("x = y + 1;  // other note")
    assert bench._code_tokens(a) != bench._code_tokens("x = y + 2; // note")


def test_committed_profiles_name_the_current_kernel():
    # both summaries carry the hash of the sources they were captured on; the bench line
    # reports their DRAM bytes only while the sources' code is unchanged
    h = bench._kernel_hash()
    for k, name in bench.PROFILES.items():
        path = os.path.join(ROOT, "profiles", name)
        text = open(path, encoding="utf-8").read()
        assert "kernel_source_hash:" in text and "dram_bytes_per_launch:" in text, name
        if f"kernel_source_hash: {h}" in text:
            assert bench._profiled_traffic(k) > 0
        else:
            assert bench._profiled_traffic(k) is None
