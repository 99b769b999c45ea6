"""Host-side helpers of bench.py (CPU only).

A profile's DRAM counters are reported only while the kernel source's code
matches the digest recorded beside them; comment edits must not break that
match and code edits must.
"""
import bench


def test_code_only_strips_comments_but_not_strings():
    src = ('int a = 1;  // trailing "quoted" comment\n'
           '/* block\n   comment */ const char* s = "//not a comment";\n'
           "char c = '\"';\n\n   x++;  /* inline */ y--;\n")
    out = bench._code_only(src)
    assert "comment" not in out.replace("//not a comment", "")
    assert '"//not a comment"' in out
    assert "'\"'" in out
    assert "x++;" in out and "y--;" in out
    assert "\n\n" not in out


def test_code_only_is_invariant_to_comment_edits_and_sensitive_to_code():
    a = "int f(int x) {\n  // add one\n  return x + 1;\n}\n"
    b = "int f(int x) {\n  /* add one, documented differently */\n  return x + 1;  // same code\n}\n"
    c = "int f(int x) {\n  // add one\n  return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_source_digest_is_stable():
    d = bench.source_digest()
    assert len(d) == 16 and int(d, 16) >= 0
    assert bench.source_digest() == d
