"""Host-side helpers of the benchmark: the statistics of the timed steps and
the key that ties the stored ncu DRAM counters to the kernel code they were
taken on (comments and layout ignored, code and literals not)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_strip_comments_drops_comments_and_layout_only():
    src = ('int a = 1; // trailing\n'
           '/* a block\n   over lines */ const char* s = "// in a string /* too */";\n'
           "char c = '\"';  char d = '/';\n"
           '\n'
           '    int b;   /* inline */ int e;\n'
           'asm("mov.u32 %0, %1; // not a comment" : "=r"(x) : "r"(y));\n')
    assert bench.strip_comments(src) == (
        'int a = 1;\n'
        'const char* s = "// in a string /* too */";\n'
        "char c = '\"';  char d = '/';\n"
        'int b;    int e;\n'
        'asm("mov.u32 %0, %1; // not a comment" : "=r"(x) : "r"(y));')


def test_strip_comments_keeps_escaped_quotes():
    src = 'const char* s = "a \\" // b"; // c\n'
    assert bench.strip_comments(src) == 'const char* s = "a \\" // b";'


def test_code_changes_change_the_key_and_comments_do_not():
    a = "int f(int x) {\n  return x + 1;   // add one\n}\n"
    b = "// f adds one\nint f(int x) {\n    return x + 1;\n}\n"
    c = "int f(int x) {\n  return x + 2;   // add one\n}\n"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)


def test_spread_median_and_deciles():
    xs = [float(i) for i in range(1, 101)]
    s = bench.spread(xs)
    assert s["n"] == 100 and s["median"] == 50.5
    assert s["p10"] == 11.0 and s["p90"] == 90.0
    assert bench.spread([])["n"] == 0
