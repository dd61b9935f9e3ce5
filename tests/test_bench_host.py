"""Host logic of bench.py that needs no GPU: the source digest that tells
whether the stored ncu traffic counters still describe the built kernels."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = '''// header comment
#define X 48u   // trailing comment

/* a block
   comment */ int f(const char *s) { return s[0] == '/' ? 1 : 2; }
const char *url = "http://example/*not a comment*/";
'''


def test_comments_and_blank_lines_do_not_count():
    code = bench.code_only(SRC)
    assert code == ("#define X 48u\n"
                    " int f(const char *s) { return s[0] == '/' ? 1 : 2; }\n"
                    'const char *url = "http://example/*not a comment*/";')
    reflowed = SRC.replace("// header comment\n", "// a header comment\n// over two lines\n\n")
    assert bench.code_only(reflowed) == code


def test_a_code_change_moves_the_digest_input():
    assert bench.code_only(SRC.replace("48u", "47u")) != bench.code_only(SRC)
    assert bench.code_only(SRC.replace("'/'", "'*'")) != bench.code_only(SRC)
    assert bench.code_only(SRC.replace("example", "exampl")) != bench.code_only(SRC)


def test_digests_separate_the_two_kernels():
    strip, row = bench.source_digest("strip"), bench.source_digest("row")
    assert len(strip) == len(row) == 64 and strip != row
