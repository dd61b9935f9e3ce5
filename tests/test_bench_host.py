"""Host logic of bench.py that needs no GPU: the source digest that tells
whether the stored ncu traffic counters still describe the built kernels, and
the bench commands the ncu summaries under profiles/ were captured on."""
import os
import re
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


def test_profile_commands_run_committed_code_on_known_workloads():
    """Every ncu summary names the bench command it was captured on; that
    command must be bench.py with flags it accepts and a workload it knows."""
    prof = os.path.join(ROOT, "profiles")
    known = set(bench.workloads())
    seen = 0
    for name in sorted(os.listdir(prof)):
        if not name.endswith(".md") or name == "README.md":
            continue
        text = open(os.path.join(prof, name), encoding="utf-8").read()
        cmds = re.findall(r"python bench\.py([^\n#\\]*)", text)
        assert cmds, f"{name} gives no bench command"
        for args in cmds:
            flags = args.split()
            if "--workload" in flags:
                assert flags[flags.index("--workload") + 1] in known, (name, args)
            assert set(f for f in flags if f.startswith("--")) <= {
                "--kernel-only", "--steps", "--warmup", "--no-cpu-baseline", "--workload"}, (name, args)
            seen += 1
    assert seen >= 9
