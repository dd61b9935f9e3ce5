"""Host logic of bench.py that needs no GPU: the source digest that tells
whether the stored ncu traffic counters still describe the built kernels, the
sample statistics of the timed region, and the bench commands the ncu
summaries under profiles/ were captured on (listed in profiles/captures.json)."""
import json
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


def test_capture_commands_run_committed_code_on_known_workloads():
    """Every summary under profiles/ has an entry in captures.json naming the
    bench command it was captured on; that command must be bench.py with flags
    it accepts and a workload it knows, and every listed summary must exist."""
    prof = os.path.join(ROOT, "profiles")
    with open(os.path.join(prof, "captures.json"), encoding="utf-8") as f:
        caps = json.load(f)["captures"]
    known = set(bench.workloads())
    listed = {c["summary"] for c in caps}
    on_disk = {n for n in os.listdir(prof) if n.endswith(".md") and n != "README.md"}
    assert listed == on_disk, (listed ^ on_disk)
    for c in caps:
        flags = c["bench_command"].split()
        assert flags[:2] == ["python", "bench.py"], c
        if "--workload" in flags:
            assert flags[flags.index("--workload") + 1] in known, c
        assert set(f for f in flags if f.startswith("--")) <= {
            "--kernel-only", "--steps", "--warmup", "--no-cpu-baseline", "--workload",
            "--samples", "--gpus"}, c
        assert "--clock-control none" in c["ncu"], c
    assert len(caps) >= 9
