"""The benchmark's own timing on a GPU: a number it prints must be physically
possible.  A CUDA-graph replay timed on the wrong stream once reported a fused
step three times faster than HBM allows; these checks catch that class of
mistake (events that do not bracket the work)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--kernel-only",
                          "--no-cpu-baseline", "--warmup", "3", *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])


@pytest.mark.parametrize("workload", ["fused", "flat_hidden"])
def test_graph_replay_is_timed_on_its_stream(workload):
    """Bandwidth-bound calls: a graph removes host launch cost, which these
    calls already hide behind the device, so the graph cannot be much faster
    than stream launches (it can be slower: the replay loses some of the
    programmatic-launch overlap), and neither beats the HBM roofline."""
    # Two stream-launch runs, compared by the faster: one process on a busy
    # host can measure a short call a third slower than the next one does.
    eager = [bench("--workload", workload, "--steps", "100") for _ in range(2)]
    graph = bench("--workload", workload, "--steps", "100", "--graph")
    assert graph["gpu_launches"] == 100
    best = min(e["ms_per_step"] for e in eager)
    assert graph["ms_per_step"] >= 0.8 * best
    assert graph["roofline"]["frac"] < 1.2 and all(e["roofline"]["frac"] < 1.2 for e in eager)
