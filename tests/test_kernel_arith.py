"""CPU checks of the arithmetic shortcuts the CUDA kernels take.

The kernels replace three divisions by cheaper sequences, and their comments
state the checks that justify each one (``tests/arith/kernel_arith.c`` restates
every shortcut in plain C and compares it with the definition it replaces):

- the UE8M0 byte from the exponent and mantissa bits of amax, with no
  division (FMAX 448 and FMAX 6);
- RN(amax / c) for c = 448, 127 and 6 by a reciprocal and two Markstein steps;
- one Markstein step (instead of two) before the E4M3 / INT8 cast of x / s;
- s / segs (strip index to row), and s / (spec * segs) in the masked decode
  form, by a multiply-high with a host-computed magic.

By default every 97th (or 4099th) case is checked, so the suite stays fast;
``PQG_EXHAUSTIVE=1`` checks every case (minutes on 8 cores for bf16, about half
an hour for fp16).  The oracle does not use any of these shortcuts.
"""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "arith", "kernel_arith.c")
FULL = os.environ.get("PQG_EXHAUSTIVE") == "1"


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("arith") / "kernel_arith")
    subprocess.run(["gcc", "-O2", "-mfma", "-fopenmp", "-ffp-contract=off", "-o", exe, SRC,
                    "-lm"], check=True)
    return exe


def run(exe, *args):
    out = subprocess.run([exe, *map(str, args)], capture_output=True, text=True, check=True,
                         timeout=7200).stdout.split()
    return int(out[0]), int(out[1])


@pytest.mark.parametrize("fmax", [448, 6])
def test_ue8m0_byte_without_division(checker, fmax):
    n, bad = run(checker, "ue8m0", fmax, 1 if FULL else 97)
    assert n > 10_000_000 and bad == 0


@pytest.mark.parametrize("c", [448, 127, 6])
def test_constant_division_is_correctly_rounded(checker, c):
    n, bad = run(checker, "cdiv", c, 1 if FULL else 97)
    assert n > 10_000_000 and bad == 0


STEP_CASES = pytest.mark.parametrize(
    "bits,kind", [(8, 0), (8, 1), (11, 0), (11, 1)],
    ids=["bf16-e4m3", "bf16-int8", "fp16-e4m3", "fp16-int8"])


@STEP_CASES
def test_one_markstein_step_gives_the_same_codes(checker, bits, kind):
    n, bad = run(checker, "steps", bits, kind, 1 if FULL else 4099)
    assert n > 1_000_000 and bad == 0


@STEP_CASES
def test_one_markstein_step_near_every_rounding_midpoint(checker, bits, kind):
    """The cases that can fail: x / s within a few ulps of a code midpoint."""
    n, bad = run(checker, "hard", bits, kind)
    assert n > 500_000 and bad == 0


def test_strip_row_division_by_magic_multiply(checker):
    """Every strips-per-row count up to 2^20 (K up to 2^29), 200 strip indices
    each: both ends of the index range next to quotient boundaries, and random."""
    n, bad = run(checker, "divsegs", 1)
    assert n == 200 * (1 << 20) and bad == 0


def test_decode_region_division_by_magic_multiply(checker):
    """The masked decode form divides by spec * segs (spec <= 8, segs <= 2^19):
    every divisor from 2^20 + 1 to 2^22, 200 strip indices each."""
    n, bad = run(checker, "divsegs", 1, (1 << 20) + 1, 1 << 22)
    assert n == 200 * 3 * (1 << 20) and bad == 0
