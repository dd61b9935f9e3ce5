"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of oracle/pqg_oracle.c: a dropped term,
a wrong sign, a wrong index, a transposed operand, or a wrong rounding rule.
The copy is built on the CPU, and the pin suite (test_oracle_pins.py) must
then fail against it.  The real oracle is never modified.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTANTS = {
    "ue8m0_no_bump": ("int bump = (bits & 0x7FFFFF) != 0;", "int bump = 0;"),
    "e4m3_ties_away": ("double n = nearbyint(a / quantum); /* exact quotient; ties to even */",
                       "double n = round(a / quantum); /* exact quotient; ties to even */"),
    "e4m3_zero_sign_lost": ("uint8_t sign = signbit(t) ? 0x80 : 0x00;",
                            "uint8_t sign = (t < 0) ? 0x80 : 0x00;"),
    "e4m3_no_saturation": ("if (a > 448.0) a = 448.0;", ";"),
    "no_eps_floor": ("if (a < PQGO_EPS) a = PQGO_EPS;", ";"),
    "int8_divides_by_448": ("return out_int8 ? amax / PQGO_FMAX_INT8",
                            "return out_int8 ? amax / PQGO_FMAX_E4M3"),
    "scale_by_reciprocal": (": amax / PQGO_FMAX_E4M3;", ": amax * (1.0f / PQGO_FMAX_E4M3);"),
    "col_layout_transposed": ("int64_t idx = e * ng * mpad + g * mpad + m;",
                              "int64_t idx = e * ng * mpad + m * ng + g;"),
    "masked_col_plane_unpadded": ("int64_t idx = e * ng * mpad + g * mpad + m;",
                                  "int64_t idx = e * ng * M + g * mpad + m;"),
    "masked_packed_plane_unpadded": ("int64_t word = e * nwords * mpad + (g / 4) * mpad + m;",
                                     "int64_t word = e * nwords * M + (g / 4) * mpad + m;"),
    "masked_tile_plane_floor": ("int64_t plane = ((M + 127) / 128) * ((ng + 3) / 4) * 512;\n"
                                "                    ((uint8_t *)scales)[e * plane",
                                "int64_t plane = (M / 128) * ((ng + 3) / 4) * 512;\n"
                                "                    ((uint8_t *)scales)[e * plane"),
    "row_layout_drops_group": ("int64_t idx = (e * M + m) * ng + g;",
                               "int64_t idx = (e * M + m) * ng;"),
    "fused_up_reads_gate": ("float up = pqgo_decode(xrow[K + g * G + i], in_fp16);",
                            "float up = pqgo_decode(xrow[g * G + i], in_fp16);"),
    "fused_gate_reads_up": ("float x = pqgo_decode(xrow[g * G + i], in_fp16);",
                            "float x = pqgo_decode(xrow[(fused ? K : 0) + g * G + i], in_fp16);"),
    "nvfp4_fused_up_reads_gate": ("float up = pqgo_decode(xrow[K + b * G + i], in_fp16);",
                                  "float up = pqgo_decode(xrow[b * G + i], in_fp16);"),
    "nvfp4_fused_gate_reads_up": ("float x = pqgo_decode(xrow[b * G + i], in_fp16);",
                                  "float x = pqgo_decode(xrow[(fused ? K : 0) + b * G + i], in_fp16);"),
    "silu_wrong_sign": ("double silu = g / (1.0 + exp(-g));",
                        "double silu = g / (1.0 + exp(g));"),
    "silu_single_precision": ("double silu = g / (1.0 + exp(-g));",
                              "double silu = (float)g / (1.0f + expf(-(float)g));"),
    "silu_product_rounded_twice": ("return (float)(silu * (double)up);",
                                   "return (float)((float)silu * (float)up);"),
    "packed_padding_not_zeroed": ("((uint8_t *)scales)[word * 4 + b] = 0;", ";"),
    "fp16_subnormal_exponent": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "int8_truncates": ("double n = nearbyint((double)t);", "double n = trunc((double)t);"),
    "e2m1_ties_away": ("double n = nearbyint(a / quantum);        /* ties to even */",
                       "double n = round(a / quantum);        /* ties to even */"),
    "mxfp4_uses_fmax448": ("ebyte = pqgo_ue8m0_exponent_fmax(amax, out_e2m1 ? PQGO_FMAX_E2M1",
                           "ebyte = pqgo_ue8m0_exponent_fmax(amax, out_e2m1 ? PQGO_FMAX_E4M3"),
    "tile_rows_not_interleaved": ("(r % 32) * 16 + (r / 32) * 4", "(r % 32) * 4 + (r / 32) * 128"),
    "nvfp4_scale_uses_fmax448": ("float r = (amax / PQGO_FMAX_E2M1) * g;",
                                 "float r = (amax / PQGO_FMAX_E4M3) * g;"),
    "nvfp4_global_scale_ignored": ("float r = (amax / PQGO_FMAX_E2M1) * g;",
                                   "float r = (amax / PQGO_FMAX_E2M1);"),
    "nvfp4_multiplier_inverted": ("return d == 0.0f ? 0.0f : g / d;",
                                  "return d == 0.0f ? 0.0f : d / g;"),
    "nvfp4_zero_scale_unguarded": ("return d == 0.0f ? 0.0f : g / d;", "return g / d;"),
    "nvfp4_nibbles_swapped": ("qrow[(b * G + i) / 2] = (uint8_t)(lo | (hi << 4));",
                              "qrow[(b * G + i) / 2] = (uint8_t)(hi | (lo << 4));"),
    "nvfp4_masked_col_plane_unpadded": ("scales[e * ng * mpad + b * mpad + m] = sf;",
                                        "scales[e * ng * M + b * mpad + m] = sf;"),
    "nvfp4_tile_plane_floor": ("const int64_t plane = ((M + 127) / 128) * ((ng + 3) / 4) * 512;",
                               "const int64_t plane = (M / 128) * ((ng + 3) / 4) * 512;"),
    "nvfp4_tile_padding_not_zeroed": ("scales[e * plane + tile128x4_offset(m, b, ng)] = 0;", ";"),
    "varlen_lens_ignored": ("        if (lens) {\n            n = lens[e];",
                            "        if (0) {\n            n = lens[e];"),
    "varlen_lens_not_clamped_to_segment": ("if (n > end - start) n = end - start;", ";"),
    "varlen_segment_from_next_offset": ("int64_t start = indptr[e], end = indptr[e + 1];",
                                        "int64_t start = indptr[e + 1], end = indptr[e + 1];"),
    "varlen_padding_rows_quantized": (
        "if (row_live && !row_live[m]) continue;   /* varlen padding row */\n"
        "            const uint16_t *xrow = in + (e * M + m) * in_width;\n"
        "            uint8_t *qrow = out + (e * M + m) * (out_e2m1",
        "if (0) continue;   /* varlen padding row */\n"
        "            const uint16_t *xrow = in + (e * M + m) * in_width;\n"
        "            uint8_t *qrow = out + (e * M + m) * (out_e2m1"),
    "varlen_nvfp4_padding_rows_quantized": (
        "if (row_live && !row_live[m]) continue;   /* varlen padding row */\n"
        "            const uint16_t *xrow = in + (e * M + m) * in_width;\n"
        "            uint8_t *qrow = out + (e * M + m) * (K / 2);",
        "if (0) continue;   /* varlen padding row */\n"
        "            const uint16_t *xrow = in + (e * M + m) * in_width;\n"
        "            uint8_t *qrow = out + (e * M + m) * (K / 2);"),
}


def _run_pins_against(name, old, new, tmp):
    src = open(os.path.join(ROOT, "oracle", "pqg_oracle.c")).read()
    assert src.count(old) == 1, f"{name}: anchor not found exactly once"
    path = os.path.join(tmp, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(force=True, src=path, out=os.path.join(tmp, f"{name}.so"))
    env = dict(os.environ, PQG_ORACLE_LIB=lib)
    res = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                         env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    return name, res.returncode, res.stdout[-600:]


@pytest.mark.slow
def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda kv: _run_pins_against(kv[0], *kv[1], tmp),
                                  MUTANTS.items()))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mistakes no pin catches: {[n for n, _ in survivors]}"
    assert all(rc == 1 for _, rc, _ in results), [(n, rc) for n, rc, _ in results]
