"""The C-ABI library loads, exports what include/pqg.h declares, and rejects bad
arguments on the host (CPU only).

No call here reaches a kernel launch.  Every pqg_quant call either carries an
argument the host-side checks reject or asks for zero rows, so these tests are
safe on any machine.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from precision_activation_quantization_b200 import pqg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pqg.h")

# a pointer-sized value that is 256-byte aligned but never dereferenced
FAKE = 1 << 40


def _no_device():
    try:
        import torch
        return not torch.cuda.is_available()
    except Exception:
        return True


# The calls below pass made-up device addresses; each one is rejected on the host
# before any launch.  Where a GPU is present they are skipped all the same, so
# that a regression in the checks could never launch a kernel on those addresses.
host_only = pytest.mark.skipif(not _no_device(), reason="made-up pointers: CPU-only check")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^PQG_API\s+[\w\s\*]*?\b(pqg_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert set(names) == set(pqg.EXPORTS)
    lib = ctypes.CDLL(pqg.LIBRARY_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_nothing_else_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", pqg.LIBRARY_PATH],
                         capture_output=True, text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if l.strip()}
    ours = {s for s in syms if s.startswith("pqg")}
    assert ours == set(declared_functions())


def test_header_compiles_as_c():
    refs = ", ".join(f"(void (*)(void)){n}" for n in declared_functions())
    src = ('#include "pqg.h"\nvoid (*table[])(void) = {' + refs + '};\n'
           'int main(void){ return table[0] == 0; }\n')
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                          "-I", os.path.join(ROOT, "include"), "-x", "c", "-"],
                         input=src, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_status_strings_and_version():
    for st in (pqg.PQG_OK, pqg.PQG_ERR_INVALID_ARG, pqg.PQG_ERR_UNSUPPORTED,
               pqg.PQG_ERR_ALIGNMENT, pqg.PQG_ERR_CUDA):
        assert pqg.pqg_status_string(st) not in ("", "unknown status")
    assert pqg.pqg_status_string(12345) == "unknown status"
    assert "sm_100a" in pqg.pqg_version()


def test_enum_values_match_header():
    text = open(HEADER).read()
    for name in ("PQG_OK", "PQG_ERR_INVALID_ARG", "PQG_ERR_UNSUPPORTED", "PQG_ERR_ALIGNMENT",
                 "PQG_ERR_CUDA", "PQG_BF16", "PQG_FP16", "PQG_E4M3", "PQG_INT8", "PQG_E2M1",
                 "PQG_SCALE_FP32", "PQG_SCALE_UE8M0", "PQG_SCALE_E4M3", "PQG_ROW_MAJOR",
                 "PQG_COL_MAJOR_TMA",
                 "PQG_UE8M0_PACKED", "PQG_UE8M0_TILED_128x4"):
        m = re.search(rf"\b{name}\s*=\s*(-?\d+)", text)
        assert m and int(m.group(1)) == getattr(pqg, name), name


def test_pdl_toggle_round_trips():
    prev = pqg.pqg_set_pdl(False)
    assert pqg.pqg_set_pdl(prev) is False
    assert pqg.pqg_set_pdl(prev) == prev


# --------------------------------------------------------------------------
# pqg_scales_bytes against the oracle's own size rule
# --------------------------------------------------------------------------

@pytest.mark.parametrize("E,M,K,G", [(1, 4, 256, 128), (1, 8192, 7168, 128), (3, 5, 640, 64),
                                     (32, 2048, 2048, 128), (2, 1, 96, 32), (1, 0, 128, 128)])
@pytest.mark.parametrize("fmt,layout", [("fp32", "row"), ("fp32", "col"), ("ue8m0", "row"),
                                        ("ue8m0", "col"), ("ue8m0", "packed"),
                                        ("ue8m0", "tile128x4")])
def test_scales_bytes_matches_oracle(E, M, K, G, fmt, layout):
    import oracle
    lib = oracle.load()
    want = lib.pqgo_scales_nbytes(E, M, K, G, int(fmt == "ue8m0"), oracle.LAYOUTS[layout])
    got = pqg.pqg_scales_bytes(E, M, K, G, pqg.SCALE_FMTS[fmt], pqg.LAYOUTS[layout])
    assert got == want
    shape, dt = pqg.scales_spec(M, K, G, fmt, layout, E)
    import torch
    assert int(np.prod(shape)) * torch.empty((), dtype=dt).element_size() == want


@pytest.mark.parametrize("E,M,K", [(1, 4, 256), (1, 8192, 7168), (3, 130, 80), (2, 1, 16)])
@pytest.mark.parametrize("layout", ["row", "col", "tile128x4"])
def test_nvfp4_scales_bytes_matches_oracle(E, M, K, layout):
    import oracle
    want = oracle.load().pqgo_scales_nbytes(E, M, K, 16, 1, oracle.LAYOUTS[layout])
    assert pqg.pqg_scales_bytes(E, M, K, 16, pqg.PQG_SCALE_E4M3, pqg.LAYOUTS[layout]) == want
    shape, dt = pqg.scales_spec(M, K, 16, "e4m3", layout, E)
    assert int(np.prod(shape)) == want


def test_per_token_scales_bytes():
    for K in (80, 7168, 16384):
        assert pqg.pqg_scales_bytes(1, 5, K, K, pqg.PQG_SCALE_FP32, pqg.PQG_ROW_MAJOR) == 5 * 4
        assert pqg.pqg_scales_bytes(2, 5, K, K, pqg.PQG_SCALE_UE8M0, pqg.PQG_UE8M0_PACKED) == 2 * 8 * 4


def test_scales_bytes_rejects():
    S, R, C, P = pqg.PQG_SCALE_FP32, pqg.PQG_ROW_MAJOR, pqg.PQG_COL_MAJOR_TMA, pqg.PQG_UE8M0_PACKED
    assert pqg.pqg_scales_bytes(1, 4, 256, 128, S, P) == pqg.PQG_ERR_UNSUPPORTED
    assert pqg.pqg_scales_bytes(1, 4, 256, 96, S, R) == pqg.PQG_ERR_UNSUPPORTED
    assert pqg.pqg_scales_bytes(1, 4, 200, 128, S, R) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(0, 4, 256, 128, S, R) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(1, -1, 256, 128, S, C) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(1, 4, 256, 128, 7, R) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(1, 4, 256, 128, S, 9) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(1, 4, 256, -128, S, R) == pqg.PQG_ERR_INVALID_ARG
    assert pqg.pqg_scales_bytes(1, 1 << 31, 512, 128, S, R) == pqg.PQG_ERR_INVALID_ARG
    E4 = pqg.PQG_SCALE_E4M3                          # NVFP4: blocks of 16, byte layouts
    assert pqg.pqg_scales_bytes(1, 4, 256, 32, E4, R) == pqg.PQG_ERR_UNSUPPORTED
    assert pqg.pqg_scales_bytes(1, 4, 256, 16, E4, P) == pqg.PQG_ERR_UNSUPPORTED
    assert pqg.pqg_scales_bytes(1, 4, 200, 16, E4, R) == pqg.PQG_ERR_INVALID_ARG


# --------------------------------------------------------------------------
# pqg_quant host-side validation (nothing is launched)
# --------------------------------------------------------------------------

def call(**kw):
    a = dict(in_ptr=FAKE, out_ptr=FAKE + (1 << 32), scales_ptr=FAKE + (2 << 32), M=4,
             num_experts=1, K=256, group=128, in_dtype=pqg.PQG_BF16, out_dtype=pqg.PQG_E4M3,
             scale_fmt=pqg.PQG_SCALE_FP32, scale_layout=pqg.PQG_ROW_MAJOR, fuse_silu_mul=0,
             masked_m_ptr=None, expected_m=0, stream=None)
    a.update(kw)
    return pqg.pqg_quant(**a)


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(in_dtype=5), pqg.PQG_ERR_INVALID_ARG),
    (dict(out_dtype=pqg.PQG_BF16), pqg.PQG_ERR_INVALID_ARG),
    (dict(scale_fmt=3), pqg.PQG_ERR_INVALID_ARG),
    (dict(scale_layout=-1), pqg.PQG_ERR_INVALID_ARG),
    (dict(group=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(group=16), pqg.PQG_ERR_UNSUPPORTED),
    (dict(group=256, K=512), pqg.PQG_ERR_UNSUPPORTED),
    (dict(group=512, K=1024), pqg.PQG_ERR_UNSUPPORTED),          # neither 32/64/128 nor K
    (dict(group=16400, K=16400), pqg.PQG_ERR_UNSUPPORTED),       # per-token K > 16384
    (dict(group=200, K=200), pqg.PQG_ERR_UNSUPPORTED),           # per-token K % 16 != 0
    (dict(K=200), pqg.PQG_ERR_INVALID_ARG),
    (dict(K=-256), pqg.PQG_ERR_INVALID_ARG),
    (dict(M=-1), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=70000), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=4097), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=4096, M=1 << 12, K=1 << 14), pqg.PQG_ERR_INVALID_ARG),  # 2^31 strips
    (dict(out_dtype=pqg.PQG_INT8, scale_fmt=pqg.PQG_SCALE_UE8M0), pqg.PQG_ERR_UNSUPPORTED),
    (dict(scale_layout=pqg.PQG_UE8M0_PACKED), pqg.PQG_ERR_UNSUPPORTED),
    (dict(scale_layout=pqg.PQG_UE8M0_TILED_128x4), pqg.PQG_ERR_UNSUPPORTED),
    (dict(out_dtype=pqg.PQG_E2M1), pqg.PQG_ERR_UNSUPPORTED),                 # needs UE8M0
    (dict(out_dtype=pqg.PQG_E2M1, scale_fmt=pqg.PQG_SCALE_UE8M0, group=256), pqg.PQG_ERR_UNSUPPORTED),
    (dict(out_dtype=5), pqg.PQG_ERR_INVALID_ARG),
    (dict(scale_layout=4), pqg.PQG_ERR_INVALID_ARG),
    (dict(in_ptr=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(out_ptr=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(scales_ptr=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(in_ptr=FAKE + 16), pqg.PQG_ERR_ALIGNMENT),
    (dict(out_ptr=FAKE + (1 << 32) + 8), pqg.PQG_ERR_ALIGNMENT),
    (dict(scales_ptr=FAKE + (2 << 32) + 2), pqg.PQG_ERR_ALIGNMENT),
    (dict(scales_ptr=FAKE + (2 << 32) + 2, scale_fmt=pqg.PQG_SCALE_UE8M0,
          scale_layout=pqg.PQG_UE8M0_PACKED), pqg.PQG_ERR_ALIGNMENT),
    (dict(scales_ptr=FAKE + (2 << 32) + 1, scale_fmt=pqg.PQG_SCALE_UE8M0,
          scale_layout=pqg.PQG_UE8M0_TILED_128x4), pqg.PQG_ERR_ALIGNMENT),   # word stores
    (dict(masked_m_ptr=FAKE + (3 << 32) + 2), pqg.PQG_ERR_ALIGNMENT),
    (dict(out_ptr=FAKE + 512), pqg.PQG_ERR_INVALID_ARG),          # overlaps the input
    (dict(scales_ptr=FAKE + (1 << 32) + 64), pqg.PQG_ERR_INVALID_ARG),  # overlaps out
    (dict(M=1 << 31), pqg.PQG_ERR_INVALID_ARG),
    (dict(K=1 << 29), pqg.PQG_ERR_INVALID_ARG),
])
def test_quant_rejects_before_launch(kw, status):
    before = pqg.pqg_launch_count()
    assert call(**kw) == status
    assert pqg.pqg_launch_count() == before


def call_nv(**kw):
    a = dict(in_ptr=FAKE, out_ptr=FAKE + (1 << 32), scales_ptr=FAKE + (2 << 32),
             global_scale_ptr=FAKE + (3 << 32), M=4, num_experts=1, K=256,
             in_dtype=pqg.PQG_BF16, scale_layout=pqg.PQG_ROW_MAJOR, fuse_silu_mul=0,
             masked_m_ptr=None, expected_m=0, stream=None)
    a.update(kw)
    return pqg.pqg_quant_nvfp4(**a)


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(global_scale_ptr=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(global_scale_ptr=FAKE + (3 << 32) + 2), pqg.PQG_ERR_ALIGNMENT),
    (dict(scale_layout=pqg.PQG_UE8M0_PACKED), pqg.PQG_ERR_UNSUPPORTED),
    (dict(scale_layout=7), pqg.PQG_ERR_INVALID_ARG),
    (dict(K=200), pqg.PQG_ERR_INVALID_ARG),
    (dict(in_dtype=9), pqg.PQG_ERR_INVALID_ARG),
    (dict(M=-1), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=4097), pqg.PQG_ERR_INVALID_ARG),
    (dict(in_ptr=FAKE + 16), pqg.PQG_ERR_ALIGNMENT),
    (dict(out_ptr=FAKE + (1 << 32) + 8), pqg.PQG_ERR_ALIGNMENT),
    (dict(out_ptr=FAKE + 256), pqg.PQG_ERR_INVALID_ARG),          # overlaps the input
])
def test_nvfp4_rejects_before_launch(kw, status):
    before = pqg.pqg_launch_count()
    assert call_nv(**kw) == status
    assert pqg.pqg_launch_count() == before


def call_var(**kw):
    a = dict(in_ptr=FAKE, out_ptr=FAKE + (1 << 32), scales_ptr=FAKE + (2 << 32),
             global_scale_ptr=None, M=64, num_experts=4, K=256, group=128,
             in_dtype=pqg.PQG_BF16, out_dtype=pqg.PQG_E4M3, scale_fmt=pqg.PQG_SCALE_UE8M0,
             scale_layout=pqg.PQG_COL_MAJOR_TMA, fuse_silu_mul=1,
             seg_indptr_ptr=FAKE + (3 << 32), seg_lens_ptr=FAKE + (4 << 32), expected_m=8,
             stream=None)
    a.update(kw)
    return pqg.pqg_quant_varlen(**a)


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(seg_indptr_ptr=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(seg_indptr_ptr=0, M=0), pqg.PQG_ERR_INVALID_ARG),         # needed even with no rows
    (dict(seg_indptr_ptr=FAKE + (3 << 32) + 2), pqg.PQG_ERR_ALIGNMENT),
    (dict(seg_lens_ptr=FAKE + (4 << 32) + 1), pqg.PQG_ERR_ALIGNMENT),
    (dict(num_experts=0), pqg.PQG_ERR_INVALID_ARG),
    (dict(num_experts=4097), pqg.PQG_ERR_INVALID_ARG),
    (dict(M=-1), pqg.PQG_ERR_INVALID_ARG),
    (dict(M=1 << 31), pqg.PQG_ERR_INVALID_ARG),
    (dict(K=200), pqg.PQG_ERR_INVALID_ARG),
    (dict(group=16), pqg.PQG_ERR_UNSUPPORTED),
    (dict(out_dtype=pqg.PQG_INT8), pqg.PQG_ERR_UNSUPPORTED),       # INT8 with UE8M0
    (dict(global_scale_ptr=FAKE + (5 << 32)), pqg.PQG_ERR_INVALID_ARG),   # g without NVFP4
    (dict(out_dtype=pqg.PQG_E2M1, scale_fmt=pqg.PQG_SCALE_E4M3, group=16),
     pqg.PQG_ERR_INVALID_ARG),                                      # NVFP4 without g
    (dict(in_ptr=FAKE + 16), pqg.PQG_ERR_ALIGNMENT),
    (dict(out_ptr=FAKE + 1024), pqg.PQG_ERR_INVALID_ARG),           # overlaps the input
    (dict(seg_indptr_ptr=FAKE + (1 << 32) + 64), pqg.PQG_ERR_INVALID_ARG),   # inside out
    (dict(seg_lens_ptr=FAKE + (2 << 32) + 4), pqg.PQG_ERR_INVALID_ARG),      # inside scales
])
def test_varlen_rejects_before_launch(kw, status):
    before = pqg.pqg_launch_count()
    assert call_var(**kw) == status
    assert pqg.pqg_launch_count() == before


@host_only
def test_varlen_zero_rows_is_ok_and_launches_nothing():
    before = pqg.pqg_launch_count()
    assert call_var(M=0, in_ptr=0, out_ptr=0, scales_ptr=0) == pqg.PQG_OK
    assert pqg.pqg_launch_count() == before


@host_only
def test_quant_refers_e4m3_block_scales_to_the_nvfp4_entry():
    assert call(out_dtype=pqg.PQG_E2M1, scale_fmt=pqg.PQG_SCALE_E4M3,
                group=16) == pqg.PQG_ERR_UNSUPPORTED


@host_only
def test_zero_rows_is_ok_and_launches_nothing():
    before = pqg.pqg_launch_count()
    assert call(M=0, in_ptr=0, out_ptr=0, scales_ptr=0) == pqg.PQG_OK
    assert pqg.pqg_launch_count() == before


@host_only
def test_ue8m0_bytes_need_no_alignment_check():
    # an odd scale pointer is fine for UE8M0 bytes; an unaligned input still fails first
    assert call(scale_fmt=pqg.PQG_SCALE_UE8M0, scales_ptr=FAKE + (2 << 32) + 1,
                in_ptr=FAKE + 8) == pqg.PQG_ERR_ALIGNMENT


def test_infer_scale_layout():
    import torch
    M, K, G = 6, 640, 128
    row = torch.empty(M, 5)
    assert pqg.infer_scale_layout(row, M, K, G) == "row"
    col = torch.empty(5, 8)[:, :M].t()
    assert pqg.infer_scale_layout(col, M, K, G) == "col"
    packed = torch.empty(2, 8, dtype=torch.int32)[:, :M].t()
    assert pqg.infer_scale_layout(packed, M, K, G) == "packed"
    with pytest.raises(ValueError):
        pqg.infer_scale_layout(torch.empty(M, 4), M, K, G)
