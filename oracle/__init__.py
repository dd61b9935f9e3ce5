"""Scalar CPU oracle for per-token-group activation quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``pqg_oracle.c`` (plain scalar C, built here with gcc,
no fast-math, no fp contraction); this module only marshals numpy arrays.
Layouts and dtypes are named by strings so that no enum value is shared with the
CUDA path's header.

Source: sglang PR #30924 report, "[JIT] Trait-driven per_token_group_quant"
(实现拆解 items 1-2; 关键源码片段 ``ref_fp8_ue8m0``; 风险与影响 on the INT8
path), the TeleFuser "tf-kernel 安装与使用" page (使用示例, silu_and_mul halves)
and "FlashInfer GEMM 学习笔记" §6-7 (packed TMA-aligned scales, masked_m /
expected_m, MXFP4 at block 32 and NVFP4 at block 16; packed tokens per segment
for the grouped-contiguous dispatch).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pqg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_LOCK = threading.Lock()
_lib = None

LAYOUTS = {"row": 0, "col": 1, "packed": 2, "tile128x4": 3}
OUT_KINDS = {"e4m3": 0, "int8": 1, "e2m1": 2}


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc into a shared object; return its path."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle library and declare its C API.

    ``PQG_ORACLE_LIB`` names another build of ``pqg_oracle.c`` to load instead;
    the mutation test uses it to run the pins against oracles with planted
    mistakes."""
    global _lib
    default = path is None
    if default and _lib is not None:
        return _lib
    if default and os.environ.get("PQG_ORACLE_LIB"):
        path = os.environ["PQG_ORACLE_LIB"]
    with _LOCK:
        if default and _lib is not None:
            return _lib
        lib = ctypes.CDLL(path or build())
        i64, i32, vp, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float
        lib.pqgo_quant.restype = i32
        lib.pqgo_quant.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32,
                                   i32, i32, vp]
        lib.pqgo_scales_nbytes.restype = i64
        lib.pqgo_scales_nbytes.argtypes = [i64, i64, i64, i32, i32, i32]
        lib.pqgo_decode.restype = f32
        lib.pqgo_decode.argtypes = [ctypes.c_uint16, i32]
        lib.pqgo_silu_mul.restype = f32
        lib.pqgo_silu_mul.argtypes = [f32, f32]
        lib.pqgo_group_amax.restype = f32
        lib.pqgo_group_amax.argtypes = [vp, i64]
        lib.pqgo_scale_fp32.restype = f32
        lib.pqgo_scale_fp32.argtypes = [f32, i32]
        lib.pqgo_ue8m0_exponent.restype = i32
        lib.pqgo_ue8m0_exponent.argtypes = [f32]
        lib.pqgo_e4m3_encode.restype = ctypes.c_uint8
        lib.pqgo_e4m3_encode.argtypes = [f32]
        lib.pqgo_int8_encode.restype = ctypes.c_int8
        lib.pqgo_int8_encode.argtypes = [f32]
        for name in ("pqgo_decode_n", "pqgo_e4m3_encode_n", "pqgo_int8_encode_n",
                     "pqgo_ue8m0_exponent_n", "pqgo_e2m1_encode_n", "pqgo_ue8m0_exponent_fmax_n"):
            getattr(lib, name).restype = None
        lib.pqgo_decode_n.argtypes = [vp, vp, i64, i32]
        lib.pqgo_silu_mul_n.restype = None
        lib.pqgo_silu_mul_n.argtypes = [vp, vp, vp, i64]
        lib.pqgo_e4m3_encode_n.argtypes = [vp, vp, i64]
        lib.pqgo_int8_encode_n.argtypes = [vp, vp, i64]
        lib.pqgo_ue8m0_exponent_n.argtypes = [vp, vp, i64]
        lib.pqgo_e2m1_encode_n.argtypes = [vp, vp, i64]
        lib.pqgo_ue8m0_exponent_fmax_n.argtypes = [vp, vp, i64, f32]
        lib.pqgo_scale_fp32_n.restype = None
        lib.pqgo_scale_fp32_n.argtypes = [vp, vp, i64, i32]
        lib.pqgo_quant_nvfp4.restype = i32
        lib.pqgo_quant_nvfp4.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, vp, f32]
        for name in ("pqgo_e4m3_decode_n", "pqgo_nvfp4_block_scale_n", "pqgo_nvfp4_multiplier_n"):
            getattr(lib, name).restype = None
        lib.pqgo_e4m3_decode_n.argtypes = [vp, vp, i64]
        lib.pqgo_nvfp4_block_scale_n.argtypes = [vp, vp, i64, f32]
        lib.pqgo_nvfp4_multiplier_n.argtypes = [vp, vp, i64, f32]
        lib.pqgo_varlen_rows.restype = None
        lib.pqgo_varlen_rows.argtypes = [vp, vp, i64, i64, vp]
        lib.pqgo_quant_varlen.restype = i32
        lib.pqgo_quant_varlen.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, i32,
                                          vp, vp, i64]
        lib.pqgo_quant_varlen_nvfp4.restype = i32
        lib.pqgo_quant_varlen_nvfp4.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp, vp,
                                                i64, f32]
        if default:
            _lib = lib
        return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


# --------------------------------------------------------------------------
# element functions (array in, array out)
# --------------------------------------------------------------------------

def decode(bits, in_dtype: str = "bf16", lib=None) -> np.ndarray:
    lib = lib or load()
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float32)
    lib.pqgo_decode_n(_ptr(b), _ptr(out), b.size, int(in_dtype == "fp16"))
    return out


def silu_mul(gate, up, lib=None) -> np.ndarray:
    lib = lib or load()
    g, u = _c(gate, np.float32), _c(up, np.float32)
    y = np.empty(g.shape, np.float32)
    lib.pqgo_silu_mul_n(_ptr(g), _ptr(u), _ptr(y), g.size)
    return y


def e4m3_encode(t, lib=None) -> np.ndarray:
    lib = lib or load()
    t = _c(t, np.float32)
    q = np.empty(t.shape, np.uint8)
    lib.pqgo_e4m3_encode_n(_ptr(t), _ptr(q), t.size)
    return q


def int8_encode(t, lib=None) -> np.ndarray:
    lib = lib or load()
    t = _c(t, np.float32)
    q = np.empty(t.shape, np.int8)
    lib.pqgo_int8_encode_n(_ptr(t), _ptr(q), t.size)
    return q


def e2m1_encode(t, lib=None) -> np.ndarray:
    lib = lib or load()
    t = _c(t, np.float32)
    q = np.empty(t.shape, np.uint8)
    lib.pqgo_e2m1_encode_n(_ptr(t), _ptr(q), t.size)
    return q


def ue8m0_exponent_fmax(amax, fmax: float, lib=None) -> np.ndarray:
    lib = lib or load()
    a = _c(amax, np.float32)
    e = np.empty(a.shape, np.uint8)
    lib.pqgo_ue8m0_exponent_fmax_n(_ptr(a), _ptr(e), a.size, float(fmax))
    return e


def ue8m0_exponent(amax, lib=None) -> np.ndarray:
    lib = lib or load()
    a = _c(amax, np.float32)
    e = np.empty(a.shape, np.uint8)
    lib.pqgo_ue8m0_exponent_n(_ptr(a), _ptr(e), a.size)
    return e


def scale_fp32(amax, out_dtype: str = "e4m3", lib=None) -> np.ndarray:
    lib = lib or load()
    a = _c(amax, np.float32)
    s = np.empty(a.shape, np.float32)
    lib.pqgo_scale_fp32_n(_ptr(a), _ptr(s), a.size, int(out_dtype == "int8"))
    return s


def e4m3_decode(codes, lib=None) -> np.ndarray:
    lib = lib or load()
    c = _c(codes, np.uint8)
    v = np.empty(c.shape, np.float32)
    lib.pqgo_e4m3_decode_n(_ptr(c), _ptr(v), c.size)
    return v


def nvfp4_block_scale(amax, global_scale: float, lib=None) -> np.ndarray:
    """E4M3 block-scale codes of blocks with these absmax values (NVFP4)."""
    lib = lib or load()
    a = _c(amax, np.float32)
    sf = np.empty(a.shape, np.uint8)
    lib.pqgo_nvfp4_block_scale_n(_ptr(a), _ptr(sf), a.size, float(global_scale))
    return sf


def nvfp4_multiplier(sf, global_scale: float, lib=None) -> np.ndarray:
    """fp32 multipliers g / value(sf) (0 for a zero block scale)."""
    lib = lib or load()
    c = _c(sf, np.uint8)
    m = np.empty(c.shape, np.float32)
    lib.pqgo_nvfp4_multiplier_n(_ptr(c), _ptr(m), c.size, float(global_scale))
    return m


def group_amax(v, lib=None) -> float:
    lib = lib or load()
    v = _c(v, np.float32)
    return float(lib.pqgo_group_amax(_ptr(v), v.size))


# --------------------------------------------------------------------------
# the whole quantization
# --------------------------------------------------------------------------

def scales_shape(E: int, M: int, K: int, group: int, scale_fmt: str, layout: str):
    """numpy (shape, dtype) of the scale buffer of one call."""
    ng = K // group
    mpad = (M + 3) // 4 * 4
    if layout == "row":
        shape = (E, M, ng)
    elif layout == "col":
        shape = (E, ng, mpad)
    elif layout == "tile128x4":
        return (E, (M + 127) // 128 * ((ng + 3) // 4) * 512), np.uint8
    else:
        return (E, (ng + 3) // 4, mpad), np.int32
    return shape, (np.float32 if scale_fmt == "fp32" else np.uint8)


def quant(x_bits, *, M: int, K: int, group: int, E: int = 1, in_dtype: str = "bf16",
          out_dtype: str = "e4m3", scale_fmt: str = "fp32", layout: str = "row",
          fused: bool = False, masked_m=None, out: np.ndarray | None = None,
          scales: np.ndarray | None = None, fill: int = 0xA5, global_scale=None, lib=None):
    """Run the oracle on host arrays.

    ``x_bits`` holds raw 16-bit patterns shaped [E, M, K] ([E, M, 2K] fused;
    the E axis may be omitted when E == 1).  ``out``/``scales`` may be given
    prefilled (rows the call must not touch are then checked by the caller);
    otherwise they are allocated filled with ``fill``.  Returns (out, scales)
    shaped [E, M, K] ([E, M, K/2] for E2M1) and per ``scales_shape``.
    NVFP4 is ``out_dtype="e2m1", scale_fmt="e4m3", group=16`` with the fp32
    ``global_scale``.
    """
    lib = lib or load()
    x = _c(x_bits, np.uint16)
    width = 2 * K if fused else K
    if x.size != E * M * width:
        raise ValueError(f"x has {x.size} elements, expected {E * M * width}")
    kbytes = K // 2 if out_dtype == "e2m1" else K
    if out is None:
        out = np.full((E, M, kbytes), fill, np.uint8)
    shape, sdt = scales_shape(E, M, K, group, scale_fmt, layout)
    if scales is None:
        scales = np.empty(shape, sdt)
        scales.view(np.uint8).fill(fill)
    nbytes = lib.pqgo_scales_nbytes(E, M, K, group, int(scale_fmt != "fp32"),
                                    LAYOUTS[layout])
    if scales.nbytes != nbytes or out.size != E * M * kbytes:
        raise ValueError("output buffers have the wrong size")
    mm = None
    if masked_m is not None:
        mm = _c(masked_m, np.int32)
        if mm.size != E:
            raise ValueError("masked_m needs one entry per expert")
    if scale_fmt == "e4m3":
        if out_dtype != "e2m1" or group != 16 or global_scale is None:
            raise ValueError("E4M3 block scales are NVFP4: e2m1 codes, group 16, a global scale")
        rc = lib.pqgo_quant_nvfp4(_ptr(x), _ptr(out), _ptr(scales), E, M, K,
                                  int(in_dtype == "fp16"), LAYOUTS[layout], int(bool(fused)),
                                  None if mm is None else _ptr(mm), float(global_scale))
        if rc != 0:
            raise ValueError(f"oracle rejected the call (status {rc})")
        return out, scales
    rc = lib.pqgo_quant(_ptr(x), _ptr(out), _ptr(scales), E, M, K, group,
                        int(in_dtype == "fp16"), OUT_KINDS[out_dtype],
                        int(scale_fmt == "ue8m0"), LAYOUTS[layout], int(bool(fused)),
                        None if mm is None else _ptr(mm))
    if rc != 0:
        raise ValueError(f"oracle rejected the call (status {rc})")
    return out, scales


# --------------------------------------------------------------------------
# grouped-contiguous (varlen) dispatch
# --------------------------------------------------------------------------

def varlen_rows(seg_indptr, seg_lens, M: int, lib=None) -> np.ndarray:
    """bool [M]: the token rows of the segments (see pqgo_varlen_rows)."""
    lib = lib or load()
    ip = _c(seg_indptr, np.int32)
    E = ip.size - 1
    ln = None if seg_lens is None else _c(seg_lens, np.int32)
    if E < 1 or (ln is not None and ln.size != E):
        raise ValueError("seg_indptr needs E + 1 entries and seg_lens E")
    live = np.empty(max(M, 1), np.uint8)
    lib.pqgo_varlen_rows(_ptr(ip), None if ln is None else _ptr(ln), E, M, _ptr(live))
    return live[:M].astype(bool)


def quant_varlen(x_bits, *, M: int, K: int, group: int, seg_indptr, seg_lens=None,
                 in_dtype: str = "bf16", out_dtype: str = "e4m3", scale_fmt: str = "fp32",
                 layout: str = "row", fused: bool = False, out: np.ndarray | None = None,
                 scales: np.ndarray | None = None, fill: int = 0xA5, global_scale=None,
                 lib=None):
    """Grouped-contiguous (varlen) call on M packed rows ([M, K], [M, 2K] fused):
    only the token rows of the segments are quantized, into the same rows of
    ``out`` and of one scale plane of M rows.  Returns (out [M, K] or [M, K/2],
    scales shaped as a flat call's [1, ...]); untouched bytes keep ``fill``."""
    lib = lib or load()
    x = _c(x_bits, np.uint16)
    width = 2 * K if fused else K
    if x.size != M * width:
        raise ValueError(f"x has {x.size} elements, expected {M * width}")
    ip = _c(seg_indptr, np.int32)
    E = ip.size - 1
    ln = None if seg_lens is None else _c(seg_lens, np.int32)
    if E < 1 or (ln is not None and ln.size != E):
        raise ValueError("seg_indptr needs E + 1 entries and seg_lens E")
    kbytes = K // 2 if out_dtype == "e2m1" else K
    if out is None:
        out = np.full((M, kbytes), fill, np.uint8)
    shape, sdt = scales_shape(1, M, K, group, scale_fmt, layout)
    if scales is None:
        scales = np.empty(shape, sdt)
        scales.view(np.uint8).fill(fill)
    nbytes = lib.pqgo_scales_nbytes(1, M, K, group, int(scale_fmt != "fp32"), LAYOUTS[layout])
    if scales.nbytes != nbytes or out.size != M * kbytes:
        raise ValueError("output buffers have the wrong size")
    lp = None if ln is None else _ptr(ln)
    if scale_fmt == "e4m3":
        if out_dtype != "e2m1" or group != 16 or global_scale is None:
            raise ValueError("E4M3 block scales are NVFP4: e2m1 codes, group 16, a global scale")
        rc = lib.pqgo_quant_varlen_nvfp4(_ptr(x), _ptr(out), _ptr(scales), M, K,
                                         int(in_dtype == "fp16"), LAYOUTS[layout],
                                         int(bool(fused)), _ptr(ip), lp, E, float(global_scale))
    else:
        rc = lib.pqgo_quant_varlen(_ptr(x), _ptr(out), _ptr(scales), M, K, group,
                                   int(in_dtype == "fp16"), OUT_KINDS[out_dtype],
                                   int(scale_fmt == "ue8m0"), LAYOUTS[layout], int(bool(fused)),
                                   _ptr(ip), lp, E)
    if rc != 0:
        raise ValueError(f"oracle rejected the call (status {rc})")
    return out, scales
