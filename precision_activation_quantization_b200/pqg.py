"""Python binding of libpqg.so (C ABI in include/pqg.h).

Argument marshalling only: every step of the quantization runs in the CUDA
library.  Importing this module loads the library, building it first with nvcc
when it is missing or older than its sources, and raises if that fails; there
is no fallback implementation.

``pqg_quant``, ``pqg_scales_bytes``, ``pqg_status_string`` and friends mirror
the C entry points one to one.  ``quant`` is the torch-facing convenience: it
takes tensors, allocates outputs when not given (torch is used for device memory
and streams only), and raises ``PqgError`` on a non-OK status.  The interface
follows the sglang PR #30924 report, "[JIT] Trait-driven per_token_group_quant"
(实现拆解 item 2: one entry taking masked_m and expected_m, an allocation helper
and a scale-layout inference helper).
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

# ---- enums (values of include/pqg.h) ---------------------------------------
PQG_OK = 0
PQG_ERR_INVALID_ARG = -1
PQG_ERR_UNSUPPORTED = -2
PQG_ERR_ALIGNMENT = -3
PQG_ERR_CUDA = -4

PQG_BF16, PQG_FP16, PQG_E4M3, PQG_INT8, PQG_E2M1 = 0, 1, 2, 3, 4
PQG_SCALE_FP32, PQG_SCALE_UE8M0, PQG_SCALE_E4M3 = 0, 1, 2
PQG_ROW_MAJOR, PQG_COL_MAJOR_TMA, PQG_UE8M0_PACKED, PQG_UE8M0_TILED_128x4 = 0, 1, 2, 3

IN_DTYPES = {"bf16": PQG_BF16, "fp16": PQG_FP16}
OUT_DTYPES = {"e4m3": PQG_E4M3, "int8": PQG_INT8, "e2m1": PQG_E2M1}
SCALE_FMTS = {"fp32": PQG_SCALE_FP32, "ue8m0": PQG_SCALE_UE8M0, "e4m3": PQG_SCALE_E4M3}
LAYOUTS = {"row": PQG_ROW_MAJOR, "col": PQG_COL_MAJOR_TMA, "packed": PQG_UE8M0_PACKED,
           "tile128x4": PQG_UE8M0_TILED_128x4}

EXPORTS = ("pqg_quant", "pqg_quant_nvfp4", "pqg_quant_varlen", "pqg_scales_bytes",
           "pqg_status_string", "pqg_last_cuda_error", "pqg_set_pdl", "pqg_launch_count",
           "pqg_version")


class PqgError(RuntimeError):
    def __init__(self, status: int, where: str = "pqg_quant"):
        self.status = status
        msg = pqg_status_string(status)
        if status == PQG_ERR_CUDA:
            msg += f" (cudaError {pqg_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [{status}]")


def _load() -> ctypes.CDLL:
    path = os.environ.get("PQG_LIBRARY") or _build.build()
    lib = ctypes.CDLL(path)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.pqg_quant.restype = i32
    lib.pqg_quant.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, i32, i32, vp,
                              i64, vp]
    lib.pqg_quant_nvfp4.restype = i32
    lib.pqg_quant_nvfp4.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, vp, i64, vp]
    lib.pqg_quant_varlen.restype = i32
    lib.pqg_quant_varlen.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, i32,
                                     i32, vp, vp, i64, vp]
    lib.pqg_scales_bytes.restype = i64
    lib.pqg_scales_bytes.argtypes = [i64, i64, i64, i32, i32, i32]
    lib.pqg_status_string.restype = ctypes.c_char_p
    lib.pqg_status_string.argtypes = [i32]
    lib.pqg_last_cuda_error.restype = i32
    lib.pqg_last_cuda_error.argtypes = []
    lib.pqg_set_pdl.restype = i32
    lib.pqg_set_pdl.argtypes = [i32]
    lib.pqg_launch_count.restype = ctypes.c_uint64
    lib.pqg_launch_count.argtypes = []
    lib.pqg_version.restype = ctypes.c_char_p
    lib.pqg_version.argtypes = []
    return lib


_lib = _load()
LIBRARY_PATH = _lib._name


# ---- the C entry points, one to one ----------------------------------------

def pqg_quant(in_ptr: int, out_ptr: int, scales_ptr: int, M: int, num_experts: int, K: int,
              group: int, in_dtype: int, out_dtype: int, scale_fmt: int, scale_layout: int,
              fuse_silu_mul: int, masked_m_ptr: int | None, expected_m: int,
              stream: int | None) -> int:
    return _lib.pqg_quant(in_ptr, out_ptr, scales_ptr, M, num_experts, K, group, in_dtype,
                          out_dtype, scale_fmt, scale_layout, fuse_silu_mul, masked_m_ptr,
                          expected_m, stream)


def pqg_quant_nvfp4(in_ptr: int, out_ptr: int, scales_ptr: int, global_scale_ptr: int, M: int,
                    num_experts: int, K: int, in_dtype: int, scale_layout: int,
                    fuse_silu_mul: int, masked_m_ptr: int | None, expected_m: int,
                    stream: int | None) -> int:
    return _lib.pqg_quant_nvfp4(in_ptr, out_ptr, scales_ptr, global_scale_ptr, M, num_experts,
                                K, in_dtype, scale_layout, fuse_silu_mul, masked_m_ptr,
                                expected_m, stream)


def pqg_quant_varlen(in_ptr: int, out_ptr: int, scales_ptr: int, global_scale_ptr: int | None,
                     M: int, num_experts: int, K: int, group: int, in_dtype: int,
                     out_dtype: int, scale_fmt: int, scale_layout: int, fuse_silu_mul: int,
                     seg_indptr_ptr: int | None, seg_lens_ptr: int | None, expected_m: int,
                     stream: int | None) -> int:
    return _lib.pqg_quant_varlen(in_ptr, out_ptr, scales_ptr, global_scale_ptr, M, num_experts,
                                 K, group, in_dtype, out_dtype, scale_fmt, scale_layout,
                                 fuse_silu_mul, seg_indptr_ptr, seg_lens_ptr, expected_m,
                                 stream)


def pqg_scales_bytes(num_experts: int, M: int, K: int, group: int, scale_fmt: int,
                     scale_layout: int) -> int:
    return _lib.pqg_scales_bytes(num_experts, M, K, group, scale_fmt, scale_layout)


def pqg_status_string(status: int) -> str:
    return _lib.pqg_status_string(status).decode()


def pqg_last_cuda_error() -> int:
    return _lib.pqg_last_cuda_error()


def pqg_set_pdl(enable: bool) -> bool:
    return bool(_lib.pqg_set_pdl(int(bool(enable))))


def pqg_launch_count() -> int:
    return int(_lib.pqg_launch_count())


def pqg_version() -> str:
    return _lib.pqg_version().decode()


# ---- torch-facing helpers ---------------------------------------------------

def scales_spec(M: int, K: int, group: int, scale_fmt: str = "fp32", layout: str = "row",
                num_experts: int = 1):
    """(shape, torch dtype) of a contiguous scale buffer for these arguments.

    row       : [E, M, ng]            fp32 or uint8
    col       : [E, ng, M_pad]        fp32 or uint8
    packed    : [E, ceil(ng/4), M_pad] int32
    tile128x4 : [E, ceil(M/128) * ceil(ng/4) * 512] uint8
    """
    import torch
    nbytes = pqg_scales_bytes(num_experts, M, K, group, SCALE_FMTS[scale_fmt], LAYOUTS[layout])
    if nbytes < 0:
        raise PqgError(nbytes, "pqg_scales_bytes")
    ng, mpad = K // group, (M + 3) // 4 * 4
    if layout == "row":
        shape = (num_experts, M, ng)
    elif layout == "col":
        shape = (num_experts, ng, mpad)
    elif layout == "tile128x4":
        return (num_experts, (M + 127) // 128 * ((ng + 3) // 4) * 512), torch.uint8
    else:
        return (num_experts, (ng + 3) // 4, mpad), torch.int32
    return shape, (torch.float32 if scale_fmt == "fp32" else torch.uint8)


def allocate_outputs(M: int, K: int, group: int, *, num_experts: int = 1,
                     out_dtype: str = "e4m3", scale_fmt: str = "fp32", layout: str = "row",
                     device=None):
    """Allocate (out, scales) for one call with torch (device memory only).
    E2M1 codes come back as uint8 [E, M, K/2], two codes per byte."""
    import torch
    if out_dtype == "e2m1":
        out = torch.empty((num_experts, M, K // 2), dtype=torch.uint8, device=device)
    else:
        odt = torch.float8_e4m3fn if out_dtype == "e4m3" else torch.int8
        out = torch.empty((num_experts, M, K), dtype=odt, device=device)
    shape, sdt = scales_spec(M, K, group, scale_fmt, layout, num_experts)
    return out, torch.empty(shape, dtype=sdt, device=device)


def infer_scale_layout(scales, M: int, K: int, group: int) -> str:
    """Scale layout of an [M, ng]-shaped view (or packed [M, ceil(ng/4)] int32 view)
    from its strides: contiguous rows -> "row"; unit stride along M -> "col", or
    "packed" for int32.  Mirrors the stride-based inference the pages describe."""
    import torch
    ng = K // group
    if scales.dim() != 2 or scales.shape[0] != M:
        raise ValueError("expected a 2-D [M, groups] view of the scales")
    if scales.dtype == torch.int32:
        if scales.shape[1] == (ng + 3) // 4 and (M <= 1 or scales.stride(0) == 1):
            return "packed"
    elif scales.shape[1] == ng:
        if scales.stride(1) == 1 and (M <= 1 or scales.stride(0) == ng):
            return "row"
        if M <= 1 or scales.stride(0) == 1:
            return "col"
    raise ValueError("scale view matches no supported layout")


def quant(x, out=None, scales=None, *, M: int | None = None, K: int | None = None,
          group: int = 128, num_experts: int | None = None, out_dtype: str = "e4m3",
          scale_fmt: str = "fp32", layout: str = "row", fuse_silu_mul: bool = False,
          masked_m=None, expected_m: int = 0, global_scale=None, stream=None):
    """Quantize a CUDA tensor; returns (out, scales).

    ``x`` is bf16/fp16, [E, M, K] / [M, K] ([..., 2K] when ``fuse_silu_mul``).
    ``masked_m`` is an int32 CUDA tensor of E row counts (masked dispatch).
    ``out``, ``scales`` and ``masked_m`` must be contiguous: the kernel addresses
    each densely.  With the column-wise layouts ("col", "packed") ``scales`` may
    also be the [.., M_pad, columns] transposed view of its contiguous plane; any
    other non-contiguous view raises.  The call runs with ``x``'s device current,
    whichever device is current in the caller.
    NVFP4 is ``out_dtype="e2m1", scale_fmt="e4m3", group=16`` with
    ``global_scale`` a one-element fp32 CUDA tensor (pqg_quant_nvfp4).
    The kernel runs on ``stream`` (default: torch's current stream).
    """
    import torch
    if x.dtype == torch.bfloat16:
        in_dtype = PQG_BF16
    elif x.dtype == torch.float16:
        in_dtype = PQG_FP16
    else:
        raise TypeError(f"unsupported input dtype {x.dtype}")
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    E = num_experts if num_experts is not None else (x.shape[0] if x.dim() == 3 else 1)
    width = x.shape[-1]
    K = K if K is not None else (width // 2 if fuse_silu_mul else width)
    M = M if M is not None else x.numel() // (E * width)
    if out is None or scales is None:
        o, s = allocate_outputs(M, K, group, num_experts=E, out_dtype=out_dtype,
                                scale_fmt=scale_fmt, layout=layout, device=x.device)
        out = o if out is None else out
        scales = s if scales is None else scales
    odt = {"e4m3": torch.float8_e4m3fn, "int8": torch.int8, "e2m1": torch.uint8}[out_dtype]
    out_bytes = E * M * (K // 2 if out_dtype == "e2m1" else K)
    if x.numel() != E * M * width:
        raise ValueError("x does not hold E x M rows of the given width")
    if out.numel() * out.element_size() != out_bytes or out.dtype not in (odt, torch.uint8):
        raise ValueError(f"out must hold {out_bytes} bytes of codes")
    nbytes = pqg_scales_bytes(E, M, K, group, SCALE_FMTS[scale_fmt], LAYOUTS[layout])
    if nbytes >= 0 and scales.numel() * scales.element_size() != nbytes:
        raise ValueError(f"scales must be {nbytes} bytes for this layout")
    if not (out.is_cuda and scales.is_cuda and out.device == x.device == scales.device):
        raise ValueError("x, out and scales must be on the same CUDA device")
    # the kernel addresses every buffer from its first byte, densely
    if not out.is_contiguous():
        raise ValueError("out must be contiguous")
    if not scales.is_contiguous():
        # only a column-wise layout can be handed over as its [.., M_pad, columns]
        # transposed view; its underlying buffer must be the dense plane
        ng = K // group
        cols = {"col": ng, "packed": (ng + 3) // 4}.get(layout)
        if (cols is None or scales.dim() < 2 or not scales.transpose(-1, -2).is_contiguous()
                or scales.shape[-1] != cols or scales.shape[-2] != (M + 3) // 4 * 4):
            raise ValueError(f"a non-contiguous scales view must be the transposed "
                             f"[M_pad, groups] view of a contiguous '{layout}' plane; "
                             f"layout '{layout}' does not match this view")
    mm_ptr = None
    if masked_m is not None:
        if (masked_m.dtype != torch.int32 or masked_m.device != x.device
                or masked_m.numel() != E or not masked_m.is_contiguous()):
            raise ValueError("masked_m must be a contiguous int32 CUDA tensor with one entry "
                             "per expert")
        mm_ptr = masked_m.data_ptr()
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    # the library sizes its grid from, and launches on, the current device
    with torch.cuda.device(x.device):
        return _launch(x, out, scales, M, E, K, group, in_dtype, out_dtype, scale_fmt, layout,
                       fuse_silu_mul, mm_ptr, expected_m, global_scale, stream)


def _launch(x, out, scales, M, E, K, group, in_dtype, out_dtype, scale_fmt, layout,
            fuse_silu_mul, mm_ptr, expected_m, global_scale, stream):
    import torch
    if scale_fmt == "e4m3":
        if (global_scale is None or global_scale.dtype != torch.float32
                or global_scale.numel() != 1 or global_scale.device != x.device):
            raise ValueError("NVFP4 needs global_scale: a one-element fp32 tensor on x's device")
        if out_dtype != "e2m1" or group != 16:
            raise ValueError("scale_fmt='e4m3' is NVFP4: out_dtype='e2m1', group=16")
        st = pqg_quant_nvfp4(x.data_ptr(), out.data_ptr(), scales.data_ptr(),
                             global_scale.data_ptr(), M, E, K, in_dtype, LAYOUTS[layout],
                             int(bool(fuse_silu_mul)), mm_ptr, int(expected_m),
                             getattr(stream, "cuda_stream", stream))
        if st != PQG_OK:
            raise PqgError(st, "pqg_quant_nvfp4")
        return out, scales
    st = pqg_quant(x.data_ptr(), out.data_ptr(), scales.data_ptr(), M, E, K, group, in_dtype,
                   OUT_DTYPES[out_dtype], SCALE_FMTS[scale_fmt], LAYOUTS[layout],
                   int(bool(fuse_silu_mul)), mm_ptr, int(expected_m),
                   getattr(stream, "cuda_stream", stream))
    if st != PQG_OK:
        raise PqgError(st)
    return out, scales


def quant_varlen(x, seg_indptr, seg_lens=None, out=None, scales=None, *, group: int = 128,
                 out_dtype: str = "e4m3", scale_fmt: str = "fp32", layout: str = "row",
                 fuse_silu_mul: bool = False, expected_m: int = 0, global_scale=None,
                 stream=None):
    """Grouped-contiguous (varlen) quantization of packed token rows; returns
    (out, scales).

    ``x`` is a contiguous bf16/fp16 CUDA tensor [M, K] ([M, 2K] when
    ``fuse_silu_mul``) holding the segments of all experts.  ``seg_indptr`` is
    an int32 CUDA tensor of E + 1 row offsets and ``seg_lens`` one of E token
    counts (or None: every row of a segment is a token).  Token rows are
    quantized into the same rows of ``out`` and of one scale plane of M rows;
    padding rows are left as they are (``torch.empty`` when allocated here).
    NVFP4 is ``out_dtype="e2m1", scale_fmt="e4m3", group=16`` with
    ``global_scale``.  The call runs with ``x``'s device current.
    """
    import torch
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError(f"unsupported input dtype {x.dtype}")
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 2:
        raise ValueError("x must be a contiguous 2-D CUDA tensor of packed rows")
    M, width = x.shape
    K = width // 2 if fuse_silu_mul else width
    E = seg_indptr.numel() - 1
    for name, t, n in (("seg_indptr", seg_indptr, E + 1), ("seg_lens", seg_lens, E)):
        if t is None:
            continue
        if (t.dtype != torch.int32 or t.device != x.device or t.numel() != n
                or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous int32 tensor of {n} entries on "
                             f"x's device")
    if E < 1:
        raise ValueError("seg_indptr needs at least two entries")
    if out is None or scales is None:
        o, sc = allocate_outputs(M, K, group, out_dtype=out_dtype, scale_fmt=scale_fmt,
                                 layout=layout, device=x.device)
        out = o[0] if out is None else out
        scales = sc[0] if scales is None else scales
    out_bytes = M * (K // 2 if out_dtype == "e2m1" else K)
    if out.numel() * out.element_size() != out_bytes or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous buffer of {out_bytes} bytes")
    nbytes = pqg_scales_bytes(1, M, K, group, SCALE_FMTS[scale_fmt], LAYOUTS[layout])
    if (nbytes >= 0 and scales.numel() * scales.element_size() != nbytes) \
            or not scales.is_contiguous():
        raise ValueError(f"scales must be a contiguous buffer of {nbytes} bytes")
    if not (out.device == scales.device == x.device):
        raise ValueError("x, out and scales must be on the same CUDA device")
    gptr = None
    if scale_fmt == "e4m3":
        if (global_scale is None or global_scale.dtype != torch.float32
                or global_scale.numel() != 1 or global_scale.device != x.device):
            raise ValueError("NVFP4 needs global_scale: a one-element fp32 tensor on x's device")
        gptr = global_scale.data_ptr()
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    in_dtype = PQG_BF16 if x.dtype == torch.bfloat16 else PQG_FP16
    with torch.cuda.device(x.device):
        st = pqg_quant_varlen(x.data_ptr(), out.data_ptr(), scales.data_ptr(), gptr, M, E, K,
                              group, in_dtype, OUT_DTYPES[out_dtype], SCALE_FMTS[scale_fmt],
                              LAYOUTS[layout], int(bool(fuse_silu_mul)), seg_indptr.data_ptr(),
                              None if seg_lens is None else seg_lens.data_ptr(),
                              int(expected_m), getattr(stream, "cuda_stream", stream))
    if st != PQG_OK:
        raise PqgError(st, "pqg_quant_varlen")
    return out, scales
