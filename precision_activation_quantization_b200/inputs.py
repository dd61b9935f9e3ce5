"""Seeded synthetic inputs for per-token-group quantization.

This module only draws numbers.  It holds none of the quantization arithmetic,
and both the CUDA-path tests and the CPU oracle read their inputs from it.

Everything is returned as raw 16-bit patterns (``np.uint16``) because that is
what both sides take.  bf16 values come from fp32 draws rounded to nearest-even
by torch's CPU cast, and fp16 values from numpy's cast, which also rounds to
nearest-even.

The workloads take their shapes from the sglang PR #30924 report,
"[JIT] Trait-driven per_token_group_quant".  Its 关键文件 section says the
benchmarks cover DeepSeek-V3/V4 shapes.  Hidden 7168 and MoE intermediate 2048
are DeepSeek-V3's sizes, and the flat/fused/masked modes come from 实现拆解
items 1-2.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import os

import numpy as np
import torch

# Draws are made in fixed chunks, each from its own generator seeded by
# (seed, chunk index), so the values do not depend on how many threads run.
_CHUNK = 1 << 22


def bf16_bits(f32: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f16_bits(f32: np.ndarray) -> np.ndarray:
    """fp32 array -> fp16 bit patterns (round to nearest even)."""
    return np.ascontiguousarray(f32, dtype=np.float32).astype(np.float16).view(np.uint16)


def to_bits(f32: np.ndarray, in_dtype: str) -> np.ndarray:
    return f16_bits(f32) if in_dtype == "fp16" else bf16_bits(f32)


def _chunked(shape, seed: int, fill) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), np.float32)
    n_chunks = (out.size + _CHUNK - 1) // _CHUNK

    def work(i):
        rng = np.random.default_rng([seed, i])
        fill(rng, out[i * _CHUNK:(i + 1) * _CHUNK])

    if n_chunks <= 1:
        for i in range(n_chunks):
            work(i)
    else:
        with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(n_chunks)))
    return out.reshape(shape)


def normal(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    def fill(rng, view):
        rng.standard_normal(out=view, dtype=np.float32)
        if scale != 1.0:
            view *= np.float32(scale)
    return _chunked(shape, seed, fill)


def laplace(shape, seed: int) -> np.ndarray:
    """Laplace(0, 1) draws by the inverse CDF of seeded uniforms."""
    def fill(rng, view):
        u = rng.random(size=view.size, dtype=np.float64) - 0.5
        view[:] = -np.sign(u) * np.log1p(-2.0 * np.abs(u))
    return _chunked(shape, seed, fill)


@dataclasses.dataclass
class Workload:
    """One synthetic call: inputs plus every argument of the quantization."""
    name: str
    x: np.ndarray            # uint16 patterns, [E, M, K] or [E, M, 2K] when fused
    M: int                   # rows (rows per expert when masked)
    K: int                   # output width
    group: int = 128
    E: int = 1
    in_dtype: str = "bf16"
    out_dtype: str = "e4m3"
    scale_fmt: str = "fp32"
    layout: str = "row"
    fused: bool = False
    masked_m: np.ndarray | None = None   # int32 [E] or None (flat)
    expected_m: int = 0
    global_scale: float | None = None    # NVFP4 (scale_fmt "e4m3") only
    # grouped-contiguous (varlen) calls: E == 1 plane of M packed rows holding
    # len(seg_indptr) - 1 segments; seg_lens are token counts (or None)
    seg_indptr: np.ndarray | None = None
    seg_lens: np.ndarray | None = None

    @property
    def segments(self) -> int:
        return 0 if self.seg_indptr is None else len(self.seg_indptr) - 1

    @property
    def rows(self) -> int:
        """Rows actually quantized (tokens).  For varlen calls this counts
        the tokens of well-formed segments (increasing offsets within the M
        rows, counts within each segment), the only kind generated here."""
        if self.seg_indptr is not None:
            if self.seg_lens is None:
                return int(self.seg_indptr[-1] - self.seg_indptr[0])
            return int(np.asarray(self.seg_lens, np.int64).sum())
        if self.masked_m is None:
            return self.E * self.M
        return int(np.clip(self.masked_m, 0, self.M).sum())

    def algorithmic_bytes(self) -> int:
        """Bytes the call must move: read inputs, write codes and scales.

        Rows at or past masked_m and the padding rows of column-major scale
        planes are excluded; masked_m itself is counted when present.
        """
        ng = self.K // self.group
        in_row = (2 if self.fused else 1) * self.K * 2
        out_row = self.K // 2 if self.out_dtype == "e2m1" else self.K
        if self.layout in ("packed", "tile128x4"):
            scale_row = 4 * ((ng + 3) // 4)
        else:
            scale_row = ng * (4 if self.scale_fmt == "fp32" else 1)
        extra = 0 if self.masked_m is None else 4 * self.E
        if self.seg_indptr is not None:
            extra += 4 * len(self.seg_indptr) + (0 if self.seg_lens is None
                                                 else 4 * len(self.seg_lens))
        if self.global_scale is not None:
            extra += 4                   # the fp32 global scale
        return self.rows * (in_row + out_row + scale_row) + extra

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# --------------------------------------------------------------------------
# The five workloads
# --------------------------------------------------------------------------

def tiny(seed: int = 0) -> Workload:
    """flat, x ~ N(0,1) [4, 256], G=128, E4M3, fp32 row-major scales."""
    x = bf16_bits(normal((1, 4, 256), seed))
    return Workload("tiny", x, M=4, K=256)


def flat_hidden(M: int = 8192, K: int = 7168, seed: int = 1, outlier_seed: int = 2,
                layout: str = "packed", scale_fmt: str = "ue8m0") -> Workload:
    """Flat quant of a DeepSeek-V3 hidden state.

    x ~ N(0,1) [M, K].  0.1% of entries, at uniform positions drawn from
    ``outlier_seed``, are multiplied by 200.  Each block of 128 rows has one
    all-zero group: in block b it is row 128b + (37b mod 128), group b mod
    (K/128).  The defaults give the UE8M0 packed column-major variant; the
    fp32 row-major variant is ``flat_hidden(layout="row", scale_fmt="fp32")``.
    """
    x = normal((M, K), seed)
    rng = np.random.default_rng(outlier_seed)
    n_out = max(1, (M * K) // 1000)
    pos = rng.integers(0, M * K, size=n_out)
    x.reshape(-1)[pos] *= np.float32(200.0)
    ng = K // 128
    for b in range((M + 127) // 128):
        row = 128 * b + (37 * b) % 128
        if row < M:
            g = b % ng
            x[row, g * 128:(g + 1) * 128] = 0.0
    return Workload(f"flat_{M}x{K}", bf16_bits(x).reshape(1, M, K), M=M, K=K,
                    scale_fmt=scale_fmt, layout=layout)


def fused(M: int = 4096, K: int = 2048, seed: int = 3) -> Workload:
    """Fused SiLU-and-mul + quant: [M, 2K] rows, gate = 3*N(0,1) | up = N(0,1)."""
    x = normal((M, 2 * K), seed)
    x[:, :K] *= np.float32(3.0)
    return Workload(f"fused_{M}x2x{K}", bf16_bits(x).reshape(1, M, 2 * K), M=M, K=K,
                    scale_fmt="ue8m0", layout="col", fused=True)


def masked(E: int = 32, M_max: int = 2048, K: int = 2048, seed: int = 4,
           count_seed: int = 5, decode: bool = False, decode_seed: int = 6) -> Workload:
    """Masked MoE dispatch with the fused prologue.

    x: [E, M_max, 2K] gate|up ~ N(0,1).  masked_m[e] ~ U{0..M_max}
    (``count_seed``), expected_m = mean rounded up.  The decode variant has
    masked_m[e] in {0, 1} (``decode_seed``) and expected_m = 1.
    """
    x = bf16_bits(normal((E, M_max, 2 * K), seed))
    if decode:
        mm = np.random.default_rng(decode_seed).integers(0, 2, size=E).astype(np.int32)
        expected = 1
    else:
        mm = np.random.default_rng(count_seed).integers(0, M_max + 1, size=E).astype(np.int32)
        expected = max(1, int(np.ceil(mm.mean())))
    name = f"masked{'_decode' if decode else ''}_{E}x{M_max}x2x{K}"
    return Workload(name, x, M=M_max, K=K, E=E, scale_fmt="ue8m0", layout="col",
                    fused=True, masked_m=mm, expected_m=expected)


def mxfp4(M: int = 8192, K: int = 7168, seed: int = 1) -> Workload:
    """The flat hidden-state input as an MXFP4 operand: G = 32, E2M1 codes, UE8M0
    scales in the 128x4 tiled layout."""
    w = flat_hidden(M=M, K=K, seed=seed)
    return w.with_(name=f"mxfp4_{M}x{K}", group=32, out_dtype="e2m1", layout="tile128x4")


# 448 * 6 / 1024: the global scale of a tensor whose absmax is about 1024 (the
# hidden-state input's x200 outliers reach a few hundred to about a thousand)
NVFP4_GLOBAL_SCALE = 2.625


def nvfp4(M: int = 8192, K: int = 7168, seed: int = 1,
          global_scale: float = NVFP4_GLOBAL_SCALE) -> Workload:
    """The flat hidden-state input as an NVFP4 operand: blocks of 16, E2M1 codes,
    E4M3 block scales in the 128x4 tiled layout, a fixed fp32 global scale."""
    w = flat_hidden(M=M, K=K, seed=seed)
    return w.with_(name=f"nvfp4_{M}x{K}", group=16, out_dtype="e2m1", scale_fmt="e4m3",
                   layout="tile128x4", global_scale=global_scale)


def sweep(M: int, K: int = 4096, in_dtype: str = "bf16", group: int = 128,
          out_dtype: str = "e4m3", seed: int | None = None) -> Workload:
    """dtype/size sweep: x ~ Laplace(0,1) [M, K], fp32 row-major scales."""
    seed = 7 + M if seed is None else seed
    x = to_bits(laplace((M, K), seed), in_dtype).reshape(1, M, K)
    return Workload(f"sweep_{in_dtype}_{out_dtype}_g{group}_{M}x{K}", x, M=M, K=K,
                    group=group, in_dtype=in_dtype, out_dtype=out_dtype)


def varlen(E: int = 32, M_max: int = 2048, K: int = 2048, seed: int = 4, count_seed: int = 5,
           align: int = 128) -> Workload:
    """Grouped-contiguous (varlen) dispatch with the fused prologue: the masked
    workload's experts and token counts (masked_m[e] ~ U{0..M_max}, seed
    ``count_seed``), packed into one buffer of [gate | up] rows whose segment e
    holds its tokens followed by padding up to a multiple of ``align`` rows (the
    M-block padding of a grouped-contiguous GEMM).  Tokens ~ N(0,1) ([seed]);
    padding rows hold N(0,1) draws too (a consumer never reads them).
    expected_m = the mean count rounded up."""
    lens = np.random.default_rng(count_seed).integers(0, M_max + 1, size=E).astype(np.int32)
    caps = -(-lens // align) * align
    indptr = np.concatenate([[0], np.cumsum(caps)]).astype(np.int32)
    M = int(indptr[-1])
    x = bf16_bits(normal((1, M, 2 * K), seed))
    return Workload(f"varlen_{E}x{M_max}x2x{K}", x, M=M, K=K, scale_fmt="ue8m0",
                    layout="col", fused=True, expected_m=max(1, int(np.ceil(lens.mean()))),
                    seg_indptr=indptr, seg_lens=lens)
