/*
 * pqg — per-token-group activation quantization for NVIDIA B200 (sm_100a).
 *
 * C ABI of libpqg.so.  Plain pointers and sizes only; every buffer is owned by
 * the caller, the library allocates no device or host memory, never
 * synchronizes, and runs asynchronously on the stream it is given.
 *
 * The operation (sglang PR #30924 report, "[JIT] Trait-driven
 * per_token_group_quant: unify the quant kernel family (flat + masked)"):
 *   - 实现拆解 item 1 names the variant axes: input dtype (bf16/fp16), output
 *     dtype (FP8-E4M3/INT8), group size, fp32 or UE8M0 scales, row- or
 *     column-major scale layout, an optional fused silu_and_mul, and flat or
 *     masked dispatch;
 *   - 实现拆解 item 2 gives the masked dispatch its inputs masked_m and
 *     expected_m;
 *   - 关键源码片段, ref_fp8_ue8m0, gives the arithmetic: the absmax of each
 *     1 x G group is floored at EPS; scale = amax / 448, or for UE8M0 the
 *     power of two 2^e with e = biased exponent of fp32(amax / 448), plus one
 *     when that quotient's mantissa is nonzero; codes = saturating cast of
 *     x / scale clamped to [-448, 448];
 *   - 风险与影响 (int8 码位差异) gives the INT8 variant with scale = amax / 127;
 *     the same passage notes that callers no longer pass eps / min / max.
 * The "FlashInfer GEMM 学习笔记" page (§6-7) states what the consumers of
 * these codes want: block-scaled GEMMs read TMA-aligned packed scales, and
 * grouped-masked GEMMs take a fixed expected_m plus a per-expert masked_m.
 * "tf-kernel 安装与使用" (TeleFuser, 使用示例) splits a silu_and_mul input
 * row into two halves of equal width.
 *
 * Numerics (every rounding to nearest, ties to even; no fast-math):
 *   amax = max(max_i |x_i|, 1e-10f)                     (fp32)
 *   FP32 scales : s = amax / 448 (E4M3) or amax / 127 (INT8), one IEEE division
 *   UE8M0 scales: r = amax / 448; e = ((bits(r) >> 23) & 0xFF)
 *                                     + ((bits(r) & 0x7FFFFF) != 0);
 *                 s = 2^(e - 127); the stored byte is e
 *   codes       : t = fp32(x / s) rounded once; E4M3 = nearest OCP E4M3 ("fn")
 *                 value of t clamped to +-448 (zero keeps t's sign);
 *                 INT8 = nearest integer of t clamped to [-128, 127]
 *   fused       : x = silu(gate) * up computed in fp32 registers, gate being
 *                 the first K columns of a 2K-wide input row, up the second;
 *                 the product is never written to memory
 * Codes and scales are bit-identical to that definition for every non-fused
 * call.  The fused prologue uses the GPU's fast exponential, so its codes may
 * move by one step where silu(gate)*up lies within a few fp32 ulps of a
 * rounding midpoint.
 */
#ifndef PQG_H
#define PQG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point below is exported from libpqg.so; nothing else is. */
#if defined(__GNUC__)
#define PQG_API __attribute__((visibility("default")))
#else
#define PQG_API
#endif

/* Same type as cudaStream_t / CUstream.  NULL means the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st *pqg_stream_t;

/* Status codes.  Every error is detected on the host before anything is
 * launched, except PQG_ERR_CUDA, which reports a failed launch. */
enum pqg_status {
    PQG_OK = 0,
    PQG_ERR_INVALID_ARG = -1, /* null pointer, bad size, unknown enum value     */
    PQG_ERR_UNSUPPORTED = -2, /* valid values that do not combine (see below)  */
    PQG_ERR_ALIGNMENT = -3,   /* a pointer misses its required alignment       */
    PQG_ERR_CUDA = -4         /* the CUDA runtime reported an error; see
                                 pqg_last_cuda_error()                          */
};

/* Element types. */
enum pqg_dtype {
    PQG_BF16 = 0, /* input: bfloat16                                  */
    PQG_FP16 = 1, /* input: IEEE binary16                             */
    PQG_E4M3 = 2, /* output: OCP FP8 E4M3 "fn" (max 448, no inf)       */
    PQG_INT8 = 3, /* output: two's-complement int8                    */
    PQG_E2M1 = 4  /* output: OCP FP4 E2M1 (max 6), two codes per byte,
                     element 2i in bits 0-3 and 2i+1 in bits 4-7 (MXFP4) */
};

/* Scale formats. */
enum pqg_scale_fmt {
    PQG_SCALE_FP32 = 0,  /* one float per group                        */
    PQG_SCALE_UE8M0 = 1, /* one biased exponent byte e, scale 2^(e-127) */
    PQG_SCALE_E4M3 = 2   /* one OCP E4M3 byte per block of 16 (NVFP4,
                            pqg_quant_nvfp4 only)                       */
};

/* Scale layouts, per expert.  ng = K / group; M_pad = M rounded up to a
 * multiple of 4 (so that every column of the plane starts on a 16-byte
 * boundary for fp32 scales and packed words).
 *   PQG_ROW_MAJOR     : S[m][g]           element (m * ng + g)
 *   PQG_COL_MAJOR_TMA : S[g][m]           element (g * M_pad + m); rows
 *                       M..M_pad-1 are padding and are never written
 *   PQG_UE8M0_PACKED  : W[j][m], int32    word (j * M_pad + m), j < ceil(ng/4);
 *                       byte b (little-endian) of W[j][m] holds the exponent of
 *                       group 4j + b; bytes for groups >= ng are written 0.
 *                       UE8M0 only ("aligned" in the pages' trait list means
 *                       ng % 4 == 0, i.e. no partial last word).
 *   PQG_UE8M0_TILED_128x4 : the 128x4 block-scale tile ("F8_128x4", the 1D
 *                       swizzled layout the FlashInfer notes name for mm_mxfp8,
 *                       section 6).  Rows in tiles of 128, groups in tiles of 4;
 *                       one 512-byte tile per (row tile, group tile), tiles in
 *                       row-tile-major order; inside a tile the exponent of
 *                       (row m, group g) is byte (m%32)*16 + ((m/32)%4)*4 + g%4.
 *                       Plane: ceil(M/128)*128 x ceil(ng/4)*4 bytes.  Bytes of
 *                       padding groups (>= ng) in a quantized row are written 0;
 *                       padding rows are not written.  UE8M0 bytes (with G = 32
 *                       the MXFP8 operand format) or, through pqg_quant_nvfp4,
 *                       E4M3 block-scale bytes (the NVFP4 operand format).
 * Expert e's plane starts pqg_scales_bytes(1, M, K, ...) * e bytes into the
 * buffer. */
enum pqg_scale_layout {
    PQG_ROW_MAJOR = 0,
    PQG_COL_MAJOR_TMA = 1,
    PQG_UE8M0_PACKED = 2,
    PQG_UE8M0_TILED_128x4 = 3
};

/*
 * pqg_quant — quantize num_experts x M rows of K outputs each.
 *
 * in       device, read-only.  [num_experts][M][K] elements of in_dtype, or
 *          [num_experts][M][2K] when fuse_silu_mul (row = gate | up).  Rows are
 *          dense (row stride = K or 2K elements).  32-byte aligned.
 * out      device.  [num_experts][M][K] one-byte codes (E4M3 or INT8), or
 *          [num_experts][M][K/2] bytes of E2M1 code pairs.  16-byte aligned.
 * scales   device.  pqg_scales_bytes(num_experts, M, K, group, scale_fmt,
 *          scale_layout) bytes in the chosen layout.  4-byte aligned for fp32
 *          scales, packed words and the 128x4 tiled layout; any alignment for
 *          row- or column-major UE8M0 bytes.
 * M        rows per expert (with masked_m: the capacity M_max of each expert).
 *          M >= 0; M == 0 launches nothing.
 * num_experts  1 ..= 4096.  With masked_m == NULL every expert's M rows
 *          are quantized (num_experts == 1 is the flat dispatch).
 * K        output elements per row, a positive multiple of group.
 * group    G in {32, 64, 128}, or G == K for one scale per row (per-token
 *          quantization, as tf_per_token_quant_fp8 on the TeleFuser page;
 *          K a multiple of 16, at most 16384).
 * in_dtype PQG_BF16 or PQG_FP16.   out_dtype PQG_E4M3, PQG_INT8 or PQG_E2M1.
 *          PQG_E2M1 (MXFP4: "block_size = 32 -> MXFP4" in the FlashInfer notes,
 *          section 6) needs PQG_SCALE_UE8M0 and G in {32, 64, 128}; its scale
 *          is 2^ceil(log2(amax / 6)) by the same bit rule with FMAX = 6.
 * scale_fmt, scale_layout   see above.  PQG_SCALE_UE8M0 rejects PQG_INT8, and
 *          PQG_UE8M0_PACKED and PQG_UE8M0_TILED_128x4 require PQG_SCALE_UE8M0
 *          (else PQG_ERR_UNSUPPORTED).  PQG_SCALE_E4M3 needs a global scale:
 *          pqg_quant returns PQG_ERR_UNSUPPORTED for it (see pqg_quant_nvfp4).
 * fuse_silu_mul  nonzero: quantize silu(gate) * up (see the numerics above).
 * masked_m device, int32[num_experts], or NULL.  Masked dispatch (grouped-masked
 *          MoE): expert e quantizes only rows m < clamp(masked_m[e], 0, M); the
 *          codes and scales of every other row are left untouched.  Read on the
 *          device, so it may be produced by the preceding kernel on `stream`.
 * expected_m  a hint for the masked grid: the typical masked_m value.  Results
 *          never depend on it; <= 0 or > M means M.  Ignored when masked_m is
 *          NULL.  A fused masked call with at most 32 experts and
 *          1 <= expected_m <= 8 (decode) reads each expert's first
 *          min(expected_m, M) input rows while masked_m is still in flight;
 *          rows past masked_m among them are read but never written.
 * stream   CUDA stream the kernel is launched on.  The launch carries the
 *          programmatic-dependent-launch attribute (see pqg_set_pdl); the kernel
 *          waits for the preceding grid before its first global-memory access.
 *
 * Returns PQG_OK, or a negative pqg_status with nothing launched (except
 * PQG_ERR_CUDA).  Limits: K <= 2^28, num_experts * M * ceil(K / 512) < 2^31
 * and num_experts * M * K <= 2^40 (else PQG_ERR_INVALID_ARG).
 * The output and scale buffers must not overlap the input.
 */
PQG_API int pqg_quant(const void *in, void *out, void *scales, int64_t M,
              int64_t num_experts, int64_t K, int group, int in_dtype,
              int out_dtype, int scale_fmt, int scale_layout, int fuse_silu_mul,
              const int32_t *masked_m, int64_t expected_m, pqg_stream_t stream);

/*
 * pqg_quant_nvfp4 — NVFP4 quantization ("block_size = 16 -> NVFP4", FlashInfer
 * GEMM notes, section 6): E2M1 codes in blocks of 16 with an E4M3 block scale
 * under a per-call fp32 global scale g.  The pages give only the block size;
 * the arithmetic below is this library's reading of the two-level NVFP4 scale.
 * Per block, in fp32 with round-to-nearest-even:
 *   amax = max(max_i |x_i|, 1e-10f)
 *   r    = (amax / 6) * g           two roundings, in this order
 *   sf   = nearest E4M3 code of r, saturating at 448       (the stored byte)
 *   mult = g / value(sf), or 0 when value(sf) == 0
 *   code = nearest E2M1 value of x_i * mult, saturating at +-6 (zero keeps
 *          the sign of the product)
 * so x_i is approximately code * value(sf) / g.  Bit-identical to that
 * definition for every non-fused call; the fused prologue follows pqg_quant's
 * note.
 *
 * in, M, num_experts, in_dtype, fuse_silu_mul, masked_m, expected_m, stream:
 *          as for pqg_quant.
 * out      device.  [num_experts][M][K/2] bytes, two E2M1 codes per byte,
 *          element 2i in bits 0-3.  16-byte aligned.
 * scales   device.  pqg_scales_bytes(num_experts, M, K, 16, PQG_SCALE_E4M3,
 *          scale_layout) bytes: one E4M3 byte per block in PQG_ROW_MAJOR,
 *          PQG_COL_MAJOR_TMA or PQG_UE8M0_TILED_128x4 (the 128x4 tile holds
 *          E4M3 bytes here); PQG_UE8M0_PACKED is rejected (PQG_ERR_UNSUPPORTED).
 * global_scale  device, one fp32 g, finite and > 0 (else the codes are
 *          unspecified; nothing faults).  Read on the device after the
 *          programmatic-dependent-launch wait, so the preceding kernel on
 *          `stream` may produce it (typically 448 * 6 / amax of the tensor).
 *          4-byte aligned.
 * K        a positive multiple of 16.
 * Same limits and return codes as pqg_quant.
 */
PQG_API int pqg_quant_nvfp4(const void *in, void *out, void *scales,
              const float *global_scale, int64_t M, int64_t num_experts, int64_t K,
              int in_dtype, int scale_layout, int fuse_silu_mul,
              const int32_t *masked_m, int64_t expected_m, pqg_stream_t stream);

/*
 * pqg_quant_varlen — grouped-contiguous (varlen) dispatch: the tokens of
 * num_experts segments packed in one buffer of M rows, as a grouped-contiguous
 * MoE GEMM reads them.  The sglang PR #30924 report (实现拆解 item 4) has the
 * varlen DeepGEMM caller (_varlen_deep_gemm_silu_mul_quant) quantize through
 * per_token_group_quant; "FlashInfer GEMM 学习笔记" section 7 describes the
 * packed-token form (GroupedContiguous: packed tokens + m_indices; segments
 * mapped by seg_lens / seg_indptr).  The pages give no arithmetic for the
 * segments; this library's reading:
 *   segment e spans rows [seg_indptr[e], seg_indptr[e+1]), both ends clamped
 *   into [0, M] and the end no lower than the start; its first seg_lens[e]
 *   rows, clamped into the segment (every row when seg_lens is NULL), are
 *   tokens, and the rest is padding (a grouped-contiguous GEMM pads each
 *   expert's segment to its M block).
 * Token rows are quantized exactly as a flat pqg_quant call over the M rows
 * would quantize them: codes in the same row of `out`, scales in the same row
 * of ONE scale plane of M rows.  Padding rows, and rows in no segment, are not
 * read and not written.  Segments that overlap write the same bytes twice.
 *
 * in       device, read-only.  [M][K] (or [M][2K] when fuse_silu_mul) packed
 *          rows of in_dtype.  32-byte aligned.
 * out      device.  [M][K] code bytes ([M][K/2] for E2M1).  16-byte aligned.
 * scales   device.  pqg_scales_bytes(1, M, K, group, scale_fmt, scale_layout)
 *          bytes: one plane over the M packed rows in the chosen layout.
 * global_scale  device fp32 g when scale_fmt is PQG_SCALE_E4M3 (NVFP4: group
 *          16, out_dtype PQG_E2M1; as in pqg_quant_nvfp4), else NULL
 *          (PQG_ERR_INVALID_ARG otherwise).
 * M        packed rows (M >= 0; M == 0 launches nothing).
 * num_experts  segments, 1 ..= 4096.
 * K, group, in_dtype, out_dtype, scale_fmt, scale_layout, fuse_silu_mul:
 *          as for pqg_quant (and pqg_quant_nvfp4 for PQG_SCALE_E4M3).
 * seg_indptr  device int32[num_experts + 1], 4-byte aligned; must not be NULL.
 * seg_lens device int32[num_experts] token counts, 4-byte aligned, or NULL.
 *          Both are read on the device after the programmatic-dependent-launch
 *          wait, so the preceding kernel on `stream` may produce them; neither
 *          may overlap `out` or `scales`.
 * expected_m  a hint for the grid: the typical token count of a segment
 *          (num_experts * expected_m tokens in all).  Results never depend on
 *          it; <= 0 or > M means M tokens.
 * stream   as for pqg_quant.
 *
 * Returns PQG_OK or a negative pqg_status with nothing launched (except
 * PQG_ERR_CUDA).  Limits: those of pqg_quant with one expert of M rows.
 */
PQG_API int pqg_quant_varlen(const void *in, void *out, void *scales,
              const float *global_scale, int64_t M, int64_t num_experts, int64_t K,
              int group, int in_dtype, int out_dtype, int scale_fmt, int scale_layout,
              int fuse_silu_mul, const int32_t *seg_indptr, const int32_t *seg_lens,
              int64_t expected_m, pqg_stream_t stream);

/*
 * pqg_scales_bytes — size in bytes of the scale buffer pqg_quant (or, for
 * PQG_SCALE_E4M3 with group 16, pqg_quant_nvfp4) writes for these arguments
 * (all experts, padding rows included).  Returns a negative pqg_status for
 * arguments the call would reject.
 */
PQG_API int64_t pqg_scales_bytes(int64_t num_experts, int64_t M, int64_t K, int group,
                         int scale_fmt, int scale_layout);

/* Static, human-readable text for a status code. */
PQG_API const char *pqg_status_string(int status);

/* The cudaError_t of the last PQG_ERR_CUDA returned on the calling thread
 * (0 if none). */
PQG_API int pqg_last_cuda_error(void);

/* Programmatic dependent launch (PDL) on (nonzero, the default) or off for
 * later pqg_quant calls of this process.  Returns the previous setting. */
PQG_API int pqg_set_pdl(int enable);

/* Number of kernels this process has launched through pqg_quant,
 * pqg_quant_nvfp4 and pqg_quant_varlen so far. */
PQG_API uint64_t pqg_launch_count(void);

/* Library version string, e.g. "pqg 0.1.0 sm_100a". */
PQG_API const char *pqg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PQG_H */
