/*
 * Scalar CPU oracle for per-token-group activation quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously correct
 * statement of what the quantization path computes.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg load it.  It shares no code,
 * header, table or constant generator with the CUDA library, and the product
 * path never calls it.
 *
 * What it follows (page title, section):
 *   [PR]  sglang PR #30924 report, "[JIT] Trait-driven per_token_group_quant:
 *         unify the quant kernel family (flat + masked)":
 *           - 实现拆解 item 1: the variant axes (input/output dtype, group size,
 *             fp32 or UE8M0 scale, row- or column-major scale layout, fused
 *             silu_and_mul, flat or masked dispatch);
 *           - 实现拆解 item 2: masked dispatch driven by masked_m / expected_m;
 *           - 关键源码片段, ref_fp8_ue8m0: group absmax floored at EPS,
 *             raw = amax / FMAX with FMAX = 448, UE8M0 exponent = biased exponent
 *             of raw plus one when raw's mantissa is nonzero, codes from a
 *             saturating quantize clamped to [-FMAX, FMAX];
 *           - _jit_module snippet: the `aligned` flag (group count a multiple
 *             of 4, UE8M0 only) and the scale layout flags;
 *           - 关键文件 / 风险与影响: the INT8 path (ref_int8) with identical
 *             scales, i.e. scale = amax / 127.
 *   [TF]  "tf-kernel 安装与使用" (TeleFuser), 使用示例: silu_and_mul splits the
 *         last dimension into two halves of equal width.
 *   [FI]  "FlashInfer GEMM 学习笔记", sections 6-7: block-scaled consumers want
 *         TMA-aligned packed scales; grouped-masked GEMMs take a fixed
 *         expected_m plus a per-expert masked_m.
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes):
 *   - EPS = 1e-10f (the snippet names EPS without printing its value).
 *   - gate is the first half of a fused row, up the second half.
 *   - the SiLU-and-mul product is formed in double and rounded once to fp32;
 *     it is never rounded to the input dtype.
 *   - every rounding is to nearest, ties to even; E4M3 is the OCP "fn"
 *     variant (no infinities, 448 largest finite), zero keeps the sign of t.
 *   - FP4 (MXFP4, the FlashInfer notes' "block_size = 32 -> MXFP4"): OCP E2M1
 *     codes (largest magnitude 6), UE8M0 scales by the same rule with FMAX = 6,
 *     two codes per byte with element 2i in bits 0-3 and 2i+1 in bits 4-7.
 *   - NVFP4 (the FlashInfer notes' "block_size = 16 -> NVFP4", section 6):
 *     E2M1 codes in blocks of 16 with an E4M3 block scale and one fp32
 *     global scale g per call (the encode-side factor, typically
 *     448 * 6 / amax of the tensor).  Per block, in this order and in fp32:
 *     r = (amax / 6) * g; sf = E4M3(r) (nearest, saturating at 448);
 *     d = value of sf; m = g / d (0 when d is 0); t_i = x_i * m; codes =
 *     E2M1(t_i), saturating at 6.  The dequantized value is code * d / g.
 *   - column-major layouts pad the row count to a multiple of 4 (16 bytes of
 *     fp32 or one int32 word per 4 rows), padding rows are never written.
 *   - the UE8M0-packed layout stores the exponents of groups 4j..4j+3 of a
 *     row in one little-endian int32 word; bytes for groups past the last one
 *     are 0.
 *   - the 128x4 tiled layout ("F8_128x4", the 1D swizzled block-scale layout
 *     the FlashInfer notes name for mm_mxfp8, section 6) is read as the public
 *     block-scale tile: rows in tiles of 128, scale columns in tiles of 4, one
 *     512-byte tile per (row tile, column tile) in row-tile-major order, and
 *     inside a tile the exponent of (row m, group g) at byte
 *     (m % 32) * 16 + ((m / 32) % 4) * 4 + (g % 4).  Bytes of padding columns
 *     (groups >= ng) in a quantized row are 0; padding rows are not written.
 *   - grouped-contiguous (varlen) dispatch ([PR] 实现拆解 item 4, the varlen
 *     DeepGEMM caller quantizing through per_token_group_quant; [FI] section 7,
 *     packed tokens of all experts in one buffer, mapped per segment by
 *     seg_indptr / seg_lens): M packed rows hold E segments; segment e spans
 *     rows [indptr[e], indptr[e+1]) (both ends clamped into [0, M], the end no
 *     lower than the start), and its first lens[e] rows (clamped into the
 *     segment; every row when lens is absent) are tokens, the rest padding.
 *     Token rows are quantized exactly as in a flat call over the M rows, with
 *     codes and scales at the same row of one scale plane of M rows; padding
 *     rows are not touched.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no fast-math).
 * Floating point: C float arithmetic is IEEE binary32 with round-to-nearest
 * (FLT_EVAL_METHOD 0 on x86-64 and aarch64); fp-contract is off so no
 * multiply-add is fused behind the reader's back.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- constants of the method (values, not code, shared with nobody) ---- */
#define PQGO_FMAX_E4M3 448.0f   /* largest finite E4M3 value ([PR] FMAX)       */
#define PQGO_FMAX_INT8 127.0f   /* INT8 scale divisor ([PR] ref_int8)          */
#define PQGO_FMAX_E2M1 6.0f     /* largest finite OCP E2M1 value (MXFP4)       */
#define PQGO_EPS 1e-10f         /* absmax floor ([PR] "不低于 EPS")             */
#define PQGO_NVFP4_BLOCK 16     /* NVFP4 block size ([FI] section 6)           */

/* output kinds and layouts understood by the oracle (numbered for the Python
 * wrapper) */
enum { PQGO_OUT_E4M3 = 0, PQGO_OUT_INT8 = 1, PQGO_OUT_E2M1 = 2 };
enum { PQGO_ROW = 0, PQGO_COL = 1, PQGO_PACKED = 2, PQGO_TILE128X4 = 3 };

/* ------------------------------------------------------------------------ */
/* Input decoding                                                            */
/* ------------------------------------------------------------------------ */

/* bfloat16 is the upper 16 bits of an IEEE binary32 (1 sign, 8 exponent,
 * 7 fraction bits), so widening is exact: put the bits back on top. */
static float decode_bf16(uint16_t h) {
    uint32_t w = (uint32_t)h << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Subnormals are m * 2^-24; normals are (1024 + m) * 2^(e - 25). */
static float decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1024.0 + (double)m, e - 25);
    return (float)(sign ? -v : v);
}

float pqgo_decode(uint16_t bits, int in_fp16) {
    return in_fp16 ? decode_f16(bits) : decode_bf16(bits);
}

/* ------------------------------------------------------------------------ */
/* Fused prologue: y = silu(gate) * up, silu(g) = g / (1 + e^-g)  [PR] item 1 */
/* ------------------------------------------------------------------------ */

float pqgo_silu_mul(float gate, float up) {
    double g = (double)gate;
    double silu = g / (1.0 + exp(-g));
    return (float)(silu * (double)up);
}

/* ------------------------------------------------------------------------ */
/* Group statistics and scales                                               */
/* ------------------------------------------------------------------------ */

/* absmax of one group, floored at EPS  ([PR] 关键源码片段, _group_amax) */
float pqgo_group_amax(const float *v, int64_t n) {
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float m = fabsf(v[i]);
        if (m > a) a = m;
    }
    if (a < PQGO_EPS) a = PQGO_EPS;
    return a;
}

/* fp32 scale: amax / 448 for E4M3, amax / 127 for INT8, one IEEE division. */
float pqgo_scale_fp32(float amax, int out_int8) {
    return out_int8 ? amax / PQGO_FMAX_INT8 : amax / PQGO_FMAX_E4M3;
}

/* UE8M0 exponent byte, the pages' steps in their order ([PR] ref_fp8_ue8m0):
 * raw = amax / FMAX in fp32; take raw's biased exponent field; add one when
 * raw's 23-bit mantissa is nonzero (rounds the scale up to a power of two).
 * The scale is 2^(byte - 127). */
int pqgo_ue8m0_exponent_fmax(float amax, float fmax) {
    float raw = amax / fmax;
    uint32_t bits;
    memcpy(&bits, &raw, sizeof bits);
    int biased = (int)((bits >> 23) & 0xFF);
    int bump = (bits & 0x7FFFFF) != 0;
    return biased + bump;
}

int pqgo_ue8m0_exponent(float amax) { return pqgo_ue8m0_exponent_fmax(amax, PQGO_FMAX_E4M3); }

/* ------------------------------------------------------------------------ */
/* Output encoders                                                           */
/* ------------------------------------------------------------------------ */

/* Saturating cast to OCP FP8 E4M3 ("fn": no infinities, S.1111.111 is NaN).
 * Codes: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Normal values
 * are (1 + m/8) * 2^(e - 7) for e = 1..15 (m <= 6 at e = 15, so 448 is the
 * largest finite value); subnormals are (m/8) * 2^-6.  The value is first
 * clamped to [-448, 448] ([PR] _quantize(..., -FMAX, FMAX)), then rounded to
 * the nearest representable magnitude with ties to an even mantissa.  A value
 * that rounds to zero keeps the sign of t. */
uint8_t pqgo_e4m3_encode(float t) {
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    if (a > 448.0) a = 448.0;
    /* spacing of the representable values that bracket a */
    int E = (a >= ldexp(1.0, -6)) ? ilogb(a) : -6;
    double quantum = ldexp(1.0, E - 3);
    double n = nearbyint(a / quantum); /* exact quotient; ties to even */
    double r = n * quantum;            /* may carry into the next binade */
    if (r == 0.0) return sign;
    int Er = ilogb(r);
    if (Er < -6) /* subnormal: r = m * 2^-9, m in 1..7 */
        return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9)));
    {
        int exp_field = Er + 7;
        int mant = (int)(r / ldexp(1.0, Er - 3)) - 8;
        return (uint8_t)(sign | (exp_field << 3) | mant);
    }
}

/* Value of an OCP E4M3 ("fn") code: (1 + m/8) * 2^(e - 7) for exponent
 * field e >= 1, (m/8) * 2^-6 for e = 0; S.1111.111 is NaN. */
float pqgo_e4m3_decode(uint8_t c) {
    int e = (c >> 3) & 0xF, m = c & 0x7;
    double v;
    if (e == 15 && m == 7) return NAN;
    v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)((c & 0x80) ? -v : v);
}

/* Saturating cast to INT8: round to nearest integer, ties to even, then
 * clamp to [-128, 127]. */
int8_t pqgo_int8_encode(float t) {
    double n = nearbyint((double)t);
    if (n > 127.0) n = 127.0;
    if (n < -128.0) n = -128.0;
    return (int8_t)n;
}

/* Saturating cast to OCP FP4 E2M1: sign bit, 2 exponent bits (bias 1), 1
 * mantissa bit.  Normal values (1 + m/2) * 2^(e - 1) for e = 1..3, subnormal
 * m * 0.5; the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  |t| is clamped to
 * 6, then rounded to the nearest magnitude with ties to an even mantissa; a
 * value that rounds to zero keeps the sign of t.  Returns the 4-bit code. */
uint8_t pqgo_e2m1_encode(float t) {
    uint8_t sign = signbit(t) ? 0x8 : 0x0;
    double a = fabs((double)t);
    if (a > 6.0) a = 6.0;
    int E = (a >= 1.0) ? ilogb(a) : 0;      /* binade; below 1 the spacing is 0.5 */
    double quantum = ldexp(1.0, E - 1);
    double n = nearbyint(a / quantum);        /* ties to even */
    double r = n * quantum;
    if (r == 0.0) return sign;
    if (r < 1.0) return (uint8_t)(sign | 0x1); /* 0.5: subnormal */
    {
        int Er = ilogb(r);
        int mant = (int)(r / ldexp(1.0, Er - 1)) - 2;
        return (uint8_t)(sign | ((Er + 1) << 1) | mant);
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 block scale ([FI] section 6, block_size = 16; steps as listed in the */
/* header comment)                                                          */
/* ------------------------------------------------------------------------ */

/* E4M3 block-scale code of a block with absmax `amax` (floored at EPS) under
 * the global scale g: r = (amax / 6) * g in fp32, then the nearest E4M3 value,
 * saturating at 448. */
uint8_t pqgo_nvfp4_block_scale(float amax, float g) {
    float r = (amax / PQGO_FMAX_E2M1) * g;
    return pqgo_e4m3_encode(r);
}

/* Multiplier that takes a block's values to E2M1 units: g / value(sf) in fp32,
 * or 0 for a zero block scale (every code of the block is then a zero). */
float pqgo_nvfp4_multiplier(uint8_t sf, float g) {
    float d = pqgo_e4m3_decode(sf);
    return d == 0.0f ? 0.0f : g / d;
}

/* ------------------------------------------------------------------------ */
/* Scale layouts                                                             */
/* ------------------------------------------------------------------------ */

/* rows of one expert's column-major scale plane: M rounded up to 4 */
static int64_t padded_rows(int64_t M) { return (M + 3) / 4 * 4; }

/* byte offset of (row m, group g) in one expert's 128x4-tiled plane */
static int64_t tile128x4_offset(int64_t m, int64_t g, int64_t ng) {
    int64_t col_tiles = (ng + 3) / 4;
    int64_t tile = (m / 128) * col_tiles + (g / 4);
    int64_t r = m % 128;
    return tile * 512 + (r % 32) * 16 + (r / 32) * 4 + (g % 4);
}

/* Size in bytes of the scale buffer for E experts of M rows of K outputs. */
int64_t pqgo_scales_nbytes(int64_t E, int64_t M, int64_t K, int G,
                           int scale_ue8m0, int layout) {
    int64_t ng = K / G;
    int64_t elem = scale_ue8m0 ? 1 : 4;
    if (layout == PQGO_ROW) return E * M * ng * elem;
    if (layout == PQGO_COL) return E * ng * padded_rows(M) * elem;
    if (layout == PQGO_TILE128X4) return E * ((M + 127) / 128) * ((ng + 3) / 4) * 512;
    /* packed: int32 words, ceil(ng / 4) per row */
    return E * ((ng + 3) / 4) * padded_rows(M) * 4;
}

/* ------------------------------------------------------------------------ */
/* The whole quantization                                                    */
/* ------------------------------------------------------------------------ */

/* Quantize E experts of M rows (E = 1, masked_m = NULL: flat dispatch).
 *   in      : [E][M][K] (or [E][M][2K] when fused: gate | up), raw 16-bit
 *             bf16 or fp16 patterns
 *   out     : [E][M][K] one code byte per element ([E][M][K/2] for E2M1, two
 *             codes per byte)
 *   scales  : layout-dependent (see pqgo_scales_nbytes)
 *   masked_m: host array of E row counts, or NULL.  Rows m >= masked_m[e]
 *             (clamped to [0, M]) are not touched; neither are padding rows.
 * Returns 0, -1 for an invalid argument, -2 for a non-finite input value. */
static int quant_rows(const uint16_t *in, uint8_t *out, void *scales, int64_t E,
                      int64_t M, int64_t K, int G, int in_fp16, int out_kind,
                      int scale_ue8m0, int layout, int fused,
                      const int32_t *masked_m, const uint8_t *row_live) {
    const int out_int8 = out_kind == PQGO_OUT_INT8;
    const int out_e2m1 = out_kind == PQGO_OUT_E2M1;
    if (E < 1 || M < 0 || K <= 0 || G <= 0 || K % G != 0) return -1;
    if (layout < PQGO_ROW || layout > PQGO_TILE128X4) return -1;
    if (out_kind < PQGO_OUT_E4M3 || out_kind > PQGO_OUT_E2M1) return -1;
    if (out_e2m1 && (!scale_ue8m0 || G % 2 != 0)) return -1;  /* MXFP4: UE8M0 */
    if (scale_ue8m0 && out_int8) return -1;       /* UE8M0 pairs with FMAX */
    if ((layout == PQGO_PACKED || layout == PQGO_TILE128X4) && !scale_ue8m0) return -1;

    const int64_t ng = K / G;
    const int64_t in_width = fused ? 2 * K : K;
    const int64_t mpad = padded_rows(M);
    float *v = (float *)malloc(sizeof(float) * (size_t)G);
    if (!v) return -1;
    int status = 0;

    for (int64_t e = 0; e < E && status == 0; ++e) {
        int64_t rows = M;
        if (masked_m) {
            rows = masked_m[e];
            if (rows < 0) rows = 0;
            if (rows > M) rows = M;
        }
        for (int64_t m = 0; m < rows && status == 0; ++m) {
            if (row_live && !row_live[m]) continue;   /* varlen padding row */
            const uint16_t *xrow = in + (e * M + m) * in_width;
            uint8_t *qrow = out + (e * M + m) * (out_e2m1 ? K / 2 : K);
            for (int64_t g = 0; g < ng; ++g) {
                /* 1. decode (and fuse) the G values of this group */
                for (int i = 0; i < G; ++i) {
                    float x = pqgo_decode(xrow[g * G + i], in_fp16);
                    if (fused) {
                        float up = pqgo_decode(xrow[K + g * G + i], in_fp16);
                        if (!isfinite(x) || !isfinite(up)) { status = -2; break; }
                        x = pqgo_silu_mul(x, up);
                    }
                    if (!isfinite(x)) { status = -2; break; }
                    v[i] = x;
                }
                if (status) break;

                /* 2. absmax and 3. scale */
                float amax = pqgo_group_amax(v, G);
                float s;
                int ebyte = 0;
                if (scale_ue8m0) {
                    ebyte = pqgo_ue8m0_exponent_fmax(amax, out_e2m1 ? PQGO_FMAX_E2M1
                                                                    : PQGO_FMAX_E4M3);
                    s = ldexpf(1.0f, ebyte - 127);
                } else {
                    s = pqgo_scale_fp32(amax, out_int8);
                }

                /* 4. codes: saturating cast of x / s */
                for (int i = 0; i < G; ++i) {
                    float t = v[i] / s;
                    if (out_e2m1) {
                        int64_t j = g * G + i;
                        uint8_t code = pqgo_e2m1_encode(t);
                        if (j % 2 == 0)
                            qrow[j / 2] = code;                       /* low nibble  */
                        else
                            qrow[j / 2] = (uint8_t)(qrow[j / 2] | (code << 4)); /* high */
                    } else {
                        qrow[g * G + i] = out_int8 ? (uint8_t)pqgo_int8_encode(t)
                                                   : pqgo_e4m3_encode(t);
                    }
                }

                /* 5. scale store */
                if (layout == PQGO_ROW) {
                    int64_t idx = (e * M + m) * ng + g;
                    if (scale_ue8m0) ((uint8_t *)scales)[idx] = (uint8_t)ebyte;
                    else ((float *)scales)[idx] = s;
                } else if (layout == PQGO_COL) {
                    int64_t idx = e * ng * mpad + g * mpad + m;
                    if (scale_ue8m0) ((uint8_t *)scales)[idx] = (uint8_t)ebyte;
                    else ((float *)scales)[idx] = s;
                } else if (layout == PQGO_PACKED) {
                    int64_t nwords = (ng + 3) / 4;
                    int64_t word = e * nwords * mpad + (g / 4) * mpad + m;
                    ((uint8_t *)scales)[word * 4 + (g % 4)] = (uint8_t)ebyte;
                } else {
                    int64_t plane = ((M + 127) / 128) * ((ng + 3) / 4) * 512;
                    ((uint8_t *)scales)[e * plane + tile128x4_offset(m, g, ng)] = (uint8_t)ebyte;
                }
            }
            /* 128x4 tiles: padding columns of this row are 0 */
            if (status == 0 && layout == PQGO_TILE128X4 && ng % 4 != 0) {
                int64_t plane = ((M + 127) / 128) * ((ng + 3) / 4) * 512;
                for (int64_t g = ng; g < (ng + 3) / 4 * 4; ++g)
                    ((uint8_t *)scales)[e * plane + tile128x4_offset(m, g, ng)] = 0;
            }
            /* packed words: exponent bytes of groups past the last are 0 */
            if (status == 0 && layout == PQGO_PACKED && ng % 4 != 0) {
                int64_t nwords = (ng + 3) / 4;
                int64_t word = e * nwords * mpad + (ng / 4) * mpad + m;
                for (int64_t b = ng % 4; b < 4; ++b)
                    ((uint8_t *)scales)[word * 4 + b] = 0;
            }
        }
    }
    free(v);
    return status;
}

int pqgo_quant(const uint16_t *in, uint8_t *out, void *scales, int64_t E,
               int64_t M, int64_t K, int G, int in_fp16, int out_kind,
               int scale_ue8m0, int layout, int fused,
               const int32_t *masked_m) {
    return quant_rows(in, out, scales, E, M, K, G, in_fp16, out_kind, scale_ue8m0, layout,
                      fused, masked_m, NULL);
}

/* NVFP4 quantization of E experts of M rows of K outputs (K a multiple of 16).
 *   in, masked_m, fused: as for pqgo_quant.
 *   out    : [E][M][K/2] bytes of E2M1 code pairs (element 2i in bits 0-3).
 *   scales : one E4M3 byte per block of 16, layout PQGO_ROW ([E][M][K/16]),
 *            PQGO_COL ([E][K/16][M_pad]) or PQGO_TILE128X4 (as for MXFP4).
 *   g      : the global scale (finite, > 0).
 * Returns 0, -1 for an invalid argument, -2 for a non-finite input value. */
static int quant_rows_nvfp4(const uint16_t *in, uint8_t *out, uint8_t *scales, int64_t E,
                            int64_t M, int64_t K, int in_fp16, int layout, int fused,
                            const int32_t *masked_m, float g, const uint8_t *row_live) {
    const int G = PQGO_NVFP4_BLOCK;
    if (E < 1 || M < 0 || K <= 0 || K % G != 0) return -1;
    if (layout != PQGO_ROW && layout != PQGO_COL && layout != PQGO_TILE128X4) return -1;
    if (!(g > 0.0f) || !isfinite(g)) return -1;

    const int64_t ng = K / G;
    const int64_t in_width = fused ? 2 * K : K;
    const int64_t mpad = padded_rows(M);
    const int64_t plane = ((M + 127) / 128) * ((ng + 3) / 4) * 512;
    float v[PQGO_NVFP4_BLOCK];

    for (int64_t e = 0; e < E; ++e) {
        int64_t rows = M;
        if (masked_m) {
            rows = masked_m[e];
            if (rows < 0) rows = 0;
            if (rows > M) rows = M;
        }
        for (int64_t m = 0; m < rows; ++m) {
            if (row_live && !row_live[m]) continue;   /* varlen padding row */
            const uint16_t *xrow = in + (e * M + m) * in_width;
            uint8_t *qrow = out + (e * M + m) * (K / 2);
            for (int64_t b = 0; b < ng; ++b) {
                /* 1. decode (and fuse) the block's 16 values */
                for (int i = 0; i < G; ++i) {
                    float x = pqgo_decode(xrow[b * G + i], in_fp16);
                    if (fused) {
                        float up = pqgo_decode(xrow[K + b * G + i], in_fp16);
                        if (!isfinite(x) || !isfinite(up)) return -2;
                        x = pqgo_silu_mul(x, up);
                    }
                    if (!isfinite(x)) return -2;
                    v[i] = x;
                }
                /* 2. absmax, 3. block scale and its multiplier */
                float amax = pqgo_group_amax(v, G);
                uint8_t sf = pqgo_nvfp4_block_scale(amax, g);
                float mult = pqgo_nvfp4_multiplier(sf, g);
                /* 4. codes, two per byte */
                for (int i = 0; i < G; i += 2) {
                    uint8_t lo = pqgo_e2m1_encode(v[i] * mult);
                    uint8_t hi = pqgo_e2m1_encode(v[i + 1] * mult);
                    qrow[(b * G + i) / 2] = (uint8_t)(lo | (hi << 4));
                }
                /* 5. block-scale byte */
                if (layout == PQGO_ROW)
                    scales[(e * M + m) * ng + b] = sf;
                else if (layout == PQGO_COL)
                    scales[e * ng * mpad + b * mpad + m] = sf;
                else
                    scales[e * plane + tile128x4_offset(m, b, ng)] = sf;
            }
            if (layout == PQGO_TILE128X4)
                for (int64_t b = ng; b % 4 != 0; ++b)
                    scales[e * plane + tile128x4_offset(m, b, ng)] = 0;
        }
    }
    return 0;
}

int pqgo_quant_nvfp4(const uint16_t *in, uint8_t *out, uint8_t *scales, int64_t E,
                     int64_t M, int64_t K, int in_fp16, int layout, int fused,
                     const int32_t *masked_m, float g) {
    return quant_rows_nvfp4(in, out, scales, E, M, K, in_fp16, layout, fused, masked_m, g,
                            NULL);
}

/* ------------------------------------------------------------------------ */
/* Grouped-contiguous (varlen) dispatch  ([PR] 实现拆解 item 4; [FI] section 7; */
/* the reading is in the header comment)                                     */
/* ------------------------------------------------------------------------ */

/* Mark the token rows of E segments of M packed rows: row_live[r] = 1 for a
 * token row, 0 for every other row.  Segment e spans rows [indptr[e],
 * indptr[e+1]) with both ends clamped into [0, M] and the end no lower than
 * the start; its first lens[e] rows, clamped into [0, segment rows], are
 * tokens (every row of the segment when lens is NULL). */
void pqgo_varlen_rows(const int32_t *indptr, const int32_t *lens, int64_t E, int64_t M,
                      uint8_t *row_live) {
    memset(row_live, 0, (size_t)M);
    for (int64_t e = 0; e < E; ++e) {
        int64_t start = indptr[e], end = indptr[e + 1];
        if (start < 0) start = 0;
        if (start > M) start = M;
        if (end < start) end = start;
        if (end > M) end = M;
        int64_t n = end - start;
        if (lens) {
            n = lens[e];
            if (n < 0) n = 0;
            if (n > end - start) n = end - start;
        }
        for (int64_t r = start; r < start + n; ++r) row_live[r] = 1;
    }
}

/* Quantize the token rows of M packed rows [M][K] ([M][2K] fused) in E
 * segments (indptr: E + 1 row offsets; lens: E token counts or NULL).  Codes go
 * to the same rows of out ([M][K], or [M][K/2] for E2M1); scales to one plane
 * of M rows in the chosen layout (pqgo_scales_nbytes(1, M, ...) bytes).  Padding
 * rows are not touched.  Same kinds and status values as pqgo_quant. */
int pqgo_quant_varlen(const uint16_t *in, uint8_t *out, void *scales, int64_t M, int64_t K,
                      int G, int in_fp16, int out_kind, int scale_ue8m0, int layout,
                      int fused, const int32_t *indptr, const int32_t *lens, int64_t E) {
    if (E < 1 || M < 0 || indptr == NULL) return -1;
    uint8_t *live = (uint8_t *)malloc((size_t)(M > 0 ? M : 1));
    if (!live) return -1;
    pqgo_varlen_rows(indptr, lens, E, M, live);
    int status = quant_rows(in, out, scales, 1, M, K, G, in_fp16, out_kind, scale_ue8m0,
                            layout, fused, NULL, live);
    free(live);
    return status;
}

/* NVFP4 form of pqgo_quant_varlen (global scale g; layouts as pqgo_quant_nvfp4). */
int pqgo_quant_varlen_nvfp4(const uint16_t *in, uint8_t *out, uint8_t *scales, int64_t M,
                            int64_t K, int in_fp16, int layout, int fused,
                            const int32_t *indptr, const int32_t *lens, int64_t E, float g) {
    if (E < 1 || M < 0 || indptr == NULL) return -1;
    uint8_t *live = (uint8_t *)malloc((size_t)(M > 0 ? M : 1));
    if (!live) return -1;
    pqgo_varlen_rows(indptr, lens, E, M, live);
    int status = quant_rows_nvfp4(in, out, scales, 1, M, K, in_fp16, layout, fused, NULL, g,
                                  live);
    free(live);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the element functions, for the pin tests                   */
/* ------------------------------------------------------------------------ */

void pqgo_decode_n(const uint16_t *bits, float *out, int64_t n, int in_fp16) {
    for (int64_t i = 0; i < n; ++i) out[i] = pqgo_decode(bits[i], in_fp16);
}

void pqgo_silu_mul_n(const float *gate, const float *up, float *y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = pqgo_silu_mul(gate[i], up[i]);
}

void pqgo_e4m3_encode_n(const float *t, uint8_t *q, int64_t n) {
    for (int64_t i = 0; i < n; ++i) q[i] = pqgo_e4m3_encode(t[i]);
}

void pqgo_e2m1_encode_n(const float *t, uint8_t *q, int64_t n) {
    for (int64_t i = 0; i < n; ++i) q[i] = pqgo_e2m1_encode(t[i]);
}

void pqgo_ue8m0_exponent_fmax_n(const float *amax, uint8_t *e, int64_t n, float fmax) {
    for (int64_t i = 0; i < n; ++i) e[i] = (uint8_t)pqgo_ue8m0_exponent_fmax(amax[i], fmax);
}

void pqgo_int8_encode_n(const float *t, int8_t *q, int64_t n) {
    for (int64_t i = 0; i < n; ++i) q[i] = pqgo_int8_encode(t[i]);
}

void pqgo_ue8m0_exponent_n(const float *amax, uint8_t *e, int64_t n) {
    for (int64_t i = 0; i < n; ++i) e[i] = (uint8_t)pqgo_ue8m0_exponent(amax[i]);
}

void pqgo_scale_fp32_n(const float *amax, float *s, int64_t n, int out_int8) {
    for (int64_t i = 0; i < n; ++i) s[i] = pqgo_scale_fp32(amax[i], out_int8);
}

void pqgo_e4m3_decode_n(const uint8_t *c, float *v, int64_t n) {
    for (int64_t i = 0; i < n; ++i) v[i] = pqgo_e4m3_decode(c[i]);
}

void pqgo_nvfp4_block_scale_n(const float *amax, uint8_t *sf, int64_t n, float g) {
    for (int64_t i = 0; i < n; ++i) sf[i] = pqgo_nvfp4_block_scale(amax[i], g);
}

void pqgo_nvfp4_multiplier_n(const uint8_t *sf, float *m, int64_t n, float g) {
    for (int64_t i = 0; i < n; ++i) m[i] = pqgo_nvfp4_multiplier(sf[i], g);
}
