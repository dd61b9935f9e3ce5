// Per-token-group quantization kernels for sm_100a.
//
// One kernel body, specialised at compile time on what changes the inner loop:
// input dtype, group size G, output/scale kind (E4M3 + fp32 scale, E4M3 +
// UE8M0 scale, INT8 + fp32 scale, MXFP4 = E2M1 + UE8M0, NVFP4 = E2M1 + E4M3
// block scale) and the fused SiLU-and-mul prologue.  What
// changes only once per group (the scale layout) or once per CTA (flat or
// masked dispatch) is a runtime field of the parameter block.  The variant axes
// are those of the sglang PR #30924 report, "[JIT] Trait-driven
// per_token_group_quant", 实现拆解 item 1; the arithmetic is its 关键源码片段
// (ref_fp8_ue8m0) and 风险与影响 (INT8, amax / 127).
//
// Work decomposition.  A "strip" is 32 lanes x 16 elements = 512 consecutive
// outputs of one row, so each lane owns 16 outputs (32 bytes of bf16/fp16
// input, one 256-bit load; the report's 执行摘要 names the same 32 B per lane
// tiling).  A 1 x G group spans L = G/16 adjacent lanes; its absmax is a
// log2(L)-step xor-shuffle.  The strips of all experts (rows < masked_m[e]
// only) form one sequence, cut into blocks of WARPS x ITEMS strips that the
// CTAs take round-robin.  With several experts each CTA first prefix-sums the
// per-expert strip counts (in each warp's registers up to 32 experts, in
// shared memory beyond), so a warp can find the expert and row of any strip;
// skewed masked_m cannot leave CTAs idle.  Grouped-contiguous (varlen)
// dispatch uses the same table over the token rows of E segments of one packed
// buffer (each segment's first row kept beside its count), so padding rows are
// never visited.
//
// Memory-level parallelism.  A warp takes ITEMS strips per chunk and issues
// all of the chunk's 32-byte loads before any arithmetic; with 32-48 resident
// warps per SM (register-light kernel) that keeps the HBM queues full.
// Keeping a second chunk in flight was measured slower both ways it was tried:
// in registers (double-buffering) and in shared memory (cp.async stages), the
// extra registers and instructions cost more warps than the prefetch won.
//
// Exact codes.  Codes must equal the rounding of fp32(x / s).  A per-element
// IEEE division is too slow for a bandwidth-bound loop, so the quotient is
// formed from y = RN(1/s) (one correctly rounded reciprocal per group) and
// residual corrections, q <- q + (x - q*s) * y with exact FMA residuals
// (Markstein's correction; P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  The
// first step leaves q within an ulp of x/s, and a second returns the correctly
// rounded quotient.  One step is enough for the codes: for every 8-bit (bf16)
// and 11-bit (fp16) significand of x, every fp32 significand of s and every
// binade of x/s that can yield a nonzero code, an exhaustive CPU comparison
// found the E4M3 and INT8 code of the one-step q equal to the code of
// RN(x/s) (2.4e10 bf16 and 1.9e11 fp16 cases for E4M3).  Where |x/s| < 2^-12
// the residual may underflow, but every such t rounds to a signed zero code,
// and the sign is restored from x.  The correction runs on packed f32x2 FMAs
// (FFMA2), two elements per instruction.
//
// UE8M0 exponent without a division.  For a normal fp32 amax = m * 2^E (m in
// [1, 2)), the smallest n with 448 * 2^n >= amax is E - 8 + [m > 1.75], because
// 448 = 1.75 * 2^8.  The pages' rule (biased exponent of fp32(amax/448), plus
// one for a nonzero mantissa) gives the same byte for every fp32 amax >= 1e-10:
// an exhaustive check over all 1.35e9 such values found no difference.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

namespace pqg {

// E2M1_UE8M0 is MXFP4 (G = 32/64/128); E2M1_E4M3 is NVFP4 (G = 16, an E4M3
// block scale under a per-call fp32 global scale).
enum class Kind : int { E4M3_FP32 = 0, E4M3_UE8M0 = 1, INT8_FP32 = 2, E2M1_UE8M0 = 3,
                        E2M1_E4M3 = 4 };

// Kinds whose scale is a UE8M0 power of two.
__host__ __device__ constexpr bool is_ue8m0(Kind k) {
    return k == Kind::E4M3_UE8M0 || k == Kind::E2M1_UE8M0;
}
// Kinds with FP4 codes, two per byte.
__host__ __device__ constexpr bool is_e2m1(Kind k) {
    return k == Kind::E2M1_UE8M0 || k == Kind::E2M1_E4M3;
}
// Kinds whose stored scale is one byte (UE8M0 exponent or E4M3 block scale).
__host__ __device__ constexpr bool byte_scale(Kind k) {
    return is_ue8m0(k) || k == Kind::E2M1_E4M3;
}

// Runtime scale layouts (same numbering as the C ABI's pqg_scale_layout).
enum : uint32_t { kRowMajor = 0, kColMajor = 1, kPacked = 2, kTiled128x4 = 3 };

// Byte of (row m, group g) in one expert's 128x4-tiled exponent plane.
__device__ __forceinline__ uint64_t tile128x4_offset(uint32_t m, uint32_t g, uint32_t ng) {
    const uint32_t col_tiles = (ng + 3u) >> 2;
    const uint64_t tile = static_cast<uint64_t>(m >> 7) * col_tiles + (g >> 2);
    return tile * 512u + (m & 31u) * 16u + ((m >> 5) & 3u) * 4u + (g & 3u);
}

// Store the UE8M0 byte of (row, group g) in the tiled plane; the last group's
// lane also zeroes the padding groups of the row's last tile column.
__device__ __forceinline__ void store_tiled(uint8_t *sc, uint32_t row, uint32_t g, uint32_t ng,
                                            uint32_t e8) {
    sc[tile128x4_offset(row, g, ng)] = static_cast<uint8_t>(e8);
    if (g == ng - 1u)
        for (uint32_t pad = ng; (pad & 3u) != 0u; ++pad) sc[tile128x4_offset(row, pad, ng)] = 0;
}

constexpr int kStripElems = 512;           // outputs per strip (32 lanes x 16)
constexpr uint32_t kStripBytes = 1024;     // input bytes per strip (16-bit elements)
constexpr uint32_t kMaxExperts = 4096;     // prefix table lives in shared memory

struct Params {
    const uint8_t *in;         // expert 0, row 0
    uint8_t *out;              // expert 0, row 0
    uint8_t *scales;           // expert 0's scale plane (byte address)
    const int32_t *masked_m;   // device int32[experts], or null: all M rows
    const int32_t *seg_indptr; // varlen: device int32[experts + 1] segment row offsets
    const int32_t *seg_lens;   // varlen: device int32[experts] token counts, or null
    const float *gscale;       // NVFP4 only: device fp32 global scale g
    int64_t in_expert_bytes;   // M * in_row_bytes
    int64_t out_expert_bytes;  // M * out_row_bytes
    int64_t scale_expert_bytes;
    uint32_t M;                // rows per expert (capacity when masked; all rows when varlen)
    uint32_t K;                // outputs per row
    uint32_t in_row_bytes;     // 2K (plain) or 4K (fused), in bytes
    uint32_t out_row_bytes;    // K (one byte per code) or K/2 (E2M1, two per byte)
    uint32_t ng;               // groups per row
    uint32_t segs;             // strips per row = ceil(K / 512)
    uint32_t segs_magic;       // s / segs = umulhi(s, segs_magic) >> segs_shift (0: segs == 1)
    uint32_t segs_shift;
    uint32_t mpad;             // rows of a column-major plane (M rounded up to 4)
    uint32_t layout;           // kRowMajor / kColMajor / kPacked
    uint32_t experts;          // <= kMaxExperts
    uint32_t items;            // strips per warp per block, 1 .. ITEMS
    uint32_t spec;             // kMaskedSpec: rows per expert loaded before masked_m is known
    uint32_t spec_magic;       // s / (spec * segs), as segs_magic
    uint32_t spec_shift;
};

// Dispatch forms: one expert's M rows (flat), E experts of M rows each with a
// per-expert row count (masked), or E segments of one buffer of M packed rows
// (varlen, grouped-contiguous: expert strides are 0 and a segment's rows
// start at its own row offset).
enum : int { kFlat = 0, kMasked = 1, kVarlen = 2, kMaskedSpec = 3 };

// Dynamic shared memory of one CTA: the expert prefix table (more than 32
// experts only), followed by the segments' first rows when varlen.
__host__ __device__ constexpr uint32_t smem_bytes(uint32_t experts, bool varlen = false) {
    return experts > 32u ? 4u * (experts + 1u) + (varlen ? 4u * experts : 0u) : 0u;
}

// ---------------------------------------------------------------------------
// Memory helpers
// ---------------------------------------------------------------------------

// 32-byte streaming load: read-only path, no L1 allocation, and a 256-byte L2
// prefetch hint (each group of G >= 32 bf16 is 64..256 contiguous bytes).
__device__ __forceinline__ void load32B(const void *p, uint32_t (&r)[8]) {
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::256B.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7])
        : "l"(p));
}

// Bring `bytes` bytes (a multiple of 16, 16-byte aligned) into L2 with the
// bulk-copy engine: one instruction, no registers, no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void store8B(void *p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void store16B(void *p, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's memory before the
// first global access; let the next grid start its prologue when we are done
// (or, with PQG_EARLY_TRIGGER, as soon as every CTA has started).
#ifndef PQG_EARLY_TRIGGER
#define PQG_EARLY_TRIGGER 0
#endif
__device__ __forceinline__ void wait_for_producer() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
#if PQG_EARLY_TRIGGER
    // A dependent grid launches only once every CTA of this grid has signalled
    // (or exited), so signalling at entry cannot starve this grid of SMs; the
    // dependent's own griddepcontrol.wait still waits for this grid to finish.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}
__device__ __forceinline__ void release_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Element conversion
// ---------------------------------------------------------------------------

template <typename In>
__device__ __forceinline__ void widen2(uint32_t w, float &lo, float &hi);

// bf16 is the top half of an fp32: widening is a shift / mask.
template <>
__device__ __forceinline__ void widen2<__nv_bfloat16>(uint32_t w, float &lo, float &hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

template <>
__device__ __forceinline__ void widen2<__half>(uint32_t w, float &lo, float &hi) {
    __half2 h = *reinterpret_cast<__half2 *>(&w);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
}

// silu(g) * u for a pair, in fp32: sigmoid(g) = 1 / (1 + 2^t), t = -g log2 e,
// with the hardware ex2 and rcp approximations, on packed f32x2 arithmetic
// where it exists.  g * u is one exact mixed-precision FMA of the two 16-bit
// inputs (8- or 11-bit significands: the product fits fp32), so the element is
// (g u) / (1 + 2^t) with the approximations' errors and one rounding.  The
// extremes stay right without a branch: for g << 0 the power is +inf (or the
// reciprocal flushes to zero) and the result is a zero with g u's sign; for
// g >> 0 the power flushes to 0 and the result is g u.  The product stays
// within a few fp32 ulps of silu(g) * u.
//
// Both approximations run on the SFU (MUFU) pipe, about 60 % busy at the
// hidden-size fused call.  Moving the reciprocal to the FMA pipe (an integer
// seed and three Newton-Raphson steps on f32x2 FMAs) was measured slower: the
// eight extra instructions per pair cost more than the freed SFU slot
// ([4096, 2 x 7168] 25.1 -> 26.3 us, masked 51.4 -> 55.6 us).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// a * b for the 16-bit halves of two packed words, exact in fp32 (adding -0
// keeps every product, -0 included)
template <typename In>
__device__ __forceinline__ float2 mul_exact2(uint32_t a, uint32_t b) {
    float lo, hi;
    if constexpr (std::is_same<In, __nv_bfloat16>::value)
        asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
            "mov.b32 {al, ah}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
            "fma.rn.f32.bf16 %0, al, bl, 0f80000000;\n\t"
            "fma.rn.f32.bf16 %1, ah, bh, 0f80000000;\n\t}"
            : "=f"(lo), "=f"(hi) : "r"(a), "r"(b));
    else
        asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
            "mov.b32 {al, ah}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
            "fma.rn.f32.f16 %0, al, bl, 0f80000000;\n\t"
            "fma.rn.f32.f16 %1, ah, bh, 0f80000000;\n\t}"
            : "=f"(lo), "=f"(hi) : "r"(a), "r"(b));
    return make_float2(lo, hi);
}
// silu(gate) * up for the pair of elements held in packed words gw and uw
template <typename In>
__device__ __forceinline__ float2 silu_mul_pair(uint32_t gw, uint32_t uw) {
    constexpr float kNegLog2e = -1.4426950408889634f;
    float g0, g1;
    widen2<In>(gw, g0, g1);
    const float2 t = __fmul2_rn(make_float2(g0, g1), make_float2(kNegLog2e, kNegLog2e));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(t.x), ex2_approx(t.y)),
                                make_float2(1.0f, 1.0f));
    return __fmul2_rn(mul_exact2<In>(gw, uw), make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Packed pair of E4M3 codes: `lo` in bits 0-7, `hi` in bits 8-15.  Round to
// nearest even; satfinite clamps to +-448 (never reached: |t| <= 448 here).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E4M3 codes as one word, (a0, a1) in the low half: two conversions and
// a vector move (measured faster than shift/or: the assembler places the
// halves).
__device__ __forceinline__ uint32_t e4m3x4(float a0, float a1, float b0, float b1) {
    uint32_t r;
    asm("{\n\t.reg .b16 p, q;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 p, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 q, %4, %3;\n\t"
        "mov.b32 %0, {p, q};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
    return r;
}

// Eight OCP E2M1 codes as one word: pair k = (a_k lo, a_k hi) becomes byte k,
// the first of the pair in bits 0-3 and the second in bits 4-7; round to
// nearest even, satfinite clamps to +-6 (MXFP4 never reaches it; NVFP4 can).
// The four bytes are joined by a vector move, so the assembler places each
// conversion's byte (measured faster than shift/or and than byte permutes).
__device__ __forceinline__ uint32_t e2m1x8(float a0, float a1, float b0, float b1, float c0,
                                           float c1, float d0, float d1) {
    uint32_t r;
    asm("{\n\t.reg .b8 p, q, s, t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 p, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 s, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %8, %7;\n\t"
        "mov.b32 %0, {p, q, s, t};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1), "f"(d0), "f"(d1));
    return r;
}

// Markstein corrections per quotient (STEPS): 2 give the correctly rounded
// fp32 x/s for every x; 1 leaves q within an ulp of it, and exhaustive CPU
// checks found the E4M3 and INT8 codes of that q equal to the codes of
// RN(x/s) for every bf16 / fp16 x and every fp32 s (all significand pairs,
// every binade of x/s that yields a nonzero code).  Both kernels use 1.
#ifndef PQG_DIV_STEPS
#define PQG_DIV_STEPS 1
#endif
constexpr int kDivSteps = PQG_DIV_STEPS;

// The fp32 quotient x/s for a pair, from y = RN(1/s) and ns = -s (Markstein
// corrections; see the file comment).
template <int STEPS>
__device__ __forceinline__ float2 div_rn2(float2 x, float2 y, float2 ns) {
    float2 q = __fmul2_rn(x, y);
    float2 r = __ffma2_rn(q, ns, x);   // x - q*s, exact
    q = __ffma2_rn(r, y, q);
    if constexpr (STEPS > 1) {
        r = __ffma2_rn(q, ns, x);
        q = __ffma2_rn(r, y, q);
    }
    return q;
}

// The same correction carried on the negated quotient, from ny = -RN(1/s) and
// s: returns -x/s with the sign of zero right for every x.  (q = x*ny and
// r = x + q*s: for x = -0 the chain gives +0, for x = +0 it gives -0, and a
// tiny x whose quotient underflows keeps the sign of -x.)  Negating the codes
// afterwards is one XOR of the packed sign bits.
template <int STEPS>
__device__ __forceinline__ float2 neg_div_rn2(float2 x, float2 ny, float2 s) {
    float2 q = __fmul2_rn(x, ny);
    float2 r = __ffma2_rn(q, s, x);    // x - (x/s)*s, exact
    q = __ffma2_rn(r, ny, q);
    if constexpr (STEPS > 1) {
        r = __ffma2_rn(q, s, x);
        q = __ffma2_rn(r, ny, q);
    }
    return q;
}

// bf16 x * 2^k with an exact bf16 power of two, widened: one mixed-precision
// FMA (bf16 x bf16 + f32 -> f32).  Adding -0 keeps every product, -0 included.
__device__ __forceinline__ float mul_bf16_pow2(uint16_t x, uint16_t p2) {
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(x), "h"(p2), "f"(-0.0f));
    return d;
}

// max |x| over the 16 bf16/fp16 values of 8 packed words, as the 16-bit
// pattern of the largest magnitude (finite values order like their magnitude
// bits).
__device__ __forceinline__ uint32_t absmax_bits16(const uint32_t (&w)[8]) {
    uint32_t m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = w[i] & 0x7FFF7FFFu;
    uint32_t a = __vimax3_u16x2(m[0], m[1], m[2]);
    uint32_t b = __vimax3_u16x2(m[3], m[4], m[5]);
    a = __vimax3_u16x2(a, b, __vimax3_u16x2(m[6], m[7], 0u));
    return max(a & 0xFFFFu, a >> 16);
}

// max |v| over 16 values as a tree (depth 4 instead of a chain of 16)
__device__ __forceinline__ float absmax16(const float (&v)[16]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    return m[0];
}

// The value of a non-negative finite bf16 / fp16 magnitude pattern (the
// per-token kernel takes its absmax on raw bits).
template <typename In>
__device__ __forceinline__ float bits16_to_float(uint32_t b);
template <>
__device__ __forceinline__ float bits16_to_float<__nv_bfloat16>(uint32_t b) {
    return __uint_as_float(b << 16);
}
template <>
__device__ __forceinline__ float bits16_to_float<__half>(uint32_t b) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

// ---------------------------------------------------------------------------
// Per-group scale math (one group per L lanes; all lanes compute it)
// ---------------------------------------------------------------------------

// UE8M0 byte of a (normal, >= 1e-10) amax: E(amax) - 8 + [mantissa > 0x600000],
// i.e. 127 + ceil(log2(amax / 448)); see the file comment.
__device__ __forceinline__ uint32_t ue8m0_exponent(float amax) {
    const uint32_t b = __float_as_uint(amax);
    return ((b >> 23) & 0xFFu) - 8u + ((b & 0x7FFFFFu) > 0x600000u ? 1u : 0u);
}

// RN(a / c) for the scale divisors: q = a * RN(1/c), then two Markstein
// corrections with exact FMA residuals.  An exhaustive CPU check over every
// fp32 a >= 1e-10 (1.35e9 values) found it equal to the IEEE quotient for both
// c = 448 and c = 127.
constexpr float kRcp448 = 0x1.24924ap-9f;   // RN(1/448)
constexpr float kRcp127 = 0x1.020408p-7f;   // RN(1/127)
__device__ __forceinline__ float div_by_const(float a, float c, float rc) {
    float q = __fmul_rn(a, rc);
    float r = __fmaf_rn(-q, c, a);
    q = __fmaf_rn(r, rc, q);
    r = __fmaf_rn(-q, c, a);
    return __fmaf_rn(r, rc, q);
}

// The same for FMAX = 6 (E2M1): 6 = 1.5 * 2^2, so the byte is
// E(amax) - 2 + [mantissa > 0x400000].  Checked exhaustively against the
// division rule over every fp32 amax >= 1e-10.
__device__ __forceinline__ uint32_t ue8m0_exponent_e2m1(float amax) {
    const uint32_t b = __float_as_uint(amax);
    return ((b >> 23) & 0xFFu) - 2u + ((b & 0x7FFFFFu) > 0x400000u ? 1u : 0u);
}

struct GroupScale {
    float mult;   // UE8M0: 2^(127-e) (exact); fp32 kinds: y = RN(1/s); NVFP4: g / value(sf)
    float neg_s;  // fp32 kinds: -s
    float s;      // fp32 kinds: the stored scale
    uint32_t e8;  // UE8M0: the stored exponent byte; NVFP4: the E4M3 block-scale byte
};

// NVFP4 ("block_size = 16 -> NVFP4", FlashInfer GEMM notes, section 6).  Per
// block of 16, in fp32: r = RN(amax / 6) * g, the block-scale byte sf = nearest
// E4M3 code of r (satfinite: 448 at most), and the codes' multiplier g /
// value(sf), 0 for sf = 0.  A block-scale code has 127 non-negative values, so
// each CTA divides once per code into a shared-memory table (nv[0..127]; nv[128]
// holds g) instead of once per block.  RN(amax / 6) uses div_by_const, checked
// exhaustively against the IEEE quotient over every fp32 amax >= 1e-10.
constexpr float kRcp6 = 0x1.555556p-3f;    // RN(1/6)
constexpr int kNvTable = 129;

__device__ __forceinline__ float e4m3_code_value(uint32_t c) {
    // (8 + m) * 2^(e - 10) for exponent field e >= 1, m * 2^-9 for e = 0
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    const float p2 = __uint_as_float((max(e, 1u) + 117u) << 23);
    return p2 * static_cast<float>(e != 0u ? 8u + m : m);
}

// Every thread of the CTA calls it (blockDim.x >= 128); ends with __syncthreads.
__device__ __forceinline__ void build_nvfp4_table(const Params &p, float *nv) {
    if (threadIdx.x < 128u) {
        const float g = __ldg(p.gscale);
        const float d = e4m3_code_value(threadIdx.x);
        nv[threadIdx.x] = d == 0.0f ? 0.0f : __fdiv_rn(g, d);
        if (threadIdx.x == 0u) nv[128] = g;
    }
    __syncthreads();
}

template <Kind KIND>
__device__ __forceinline__ GroupScale make_scale(float amax, const float *nv = nullptr) {
    GroupScale gs;
    amax = fmaxf(amax, 1e-10f);   // EPS floor
    if constexpr (KIND == Kind::E2M1_E4M3) {
        const float r = __fmul_rn(div_by_const(amax, 6.0f, kRcp6), nv[128]);
        gs.e8 = e4m3x2(r, 0.0f) & 0xFFu;
        gs.mult = nv[gs.e8 & 0x7Fu];   // r >= 0: the sign bit is clear
        gs.s = 0.0f;
        gs.neg_s = 0.0f;
    } else if constexpr (is_ue8m0(KIND)) {
        gs.e8 = KIND == Kind::E2M1_UE8M0 ? ue8m0_exponent_e2m1(amax) : ue8m0_exponent(amax);
        gs.mult = __uint_as_float((254u - gs.e8) << 23);
        gs.s = 0.0f;
        gs.neg_s = 0.0f;
    } else {
        gs.s = KIND == Kind::INT8_FP32 ? div_by_const(amax, 127.0f, kRcp127)
                                       : div_by_const(amax, 448.0f, kRcp448);
        gs.mult = __frcp_rn(gs.s);
        gs.neg_s = -gs.s;
        gs.e8 = 0;
    }
    return gs;
}

// 16 values -> 16 code bytes (4 words, element 0 in the lowest byte).
template <Kind KIND, int STEPS = kDivSteps>
__device__ __forceinline__ void encode16(const float (&v)[16], const GroupScale &gs,
                                         uint32_t (&w)[4]) {
    if constexpr (is_e2m1(KIND)) {
        // 16 codes in 8 bytes: w[0] elements 0..7, w[1] elements 8..15
        const float2 m2 = make_float2(gs.mult, gs.mult);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float2 t[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                t[k] = __fmul2_rn(make_float2(v[8 * j + 2 * k], v[8 * j + 2 * k + 1]), m2);
            w[j] = e2m1x8(t[0].x, t[0].y, t[1].x, t[1].y, t[2].x, t[2].y, t[3].x, t[3].y);
        }
    } else if constexpr (KIND == Kind::E4M3_UE8M0) {
        const float2 m2 = make_float2(gs.mult, gs.mult);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // multiplying by a power of two is exact: t = x / s
            float2 a = __fmul2_rn(make_float2(v[4 * j], v[4 * j + 1]), m2);
            float2 b = __fmul2_rn(make_float2(v[4 * j + 2], v[4 * j + 3]), m2);
            w[j] = e4m3x4(a.x, a.y, b.x, b.y);
        }
    } else if constexpr (KIND == Kind::E4M3_FP32) {
        // codes of -t, then the four sign bits flipped at once
        const float2 ny2 = make_float2(-gs.mult, -gs.mult);
        const float2 s2 = make_float2(gs.s, gs.s);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 a = neg_div_rn2<STEPS>(make_float2(v[4 * j], v[4 * j + 1]), ny2, s2);
            const float2 b = neg_div_rn2<STEPS>(make_float2(v[4 * j + 2], v[4 * j + 3]), ny2, s2);
            w[j] = e4m3x4(a.x, a.y, b.x, b.y) ^ 0x80808080u;
        }
    } else {
        // INT8: adding 1.5 * 2^23 rounds |t| < 2^22 to an integer (ties to even)
        // and leaves it in the low mantissa bits; |t| <= 127 + 2^-17 here, so
        // the clamp to [-128, 127] never binds.
        const float2 y2 = make_float2(gs.mult, gs.mult);
        const float2 ns2 = make_float2(gs.neg_s, gs.neg_s);
        const float2 magic = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 a =
                __fadd2_rn(div_rn2<STEPS>(make_float2(v[4 * j], v[4 * j + 1]), y2, ns2), magic);
            float2 b =
                __fadd2_rn(div_rn2<STEPS>(make_float2(v[4 * j + 2], v[4 * j + 3]), y2, ns2), magic);
            uint32_t ab = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040);
            uint32_t cd = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040);
            w[j] = __byte_perm(ab, cd, 0x5410);
        }
    }
}

// ---------------------------------------------------------------------------
// The strip sequence: which expert, row and strip-in-row a strip index is
// ---------------------------------------------------------------------------
//
// Strips of expert e are [start_e, start_e + strips_e); strips_e =
// rows_e * segs with rows_e = clamp(masked_m[e], 0, M) (M without masked_m),
// or, varlen, the token rows of segment e (see segment() below), whose first
// row base_e is the segment's offset.  Three representations, picked per
// launch:
//   one expert   : start 0, strips = total (no table at all);
//   <= 32 experts: a warp-register table, lane e holding expert e's count,
//                  inclusive prefix (and first row); a lookup is one ballot and
//                  two (three) shuffles;
//   more experts : a shared-memory prefix table built by the CTA (followed by
//                  the first rows).

constexpr uint32_t kWarpTableExperts = 32;

struct ExpertTable {
    uint32_t mode;     // 0 one expert, 1 warp table, 2 shared-memory table
    uint32_t total;    // strips of all experts
    uint32_t incl;     // mode 1: this lane's inclusive prefix (total for lanes >= E)
    uint32_t cnt;      // mode 1: this lane's expert's strips
    uint32_t base;     // varlen, modes 0-1: first row of (this lane's) segment
    const uint32_t *prefix;  // mode 2: prefix[e] = start_e, prefix[E] = total;
                             // varlen: prefix[E + 1 + e] = first row of segment e
};

struct Span {
    uint32_t e, start, strips, base;   // base: first row (varlen), else 0
};

// Segment e of a varlen call: rows [indptr[e], indptr[e+1]) clamped into
// [0, M] with the end no lower than the start; its first lens[e] rows,
// clamped into the segment (all of them without lens), are tokens.
__device__ __forceinline__ uint32_t segment_rows(const Params &p, uint32_t e, uint32_t &first) {
    const int M = static_cast<int>(p.M);
    const int s = min(max(__ldg(p.seg_indptr + e), 0), M);
    const int end = min(max(__ldg(p.seg_indptr + e + 1), s), M);
    int n = end - s;
    if (p.seg_lens != nullptr) n = min(max(__ldg(p.seg_lens + e), 0), n);
    first = static_cast<uint32_t>(s);
    return static_cast<uint32_t>(n);
}

template <bool VARLEN>
__device__ __forceinline__ uint32_t expert_strips(const Params &p, uint32_t e, uint32_t &first) {
    uint32_t rows = p.M;
    first = 0;
    if constexpr (VARLEN) {
        rows = segment_rows(p, e, first);
    } else if (p.masked_m != nullptr) {
        const int mm = __ldg(p.masked_m + e);
        rows = static_cast<uint32_t>(min(max(mm, 0), static_cast<int>(p.M)));
    }
    return rows * p.segs;
}

// prefix[e] = strips of experts 0..e-1 (varlen: and prefix[E + 1 + e] = first
// row of segment e).  Every thread of the CTA calls it; it ends with
// __syncthreads.
template <bool VARLEN>
__device__ __forceinline__ void build_prefix(const Params &p, uint32_t *prefix) {
    __shared__ uint32_t warp_sums[32];
    const uint32_t n = blockDim.x, t = threadIdx.x, lane = t & 31u, warp = t >> 5;
    const uint32_t per = (p.experts + n - 1) / n;
    const uint32_t lo = min(t * per, p.experts), hi = min(lo + per, p.experts);
    uint32_t local = 0, first = 0;
    for (uint32_t e = lo; e < hi; ++e) local += expert_strips<VARLEN>(p, e, first);
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= static_cast<uint32_t>(o)) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    uint32_t base = 0;
    for (uint32_t w = 0; w < warp; ++w) base += warp_sums[w];
    uint32_t run = base + incl - local;
    for (uint32_t e = lo; e < hi; ++e) {
        prefix[e] = run;
        run += expert_strips<VARLEN>(p, e, first);
        if constexpr (VARLEN) prefix[p.experts + 1u + e] = first;
    }
    if (t == n - 1) prefix[p.experts] = base + incl;
    __syncthreads();
}

// Build the table (every thread of the CTA calls it).
template <bool VARLEN>
__device__ __forceinline__ ExpertTable make_table(const Params &p, uint32_t *smem_prefix,
                                                  uint32_t lane) {
    ExpertTable t;
    t.incl = t.cnt = t.base = 0;
    t.prefix = smem_prefix;
    if (p.experts == 1) {
        t.mode = 0;
        t.total = expert_strips<VARLEN>(p, 0, t.base);
    } else if (p.experts <= kWarpTableExperts) {
        t.mode = 1;
        t.cnt = lane < p.experts ? expert_strips<VARLEN>(p, lane, t.base) : 0u;
        uint32_t incl = t.cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= static_cast<uint32_t>(o)) incl += v;
        }
        t.incl = incl;
        t.total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    } else {
        t.mode = 2;
        build_prefix<VARLEN>(p, smem_prefix);
        t.total = smem_prefix[p.experts];
    }
    return t;
}

// The expert holding strip s (s < total).  Warp-uniform s; every lane calls.
template <bool VARLEN>
__device__ __forceinline__ Span locate(const ExpertTable &t, uint32_t experts, uint32_t s) {
    Span sp;
    sp.base = 0;
    if (t.mode == 0) {
        sp.e = 0;
        sp.start = 0;
        sp.strips = t.total;
        if constexpr (VARLEN) sp.base = t.base;
    } else if (t.mode == 1) {
        // experts whose whole range lies at or below s come first
        sp.e = __popc(__ballot_sync(0xFFFFFFFFu, t.incl <= s));
        const uint32_t incl = __shfl_sync(0xFFFFFFFFu, t.incl, sp.e);
        sp.strips = __shfl_sync(0xFFFFFFFFu, t.cnt, sp.e);
        sp.start = incl - sp.strips;
        if constexpr (VARLEN) sp.base = __shfl_sync(0xFFFFFFFFu, t.base, sp.e);
    } else {
        uint32_t lo = 0, hi = experts;  // prefix[lo] <= s < prefix[hi]
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (t.prefix[mid] <= s) lo = mid; else hi = mid;
        }
        sp.e = lo;
        sp.start = t.prefix[lo];
        sp.strips = t.prefix[lo + 1] - sp.start;
        if constexpr (VARLEN) sp.base = t.prefix[experts + 1u + lo];
    }
    return sp;
}

// s / segs for s < 2^31 without a division instruction sequence (which costs
// about twenty instructions and an SFU operation per call): with l =
// ceil(log2 segs) >= 1, magic = ceil(2^(31 + l) / segs) < 2^32 and shift = l - 1,
// the quotient is umulhi(s, magic) >> shift.  Exact for every s < 2^31 because
// magic * segs - 2^(31 + l) < segs <= 2^l (Granlund and Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994, Theorem 4.2, with N = 31).
// segs == 1 has magic 0 and returns s.  The host computes magic and shift.
__device__ __forceinline__ uint32_t div_segs(uint32_t s, const Params &p) {
    return p.segs_magic == 0u ? s : (__umulhi(s, p.segs_magic) >> p.segs_shift);
}

// ---------------------------------------------------------------------------
// One chunk of up to ITEMS strips held in registers
// ---------------------------------------------------------------------------

template <int ITEMS, bool FUSED>
struct Chunk {
    uint32_t x[ITEMS][8];              // raw 16-bit pairs (gate when fused)
    uint32_t u[ITEMS][FUSED ? 8 : 1];  // up half when fused
    uint32_t e[ITEMS], row[ITEMS], col[ITEMS];
    uint32_t n;                        // strips in this chunk (warp-uniform)
};

// Issue the loads of strips [s, s + n) (n <= ITEMS).  Lanes past the end of a
// ragged row load nothing.  With flat dispatch (kFlat) the strip index maps
// to (row, strip-in-row) by one division; otherwise through the expert table.
template <int ITEMS, bool FUSED, int DISP>
__device__ __forceinline__ void load_chunk(Chunk<ITEMS, FUSED> &ch, uint32_t s, uint32_t n,
                                           const ExpertTable &t, const Params &p,
                                           uint32_t lane) {
    constexpr bool kVar = DISP == kVarlen || DISP == kMaskedSpec;   // the table holds first rows
    ch.n = n;
    uint32_t e = 0, start = 0, end_e = t.total, base = 0;
    if constexpr (DISP != kFlat) {
        const Span sp = locate<kVar>(t, p.experts, s);
        e = sp.e;
        start = sp.start;
        end_e = sp.start + sp.strips;
        base = sp.base;
    }
    uint32_t row = div_segs(s - start, p);
    uint32_t seg = (s - start) - row * p.segs;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        const bool live = static_cast<uint32_t>(k) < n;
        if constexpr (DISP != kFlat) {
            if (live && s + k >= end_e) {        // the chunk runs into the next expert
                const Span sp = locate<kVar>(t, p.experts, s + k);
                e = sp.e;
                start = sp.start;
                end_e = sp.start + sp.strips;
                base = sp.base;
                row = 0;
                seg = 0;
            }
        }
        ch.e[k] = e;
        ch.row[k] = base + row;             // varlen: the row in the packed buffer
        ch.col[k] = seg * kStripElems + lane * 16u;
        if (live && ch.col[k] < p.K) {
            const uint8_t *src = p.in + e * p.in_expert_bytes +
                                 static_cast<uint64_t>(ch.row[k]) * p.in_row_bytes +
                                 static_cast<uint64_t>(ch.col[k]) * 2u;
            load32B(src, ch.x[k]);
            if constexpr (FUSED) load32B(src + static_cast<uint64_t>(p.K) * 2u, ch.u[k]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ch.x[k][i] = 0u;
                if constexpr (FUSED) ch.u[k][i] = 0u;
            }
        }
        if (++seg == p.segs) {
            seg = 0;
            ++row;
        }
    }
}

// The speculative region of a small masked call (kMaskedSpec, at most 32
// experts): the first p.spec rows of every expert, strips in (expert, row,
// strip-in-row) order, loaded without waiting for masked_m.  Every address
// lies inside the expert's M rows (spec <= M); whether a row is live is
// decided after the loads, and dead rows are neither quantized nor written.
template <int ITEMS, bool FUSED>
__device__ __forceinline__ void load_spec_chunk(Chunk<ITEMS, FUSED> &ch, uint32_t s, uint32_t n,
                                                const Params &p, uint32_t lane) {
    ch.n = n;
    const uint32_t per_e = p.spec * p.segs;
    uint32_t e = p.spec_magic == 0u ? s : (__umulhi(s, p.spec_magic) >> p.spec_shift);
    const uint32_t r = s - e * per_e;
    uint32_t row = div_segs(r, p);
    uint32_t seg = r - row * p.segs;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        const bool live = static_cast<uint32_t>(k) < n;
        ch.e[k] = e;
        ch.row[k] = row;
        ch.col[k] = seg * kStripElems + lane * 16u;
        if (live && ch.col[k] < p.K) {
            const uint8_t *src = p.in + e * p.in_expert_bytes +
                                 static_cast<uint64_t>(row) * p.in_row_bytes +
                                 static_cast<uint64_t>(ch.col[k]) * 2u;
            load32B(src, ch.x[k]);
            if constexpr (FUSED) load32B(src + static_cast<uint64_t>(p.K) * 2u, ch.u[k]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ch.x[k][i] = 0u;
                if constexpr (FUSED) ch.u[k][i] = 0u;
            }
        }
        if (++seg == p.segs) {
            seg = 0;
            if (++row == p.spec) {
                row = 0;
                ++e;
            }
        }
    }
}

// bf16 UE8M0 through the mixed-precision FMA path (1) or by widening (0).
#ifndef PQG_UE8M0_MIXED
#define PQG_UE8M0_MIXED 1
#endif

// Quantize one strip held in registers and store its codes and scales.
template <typename In, int G, Kind KIND, bool FUSED>
__device__ __forceinline__ void quantize_strip(const uint32_t (&x)[8], const uint32_t *u,
                                               uint32_t e, uint32_t row, uint32_t col,
                                               const Params &p, uint32_t lane, const float *nv) {
    constexpr int L = G / 16;  // lanes per group
    const bool ok = col < p.K;
    const uint32_t g = col / G;  // group within the row (valid lanes)
    const uint32_t sub = lane % L;
    uint32_t w[4];
    GroupScale gs;

    constexpr bool kMixed = PQG_UE8M0_MIXED && is_ue8m0(KIND) && !FUSED &&
                            std::is_same<In, __nv_bfloat16>::value;
    if constexpr (kMixed) {
        // absmax on the raw bits, t = x * 2^k by a mixed bf16 FMA: no widening
        uint32_t ab = absmax_bits16(x);
#pragma unroll
        for (int o = 1; o < L; o <<= 1) ab = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, o));
        const float amax = fmaxf(__uint_as_float(ab << 16), 1e-10f);
        gs.e8 = KIND == Kind::E2M1_UE8M0 ? ue8m0_exponent_e2m1(amax) : ue8m0_exponent(amax);
        const uint16_t p2 = static_cast<uint16_t>((254u - gs.e8) << 7);  // bf16 2^(127-e)
        if constexpr (KIND == Kind::E2M1_UE8M0) {
            float t[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                t[2 * i] = mul_bf16_pow2(static_cast<uint16_t>(x[i] & 0xFFFFu), p2);
                t[2 * i + 1] = mul_bf16_pow2(static_cast<uint16_t>(x[i] >> 16), p2);
            }
            w[0] = e2m1x8(t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]);
            w[1] = e2m1x8(t[8], t[9], t[10], t[11], t[12], t[13], t[14], t[15]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t a = x[2 * j], b = x[2 * j + 1];
                const float t0 = mul_bf16_pow2(static_cast<uint16_t>(a & 0xFFFFu), p2);
                const float t1 = mul_bf16_pow2(static_cast<uint16_t>(a >> 16), p2);
                const float t2 = mul_bf16_pow2(static_cast<uint16_t>(b & 0xFFFFu), p2);
                const float t3 = mul_bf16_pow2(static_cast<uint16_t>(b >> 16), p2);
                w[j] = e4m3x4(t0, t1, t2, t3);
            }
        }
    } else {
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if constexpr (FUSED) {
                const float2 y = silu_mul_pair<In>(x[i], u[i]);
                v[2 * i] = y.x;
                v[2 * i + 1] = y.y;
            } else {
                widen2<In>(x[i], v[2 * i], v[2 * i + 1]);
            }
        }
        float amax = absmax16(v);
#pragma unroll
        for (int o = 1; o < L; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        gs = make_scale<KIND>(amax, nv);
        encode16<KIND>(v, gs, w);
    }

    uint32_t packed_word = 0;
    if constexpr (is_ue8m0(KIND)) {
        // little-endian word of groups 4j..4j+3 assembled across the 4 groups'
        // lanes (invalid groups contribute 0), for the layouts that store
        // words; the fused kernels skip the two shuffles for the byte layouts
        // (the plain ones keep them: the branch costs them registers)
        if (!FUSED || p.layout == kPacked || p.layout == kTiled128x4) {   // warp-uniform
            packed_word = ok ? (gs.e8 << (8u * (g & 3u))) : 0u;
            packed_word |= __shfl_xor_sync(0xFFFFFFFFu, packed_word, L);
            packed_word |= __shfl_xor_sync(0xFFFFFFFFu, packed_word, 2 * L);
        }
    }
    if (!ok) return;

    uint8_t *dst = p.out + e * p.out_expert_bytes + static_cast<uint64_t>(row) * p.out_row_bytes;
    if constexpr (is_e2m1(KIND))
        store8B(dst + col / 2u, w[0], w[1]);
    else
        store16B(dst + col, w[0], w[1], w[2], w[3]);
    if (sub == 0) {
        uint8_t *sc = p.scales + e * p.scale_expert_bytes;
        if (p.layout == kPacked) {
            if ((g & 3u) == 0u)
                reinterpret_cast<uint32_t *>(sc)[static_cast<uint64_t>(g >> 2) * p.mpad + row] =
                    packed_word;
        } else if (p.layout == kTiled128x4) {
            if constexpr (is_ue8m0(KIND)) {
                // groups 4j..4j+3 of the row are 4 consecutive bytes of one tile:
                // one word, its padding bytes already 0 (the buffer is 4-byte
                // aligned)
                if ((g & 3u) == 0u)
                    *reinterpret_cast<uint32_t *>(sc + tile128x4_offset(row, g, p.ng)) =
                        packed_word;
            } else {
                store_tiled(sc, row, g, p.ng, gs.e8);   // NVFP4 E4M3 block-scale bytes
            }
        } else {
            const uint64_t idx = (p.layout == kRowMajor) ? static_cast<uint64_t>(row) * p.ng + g
                                                         : static_cast<uint64_t>(g) * p.mpad + row;
            if constexpr (byte_scale(KIND))
                sc[idx] = static_cast<uint8_t>(gs.e8);
            else
                reinterpret_cast<float *>(sc)[idx] = gs.s;
        }
    }
}

template <typename In, int G, Kind KIND, bool FUSED, int ITEMS>
__device__ __forceinline__ void quantize_chunk(const Chunk<ITEMS, FUSED> &ch, const Params &p,
                                               uint32_t lane, const float *nv) {
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        if (static_cast<uint32_t>(k) >= ch.n) break;  // warp-uniform
        quantize_strip<In, G, KIND, FUSED>(ch.x[k], FUSED ? ch.u[k] : nullptr, ch.e[k],
                                           ch.row[k], ch.col[k], p, lane, nv);
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// Resident CTAs per SM the register allocation must allow (0: no constraint).
// The fp32-scale plain variants run best at 5 (they take 46-48 registers; a
// bound of 6 spills and was measured no better), flat NVFP4 at 6 (<= 40
// registers, no spills) and the fused ones at 8; the rest need no constraint.
#ifndef PQG_MIN_BLOCKS_FP32
#define PQG_MIN_BLOCKS_FP32 5
#endif
#ifndef PQG_MIN_BLOCKS_NVFP4
#define PQG_MIN_BLOCKS_NVFP4 6
#endif
// Fused kernels (4 warps per CTA) with one strip per chunk are held to 12
// resident CTAs (40 registers; the short [4096, 2 x 2048] call 8.80 -> 8.71 us).
// The 2-strip variants run best unbounded (65 registers, 7 CTAs): held to 8
// CTAs they were slower ([4096, 2 x 7168] 25.09 -> 25.60 us).
#ifndef PQG_MIN_BLOCKS_FUSED1
#define PQG_MIN_BLOCKS_FUSED1 12
#endif
#ifndef PQG_MIN_BLOCKS_FUSED2
#define PQG_MIN_BLOCKS_FUSED2 0
#endif
template <Kind KIND, bool FUSED, int DISP, int ITEMS>
constexpr int min_blocks() {
    if constexpr (FUSED) return ITEMS == 1 ? PQG_MIN_BLOCKS_FUSED1 : PQG_MIN_BLOCKS_FUSED2;
    if constexpr (KIND == Kind::E4M3_FP32 || KIND == Kind::INT8_FP32) return PQG_MIN_BLOCKS_FP32;
    if constexpr (KIND == Kind::E2M1_E4M3 && DISP == kFlat) return PQG_MIN_BLOCKS_NVFP4;
    return 0;
}

template <typename In, int G, Kind KIND, bool FUSED, int ITEMS, int WARPS, int DISP>
__global__ void __launch_bounds__(WARPS * 32, min_blocks<KIND, FUSED, DISP, ITEMS>())
    quant_kernel(const __grid_constant__ Params p) {
    static_assert((G == 32 || G == 64 || G == 128) == (KIND != Kind::E2M1_E4M3) &&
                      (G == 16) == (KIND == Kind::E2M1_E4M3),
                  "G is 32, 64 or 128, or 16 for NVFP4");
    static_assert(WARPS * 32 >= 128, "the NVFP4 table is built by 128 threads");
    extern __shared__ __align__(16) uint32_t smem_prefix[];
    __shared__ float nv[KIND == Kind::E2M1_E4M3 ? kNvTable : 1];

    wait_for_producer();                        // before the first global access
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    if constexpr (KIND == Kind::E2M1_E4M3) build_nvfp4_table(p, nv);
    ExpertTable t;
    if constexpr (DISP == kMaskedSpec) {
        // Small masked calls (decode): the rows every expert is expected to
        // have are loaded at once, in parallel with masked_m, instead of after
        // it; the rest of each expert's rows follow through the warp table.
        uint32_t live_rows = 0;                 // lane e: rows of expert e (E <= 32)
        if (lane < p.experts)
            live_rows = static_cast<uint32_t>(
                min(max(__ldg(p.masked_m + lane), 0), static_cast<int>(p.M)));
        const uint32_t items = p.items, block = WARPS * items;
        const uint32_t total_spec = p.experts * p.spec * p.segs;
        const uint32_t nblocks_spec = (total_spec + block - 1) / block;
        for (uint32_t blk = blockIdx.x; blk < nblocks_spec; blk += gridDim.x) {
            const uint32_t s = blk * block + warp * items;
            if (s >= total_spec) break;         // warp-uniform
            Chunk<ITEMS, FUSED> ch;
            load_spec_chunk<ITEMS, FUSED>(ch, s, min(items, total_spec - s), p, lane);
#pragma unroll
            for (int k = 0; k < ITEMS; ++k) {
                if (static_cast<uint32_t>(k) >= ch.n) break;   // warp-uniform
                const uint32_t rows = __shfl_sync(0xFFFFFFFFu, live_rows, ch.e[k]);
                if (ch.row[k] < rows)           // warp-uniform
                    quantize_strip<In, G, KIND, FUSED>(ch.x[k], FUSED ? ch.u[k] : nullptr,
                                                       ch.e[k], ch.row[k], ch.col[k], p, lane, nv);
            }
        }
        // rows [spec, live) of each expert: a warp table whose first row is spec
        t.mode = 1;
        t.prefix = nullptr;
        t.base = p.spec;
        t.cnt = lane < p.experts && live_rows > p.spec ? (live_rows - p.spec) * p.segs : 0u;
        uint32_t incl = t.cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= static_cast<uint32_t>(o)) incl += v;
        }
        t.incl = incl;
        t.total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    } else if constexpr (DISP != kFlat) {
        t = make_table<DISP == kVarlen>(p, smem_prefix, lane);
    } else {
        uint32_t first;
        t.total = expert_strips<false>(p, 0, first);
    }

    // Block-cyclic schedule: a block is WARPS x items consecutive strips, CTA
    // c takes blocks c, c + gridDim.x, ...; warp w takes the w-th `items`
    // strips of each block.  All CTAs sweep the address space together, which
    // keeps concurrent DRAM accesses close (row-buffer locality).
    const uint32_t items = p.items;             // 1 .. ITEMS (launch-time)
    const uint32_t block = WARPS * items;
    const uint32_t nblocks = (t.total + block - 1) / block;
    for (uint32_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
        const uint32_t s = blk * block + warp * items;
        if (s >= t.total) break;                // warp-uniform
        Chunk<ITEMS, FUSED> ch;
        load_chunk<ITEMS, FUSED, DISP>(ch, s, min(items, t.total - s), t, p, lane);
        quantize_chunk<In, G, KIND, FUSED, ITEMS>(ch, p, lane, nv);
    }
    release_dependents();
}

}  // namespace pqg
