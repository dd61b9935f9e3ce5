// Per-token-group quantization kernels for sm_100a.
//
// One kernel body, specialised at compile time on what changes the inner loop:
// input dtype, group size G, output/scale kind (E4M3 + fp32 scale, E4M3 +
// UE8M0 scale, INT8 + fp32 scale) and the fused SiLU-and-mul prologue.  What
// changes only once per group (the scale layout) or once per CTA (flat or
// masked dispatch) is a runtime field of the parameter block.  The variant axes
// are those of the sglang PR #30924 report, "[JIT] Trait-driven
// per_token_group_quant", 实现拆解 item 1; the arithmetic is its 关键源码片段
// (ref_fp8_ue8m0) and 风险与影响 (INT8, amax / 127).
//
// Work decomposition.  A "strip" is 32 lanes x 16 elements = 512 consecutive
// outputs of one row, so each lane owns 16 outputs (32 bytes of bf16/fp16
// input, read with one 256-bit load; the report's 执行摘要 names the same 32 B
// per lane tiling).  A 1 x G group spans L = G/16 adjacent lanes; its absmax is
// a log2(L)-step xor-shuffle.  Each warp takes ITEMS consecutive strips per
// iteration and issues all their loads before any arithmetic, so every lane has
// ITEMS (x2 when fused) independent 32-byte loads in flight.  Rows whose width
// is not a multiple of 512 leave the tail lanes of their last strip idle.
//
// Exact division.  Codes must equal a rounding of fp32(x / s).  A per-element
// IEEE division is too slow for a bandwidth-bound loop, so the quotient is
// formed from y = RN(1/s) (one correctly rounded reciprocal per group) and two
// residual corrections, q <- q + (x - q*s) * y with exact FMA residuals
// (Markstein's correction; P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  The
// first step leaves q within an ulp of x/s, and the second then returns the
// correctly rounded quotient.  Where |x/s| < 2^-12 the residual may underflow,
// but every such t rounds to a signed zero code, and the sign is restored from
// x.  The correction runs on packed f32x2 FMAs (FFMA2), two elements per
// instruction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace pqg {

enum class Kind : int { E4M3_FP32 = 0, E4M3_UE8M0 = 1, INT8_FP32 = 2 };

// Runtime scale layouts (same numbering as the C ABI's pqg_scale_layout).
enum : uint32_t { kRowMajor = 0, kColMajor = 1, kPacked = 2 };

constexpr int kWarps = 8;                  // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kStripElems = 512;           // outputs per strip (32 lanes x 16)

struct Params {
    const uint8_t *in;         // expert 0, row 0
    uint8_t *out;              // expert 0, row 0
    uint8_t *scales;           // expert 0's scale plane (byte address)
    const int32_t *masked_m;   // device int32[E], or null: all M rows
    int64_t in_expert_bytes;   // M * in_row_bytes
    int64_t out_expert_bytes;  // M * K
    int64_t scale_expert_bytes;
    uint32_t M;                // rows per expert (capacity when masked)
    uint32_t K;                // outputs per row
    uint32_t in_row_bytes;     // 2K (plain) or 4K (fused), in bytes
    uint32_t ng;               // groups per row
    uint32_t segs;             // strips per row = ceil(K / 512)
    uint32_t mpad;             // rows of a column-major plane (M rounded up to 4)
    uint32_t layout;           // kRowMajor / kColMajor / kPacked
};

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

__device__ __forceinline__ void store16B(void *p, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's memory before the
// first global access; let the next grid start its prologue when we are done.
__device__ __forceinline__ void wait_for_producer() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
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

// silu(g) * u in fp32, silu(g) = g * sigmoid(g).  With e = exp(-|g|) in (0, 1],
// sigmoid(g) is 1/(1+e) for g >= 0 and e/(1+e) for g < 0, so neither the
// exponential nor the reciprocal (of a value in [1, 2]) can overflow.  exp is
// the hardware ex2 approximation and the reciprocal rcp.approx; the product
// stays within a few fp32 ulps of silu(g) * u.
__device__ __forceinline__ float silu_mul(float g, float u) {
    const float e = __expf(-fabsf(g));
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
    const float sig = g >= 0.0f ? r : e * r;
    return g * sig * u;
}

// Packed pair of E4M3 codes: `lo` in bits 0-7, `hi` in bits 8-15.  Round to
// nearest even; satfinite clamps to +-448 (never reached: |t| <= 448 here).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// The correctly rounded fp32 quotient x/s for a pair, from y = RN(1/s) and
// ns = -s (two Markstein corrections; see the file comment).
__device__ __forceinline__ float2 div_rn2(float2 x, float2 y, float2 ns) {
    float2 q = __fmul2_rn(x, y);
    float2 r = __ffma2_rn(q, ns, x);   // x - q*s, exact
    q = __ffma2_rn(r, y, q);
    r = __ffma2_rn(q, ns, x);
    q = __ffma2_rn(r, y, q);
    return q;
}

// t keeps the sign of x: differs from q only when q is a zero of the wrong sign.
__device__ __forceinline__ float with_sign_of(float q, float x) {
    return __uint_as_float(__float_as_uint(q) | (__float_as_uint(x) & 0x80000000u));
}

// ---------------------------------------------------------------------------
// Per-group scale math (one group per L lanes; all lanes compute it)
// ---------------------------------------------------------------------------

struct GroupScale {
    float mult;   // UE8M0: 2^(127-e) (exact); fp32 kinds: y = RN(1/s)
    float neg_s;  // fp32 kinds: -s
    float s;      // fp32 kinds: the stored scale
    uint32_t e8;  // UE8M0: the stored exponent byte
};

template <Kind KIND>
__device__ __forceinline__ GroupScale make_scale(float amax) {
    GroupScale gs;
    amax = fmaxf(amax, 1e-10f);   // EPS floor
    if constexpr (KIND == Kind::E4M3_UE8M0) {
        const float raw = __fdiv_rn(amax, 448.0f);
        const uint32_t b = __float_as_uint(raw);
        gs.e8 = ((b >> 23) & 0xFFu) + ((b & 0x7FFFFFu) != 0u);
        gs.mult = __uint_as_float((254u - gs.e8) << 23);
        gs.s = 0.0f;
        gs.neg_s = 0.0f;
    } else {
        gs.s = __fdiv_rn(amax, KIND == Kind::INT8_FP32 ? 127.0f : 448.0f);
        gs.mult = __frcp_rn(gs.s);
        gs.neg_s = -gs.s;
        gs.e8 = 0;
    }
    return gs;
}

// 16 values -> 16 code bytes (4 words, element 0 in the lowest byte).
template <Kind KIND>
__device__ __forceinline__ void encode16(const float (&v)[16], const GroupScale &gs,
                                         uint32_t (&w)[4]) {
    if constexpr (KIND == Kind::E4M3_UE8M0) {
        const float2 m2 = make_float2(gs.mult, gs.mult);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // multiplying by a power of two is exact: t = x / s
            float2 a = __fmul2_rn(make_float2(v[4 * j], v[4 * j + 1]), m2);
            float2 b = __fmul2_rn(make_float2(v[4 * j + 2], v[4 * j + 3]), m2);
            w[j] = e4m3x2(a.x, a.y) | (e4m3x2(b.x, b.y) << 16);
        }
    } else if constexpr (KIND == Kind::E4M3_FP32) {
        const float2 y2 = make_float2(gs.mult, gs.mult);
        const float2 ns2 = make_float2(gs.neg_s, gs.neg_s);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 xa = make_float2(v[4 * j], v[4 * j + 1]);
            float2 xb = make_float2(v[4 * j + 2], v[4 * j + 3]);
            float2 a = div_rn2(xa, y2, ns2);
            float2 b = div_rn2(xb, y2, ns2);
            w[j] = e4m3x2(with_sign_of(a.x, xa.x), with_sign_of(a.y, xa.y)) |
                   (e4m3x2(with_sign_of(b.x, xb.x), with_sign_of(b.y, xb.y)) << 16);
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
            float2 a = __fadd2_rn(div_rn2(make_float2(v[4 * j], v[4 * j + 1]), y2, ns2), magic);
            float2 b =
                __fadd2_rn(div_rn2(make_float2(v[4 * j + 2], v[4 * j + 3]), y2, ns2), magic);
            uint32_t ab = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040);
            uint32_t cd = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040);
            w[j] = __byte_perm(ab, cd, 0x5410);
        }
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

template <typename In, int G, Kind KIND, bool FUSED, int ITEMS>
__global__ void __launch_bounds__(kThreads) quant_kernel(const __grid_constant__ Params p) {
    constexpr int L = G / 16;                   // lanes per group
    static_assert(L >= 2 && L <= 8 && (L & (L - 1)) == 0, "G must be 32, 64 or 128");

    wait_for_producer();

    const uint32_t expert = blockIdx.y;
    uint32_t rows = p.M;
    if (p.masked_m != nullptr) {
        const int mm = __ldg(p.masked_m + expert);
        rows = static_cast<uint32_t>(min(max(mm, 0), static_cast<int>(p.M)));
    }
    const uint32_t total = rows * p.segs;       // strips of this expert
    const uint8_t *in = p.in + expert * p.in_expert_bytes;
    uint8_t *out = p.out + expert * p.out_expert_bytes;
    uint8_t *sc = p.scales + expert * p.scale_expert_bytes;

    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t sub = lane % L;              // lane within its group

    // Each warp owns an equal contiguous share [begin, end) of this expert's
    // strips, so a one-wave grid finishes together (no partial last wave).
    const uint64_t nwarps = static_cast<uint64_t>(gridDim.x) * kWarps;
    const uint64_t wid = static_cast<uint64_t>(blockIdx.x) * kWarps + warp;
    const uint32_t begin = static_cast<uint32_t>(wid * total / nwarps);
    const uint32_t end = static_cast<uint32_t>((wid + 1) * total / nwarps);

    uint32_t r0 = begin / p.segs;               // row and strip-in-row of s0
    uint32_t sg0 = begin - r0 * p.segs;
    for (uint32_t s0 = begin; s0 < end; s0 += ITEMS) {
        uint32_t xr[ITEMS][8];
        uint32_t ur[ITEMS][FUSED ? 8 : 1];
        uint32_t row[ITEMS], col[ITEMS];
        bool ok[ITEMS];

        // -- issue every load of this iteration first ------------------------
#pragma unroll
        for (int k = 0; k < ITEMS; ++k) {
            row[k] = r0;
            col[k] = sg0 * kStripElems + lane * 16u;
            ok[k] = (s0 + k < end) && (col[k] < p.K);
            if (++sg0 == p.segs) {              // warp-uniform carry into the next row
                sg0 = 0;
                ++r0;
            }
            if (ok[k]) {
                const uint8_t *src = in + static_cast<uint64_t>(row[k]) * p.in_row_bytes +
                                     static_cast<uint64_t>(col[k]) * 2u;
                load32B(src, xr[k]);
                if constexpr (FUSED) load32B(src + static_cast<uint64_t>(p.K) * 2u, ur[k]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    xr[k][i] = 0u;
                    if constexpr (FUSED) ur[k][i] = 0u;
                }
            }
        }

        // -- then the arithmetic, strip by strip ------------------------------
#pragma unroll
        for (int k = 0; k < ITEMS; ++k) {
            if (s0 + k >= end) break;           // warp-uniform
            float v[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                widen2<In>(xr[k][i], v[2 * i], v[2 * i + 1]);
                if constexpr (FUSED) {
                    float u0, u1;
                    widen2<In>(ur[k][i], u0, u1);
                    v[2 * i] = silu_mul(v[2 * i], u0);
                    v[2 * i + 1] = silu_mul(v[2 * i + 1], u1);
                }
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int o = 1; o < L; o <<= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));

            const GroupScale gs = make_scale<KIND>(amax);
            uint32_t w[4];
            encode16<KIND>(v, gs, w);

            // group index within the row; every lane of a group agrees on it
            const uint32_t g = col[k] / G;
            uint32_t packed_word = 0;
            if constexpr (KIND == Kind::E4M3_UE8M0) {
                // assemble the little-endian word of groups 4j..4j+3 across the
                // 4 groups' lanes (invalid groups contribute 0)
                packed_word = ok[k] ? (gs.e8 << (8u * (g & 3u))) : 0u;
                packed_word |= __shfl_xor_sync(0xFFFFFFFFu, packed_word, L);
                packed_word |= __shfl_xor_sync(0xFFFFFFFFu, packed_word, 2 * L);
            }
            if (!ok[k]) continue;

            store16B(out + static_cast<uint64_t>(row[k]) * p.K + col[k], w[0], w[1], w[2], w[3]);

            if (sub == 0) {
                const uint32_t r = row[k];
                if (p.layout == kPacked) {
                    if ((g & 3u) == 0u) {
                        uint32_t *W = reinterpret_cast<uint32_t *>(sc);
                        W[static_cast<uint64_t>(g >> 2) * p.mpad + r] = packed_word;
                    }
                } else {
                    const uint64_t idx = (p.layout == kRowMajor)
                                             ? static_cast<uint64_t>(r) * p.ng + g
                                             : static_cast<uint64_t>(g) * p.mpad + r;
                    if constexpr (KIND == Kind::E4M3_UE8M0)
                        sc[idx] = static_cast<uint8_t>(gs.e8);
                    else
                        reinterpret_cast<float *>(sc)[idx] = gs.s;
                }
            }
        }
    }
    release_dependents();
}

}  // namespace pqg
