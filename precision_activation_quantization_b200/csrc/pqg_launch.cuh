// Host-side launch of the quantization kernel family: picks the compile-time
// variant, sizes the grid and the dynamic shared memory, and launches with
// cudaLaunchKernelEx on the caller's stream (with the programmatic-dependent-
// launch attribute when enabled).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <type_traits>

#include "pqg_kernel.cuh"
#include "pqg_row_kernel.cuh"

namespace pqg {

// Everything the launcher needs, already validated by the C-ABI shim.
struct LaunchArgs {
    Params p;
    uint64_t expected_strips;  // strips the grid is sized for (all experts)
    uint64_t expected_rows;    // rows the grid is sized for (per-token kernel)
    int group;                 // 32 / 64 / 128, or K (per-token)
    Kind kind;
    int disp;                  // kFlat, kMasked, kVarlen or kMaskedSpec
    bool fused;
    bool pdl;
    cudaStream_t stream;
};

int sm_count(int device);  // cached cudaDevAttrMultiProcessorCount
void segs_divider(uint32_t segs, uint32_t *magic, uint32_t *shift);

// Resident CTAs per SM of one kernel variant, cached per device: the
// occupancy query (and the shared-memory attribute it needs) applies to the
// current device, so a process driving several devices queries each once.
constexpr int kOccDevices = 64;
struct OccupancyCache {
    std::atomic<int> n[kOccDevices][2];   // [device][0: no table, 1: largest table]; 0 = unknown
};

template <typename Kernel>
inline int blocks_per_sm(OccupancyCache &cache, Kernel kernel, int device, int threads,
                         uint32_t max_smem, uint32_t smem) {
    const int which = smem == 0 ? 0 : 1;
    const bool cached = device >= 0 && device < kOccDevices;
    if (cached) {
        const int n = cache.n[device][which].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(max_smem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads,
                                                      which ? max_smem : 0u) != cudaSuccess ||
        n < 1)
        n = 1;
    if (cached) cache.n[device][which].store(n, std::memory_order_relaxed);
    return n;
}

// Strips per register chunk (ITEMS) and warps per CTA, tunable at build time.
// Each lane issues ITEMS 32-byte loads (twice that fused) per chunk.
#ifndef PQG_ITEMS_PLAIN
#define PQG_ITEMS_PLAIN 2
#endif
#ifndef PQG_WARPS_PLAIN
#define PQG_WARPS_PLAIN 8
#endif
#ifndef PQG_WARPS_UE8M0
#define PQG_WARPS_UE8M0 4
#endif
#ifndef PQG_ITEMS_FUSED
#define PQG_ITEMS_FUSED 1
#endif
#ifndef PQG_ITEMS_FUSED_MULTI
#define PQG_ITEMS_FUSED_MULTI 2
#endif
// Fused calls run 4 warps per CTA (masked 51.65 -> 50.73 us; the short flat
// fused call 8.88 -> 8.83 us).
#ifndef PQG_WARPS_FUSED
#define PQG_WARPS_FUSED 4
#endif

// Grid cap in waves of resident CTAs, and the size (in waves of blocks) up to
// which a call runs as a single looping wave.
#ifndef PQG_WAVES
#define PQG_WAVES 8
#endif
#ifndef PQG_SHORT_WAVES
#define PQG_SHORT_WAVES 4
#endif


// Fused multi-expert (masked) calls take 2 strips per chunk: they are long
// enough for the deeper chunk to pay (masked 52.9 -> 51.5 us), while a short
// flat fused call loses warps with work (8.8 -> 9.7 us); long flat fused
// calls take 2 as well (launch_kind picks the variant by call length).
// Plain bf16 MXFP4 at G = 32 takes 3 strips per chunk (24.86 vs 25.11 us; it
// stays at 48 registers, where fp16 or G = 64/128 would need 55-62); NVFP4,
// bounded to 40 registers, loses with 3 (29.2 vs 25.3 us), and masked too.
#ifndef PQG_ITEMS_MXFP4
#define PQG_ITEMS_MXFP4 3
#endif
template <typename In, Kind KIND, int G, bool FUSED, bool MULTI>
struct Shape {   // MULTI: several experts (masked or varlen dispatch)
    static constexpr bool kMx32 = KIND == Kind::E2M1_UE8M0 && G == 32 &&
                                  std::is_same<In, __nv_bfloat16>::value;
    static constexpr int kItems = FUSED ? (MULTI ? PQG_ITEMS_FUSED_MULTI : PQG_ITEMS_FUSED)
                                        : (kMx32 ? PQG_ITEMS_MXFP4 : PQG_ITEMS_PLAIN);
    // plain UE8M0 kinds (FP8 and MXFP4) run 4 warps per CTA (flat 27.38 ->
    // 27.23 us, MXFP4 24.85 -> 24.50 us); fp32-scale kinds and NVFP4 lose with 4
    static constexpr int kWarps =
        FUSED ? PQG_WARPS_FUSED : (is_ue8m0(KIND) ? PQG_WARPS_UE8M0 : PQG_WARPS_PLAIN);
};

// Grid cap in waves of resident CTAs for a call of `blocks` blocks, by variant
// (measured on B200 at the bench workloads): UE8M0 FP8 and the fused kernels
// run best with up to PQG_WAVES waves; the FP4 kinds with 4; the fp32-scale
// plain kinds with 2, unless the call is long (>= 24 waves of blocks, e.g.
// the 65536-row sweeps), where 8 win again.
#ifndef PQG_WAVES_FP4
#define PQG_WAVES_FP4 4
#endif
#ifndef PQG_WAVES_FP32
#define PQG_WAVES_FP32 2
#endif
template <Kind KIND, bool FUSED>
inline uint64_t grid_waves(uint64_t blocks, uint64_t wave) {
    if (FUSED || KIND == Kind::E4M3_UE8M0) return PQG_WAVES;
    if (is_e2m1(KIND)) return PQG_WAVES_FP4;
    return blocks >= 24u * wave ? PQG_WAVES : PQG_WAVES_FP32;
}

// ITEMS_SEL > 0 overrides the variant's strips per chunk (the long flat fused
// calls, see launch_kind).
template <typename In, int G, Kind KIND, bool FUSED, int DISP, int ITEMS_SEL = 0>
cudaError_t launch_variant(const LaunchArgs &a) {
    using Sh = Shape<In, KIND, G, FUSED, DISP != kFlat>;
    constexpr int kItems = ITEMS_SEL > 0 ? ITEMS_SEL : Sh::kItems;
    constexpr int kWarps = Sh::kWarps;
    constexpr int kThreads = kWarps * 32;
    constexpr bool kVar = DISP == kVarlen;
    auto kernel = quant_kernel<In, G, KIND, FUSED, kItems, kWarps, DISP>;

    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) return err;
    // Resident CTAs per SM on this device, without or with the largest
    // shared-memory expert table (more than 32 experts).
    static OccupancyCache cache;
    const int bps = blocks_per_sm(cache, kernel, device, kThreads, smem_bytes(kMaxExperts, kVar),
                                  smem_bytes(a.p.experts, kVar));

    // Strips per warp: ITEMS, or 1 when the expected work would not fill one
    // wave (latency-bound calls spread over more SMs).  Grid: one CTA per
    // block of the expected work, but a short call (at most PQG_SHORT_WAVES
    // waves of blocks) runs one resident wave that loops over the blocks (no
    // ragged last wave), and a long one at most PQG_WAVES waves.  Blocks are
    // taken round-robin, so any real total is covered.
    const uint64_t wave = static_cast<uint64_t>(sm_count(device)) * bps;
    Params p = a.p;
    p.items = kItems;
    if (a.expected_strips < wave * kWarps * kItems) p.items = 1;
    const uint64_t per_cta = static_cast<uint64_t>(kWarps) * p.items;
    uint64_t ctas = (a.expected_strips + per_cta - 1) / per_cta;
    const uint64_t cap =
        ctas <= wave * PQG_SHORT_WAVES ? wave : wave * grid_waves<KIND, FUSED>(ctas, wave);
    if (ctas > cap) ctas = cap;
    if (ctas < 1) ctas = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes(a.p.experts, kVar);
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <typename In, int G, Kind KIND>
cudaError_t launch_kind(const LaunchArgs &a) {
    if (a.disp == kVarlen)
        return a.fused ? launch_variant<In, G, KIND, true, kVarlen>(a)
                       : launch_variant<In, G, KIND, false, kVarlen>(a);
    if (a.disp == kMaskedSpec)   // fused only (chosen by the caller)
        return launch_variant<In, G, KIND, true, kMaskedSpec>(a);
    const bool multi = a.p.experts > 1;
    if (a.fused) {
        if (multi) return launch_variant<In, G, KIND, true, kMasked>(a);
        // A long flat fused call (4 or more waves of 1-strip work at 48 warps
        // per SM) runs a variant compiled for 2 strips per chunk: [4096, 2 x
        // 7168] 26.4 -> 24.6 us.  Short calls keep the 1-strip variant, whose
        // lower register count holds more CTAs ([4096, 2 x 2048]: 8.8 us
        // against 10.4 us with the 2-strip build).
        int device = 0;
        cudaError_t err = cudaGetDevice(&device);
        if (err != cudaSuccess) return err;
        const uint64_t long_call = 4ull * static_cast<uint64_t>(sm_count(device)) * 48u;
        return a.expected_strips >= long_call ? launch_variant<In, G, KIND, true, kFlat, 2>(a)
                                              : launch_variant<In, G, KIND, true, kFlat>(a);
    }
    return multi ? launch_variant<In, G, KIND, false, kMasked>(a)
                 : launch_variant<In, G, KIND, false, kFlat>(a);
}

template <typename In, int G>
cudaError_t launch_group(const LaunchArgs &a) {
    switch (a.kind) {
        case Kind::E4M3_FP32: return launch_kind<In, G, Kind::E4M3_FP32>(a);
        case Kind::E4M3_UE8M0: return launch_kind<In, G, Kind::E4M3_UE8M0>(a);
        case Kind::INT8_FP32: return launch_kind<In, G, Kind::INT8_FP32>(a);
        case Kind::E2M1_UE8M0: return launch_kind<In, G, Kind::E2M1_UE8M0>(a);
        case Kind::E2M1_E4M3: break;  // G = 16 only (launch_dtype)
    }
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Per-token (G = K) launches
// ---------------------------------------------------------------------------

// Grid cap of the per-token kernel in waves of resident CTAs: one resident
// wave whose CTAs loop over rows (measured 3.7% faster than 8 waves at
// [8192, 7168]).
#ifndef PQG_ROW_WAVES
#define PQG_ROW_WAVES 1
#endif

// Warps sharing a row and 16-element slots per thread for a row of K outputs:
// slots grow to PQG_ROW_SLOTS before warps are added (K = 7168: 4 warps per
// row, 4 slots, 2 rows per CTA iteration; measured 31.3 vs 32.3 us for 8 warps
// x 2 slots once the kernel ran in one wave).
#ifndef PQG_ROW_SLOTS
#define PQG_ROW_SLOTS 4
#endif
inline void row_shape(uint32_t K, uint32_t *wpr, int *slots) {
    const uint32_t nslots = K / 16u;
    const uint32_t cap = PQG_ROW_SLOTS;
    *slots = 1;
    *wpr = 1;
    while (*wpr * 32u * static_cast<uint32_t>(*slots) < nslots) {
        if (static_cast<uint32_t>(*slots) < cap) *slots *= 2;
        else if (*wpr < 8u) *wpr *= 2;
        else *slots *= 2;  // K > 256 * 16 * cap: up to 4 slots
    }
}

template <typename In, Kind KIND, bool FUSED, int SLOTS, bool VARLEN>
cudaError_t launch_row_variant(const LaunchArgs &a, uint32_t wpr) {
    auto kernel = row_quant_kernel<In, KIND, FUSED, SLOTS, VARLEN>;
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) return err;
    // sized with the largest expert table, whatever this call's table
    static OccupancyCache cache;
    const int bps = blocks_per_sm(cache, kernel, device, kRowThreads,
                                  smem_bytes(kMaxExperts, VARLEN), smem_bytes(kMaxExperts, VARLEN));

    Params p = a.p;
    p.segs = 1;        // the expert table counts rows
    p.segs_magic = 0;  // (no strip division)
    p.segs_shift = 0;
    p.items = wpr;     // warps per row
    const uint64_t rows_per_cta = (kRowThreads / 32) / wpr;
    uint64_t ctas = (a.expected_rows + rows_per_cta - 1) / rows_per_cta;
    const uint64_t cap = static_cast<uint64_t>(sm_count(device)) * bps * PQG_ROW_WAVES;
    if (ctas > cap) ctas = cap;
    if (ctas < 1) ctas = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.blockDim = dim3(kRowThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes(a.p.experts, VARLEN);
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <typename In, Kind KIND, bool FUSED, bool VARLEN>
cudaError_t launch_row_slots(const LaunchArgs &a) {
    uint32_t wpr = 1;
    int slots = 1;
    row_shape(a.p.K, &wpr, &slots);
    switch (slots) {
        case 1: return launch_row_variant<In, KIND, FUSED, 1, VARLEN>(a, wpr);
        case 2: return launch_row_variant<In, KIND, FUSED, 2, VARLEN>(a, wpr);
        default: return launch_row_variant<In, KIND, FUSED, 4, VARLEN>(a, wpr);
    }
}

template <typename In, Kind KIND, bool FUSED>
cudaError_t launch_row_kind(const LaunchArgs &a) {
    return a.disp == kVarlen ? launch_row_slots<In, KIND, FUSED, true>(a)
                             : launch_row_slots<In, KIND, FUSED, false>(a);
}

template <typename In>
cudaError_t launch_row(const LaunchArgs &a) {
    switch (a.kind) {
        case Kind::E4M3_FP32:
            return a.fused ? launch_row_kind<In, Kind::E4M3_FP32, true>(a)
                           : launch_row_kind<In, Kind::E4M3_FP32, false>(a);
        case Kind::E4M3_UE8M0:
            return a.fused ? launch_row_kind<In, Kind::E4M3_UE8M0, true>(a)
                           : launch_row_kind<In, Kind::E4M3_UE8M0, false>(a);
        case Kind::INT8_FP32:
            return a.fused ? launch_row_kind<In, Kind::INT8_FP32, true>(a)
                           : launch_row_kind<In, Kind::INT8_FP32, false>(a);
        case Kind::E2M1_UE8M0:
        case Kind::E2M1_E4M3:
            break;  // rejected by the caller: FP4 groups are 16 (NVFP4) or 32/64/128
    }
    return cudaErrorInvalidValue;
}

template <typename In>
cudaError_t launch_dtype(const LaunchArgs &a) {
    if (a.kind == Kind::E2M1_E4M3)
        return a.group == 16 ? launch_kind<In, 16, Kind::E2M1_E4M3>(a) : cudaErrorInvalidValue;
    switch (a.group) {
        case 32: return launch_group<In, 32>(a);
        case 64: return launch_group<In, 64>(a);
        case 128: return launch_group<In, 128>(a);
    }
    return launch_row<In>(a);   // per-token: group == K (checked by the caller)
}

cudaError_t launch_bf16(const LaunchArgs &a);
cudaError_t launch_fp16(const LaunchArgs &a);

}  // namespace pqg
