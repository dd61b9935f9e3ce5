// Host-side launch of the quantization kernel family: picks the compile-time
// variant, sizes the grid and launches with cudaLaunchKernelEx on the caller's
// stream (with the programmatic-dependent-launch attribute when enabled).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "pqg_kernel.cuh"

namespace pqg {

// Everything the launcher needs, already validated by the C-ABI shim.
struct LaunchArgs {
    Params p;
    uint32_t experts;       // grid.y
    uint32_t grid_rows;     // rows per expert the grid is sized for
    int group;              // 32 / 64 / 128
    Kind kind;
    bool fused;
    bool pdl;
    cudaStream_t stream;
};

int sm_count(int device);  // cached cudaDevAttrMultiProcessorCount

// Strips each warp takes per iteration: each lane keeps this many 32-byte
// loads in flight (twice as many when fused).  Tunable at build time.
#ifndef PQG_ITEMS_PLAIN
#define PQG_ITEMS_PLAIN 2
#endif
#ifndef PQG_ITEMS_FUSED
#define PQG_ITEMS_FUSED 2
#endif
template <bool FUSED>
constexpr int items_per_warp() {
    return FUSED ? PQG_ITEMS_FUSED : PQG_ITEMS_PLAIN;
}

template <typename In, int G, Kind KIND, bool FUSED>
cudaError_t launch_variant(const LaunchArgs &a) {
    constexpr int ITEMS = items_per_warp<FUSED>();
    auto kernel = quant_kernel<In, G, KIND, FUSED, ITEMS>;

    // resident CTAs per SM for this variant (queried once per variant)
    static const int blocks_per_sm = [&] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) !=
                cudaSuccess ||
            n < 1)
            n = 1;
        return n;
    }();

    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) return err;

    // One wave of resident CTAs at most; fewer when the work is small, so that
    // every warp has at least ITEMS strips.
    const uint64_t strips = static_cast<uint64_t>(a.grid_rows) * a.p.segs;
    const uint64_t per_cta = static_cast<uint64_t>(kWarps) * ITEMS;
    uint64_t ctas = (strips + per_cta - 1) / per_cta;
    uint64_t wave = static_cast<uint64_t>(sm_count(device)) * blocks_per_sm;
    if (a.experts > 1) wave = (wave + a.experts - 1) / a.experts;
    if (ctas > wave) ctas = wave;
    if (ctas < 1) ctas = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), a.experts, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, a.p);
}

template <typename In, int G>
cudaError_t launch_group(const LaunchArgs &a) {
    switch (a.kind) {
        case Kind::E4M3_FP32:
            return a.fused ? launch_variant<In, G, Kind::E4M3_FP32, true>(a)
                           : launch_variant<In, G, Kind::E4M3_FP32, false>(a);
        case Kind::E4M3_UE8M0:
            return a.fused ? launch_variant<In, G, Kind::E4M3_UE8M0, true>(a)
                           : launch_variant<In, G, Kind::E4M3_UE8M0, false>(a);
        case Kind::INT8_FP32:
            return a.fused ? launch_variant<In, G, Kind::INT8_FP32, true>(a)
                           : launch_variant<In, G, Kind::INT8_FP32, false>(a);
    }
    return cudaErrorInvalidValue;
}

template <typename In>
cudaError_t launch_dtype(const LaunchArgs &a) {
    switch (a.group) {
        case 32: return launch_group<In, 32>(a);
        case 64: return launch_group<In, 64>(a);
        case 128: return launch_group<In, 128>(a);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_bf16(const LaunchArgs &a);
cudaError_t launch_fp16(const LaunchArgs &a);

}  // namespace pqg
