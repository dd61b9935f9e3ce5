// C ABI of libpqg.so (declared in include/pqg.h): argument validation, scale
// buffer geometry and dispatch into the kernel family.
//
// Every argument is checked on the host before anything is launched.  This
// guards against the failure mode the sglang PR #30924 report (评论区精华 and
// 风险与影响) records for its predecessor: negative dimension indices passed to
// size_t accessors.  The library allocates nothing and never synchronizes.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "pqg.h"
#include "pqg_launch.cuh"

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_pdl{1};
std::atomic<uint64_t> g_launches{0};

constexpr int64_t kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
int64_t padded_rows(int64_t M) { return (M + 3) / 4 * 4; }

constexpr int64_t kMaxPerTokenK = 16384;
constexpr int64_t kMaxSpecRows = 8;   // expected_m up to which masked calls load rows speculatively

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks the enum values and sizes shared by pqg_quant and pqg_scales_bytes,
// and returns the bytes of one expert's scale plane through *plane.
int check_geometry(int64_t num_experts, int64_t M, int64_t K, int group, int scale_fmt,
                   int scale_layout, int64_t *plane) {
    if (scale_fmt != PQG_SCALE_FP32 && scale_fmt != PQG_SCALE_UE8M0 &&
        scale_fmt != PQG_SCALE_E4M3)
        return PQG_ERR_INVALID_ARG;
    if (scale_layout != PQG_ROW_MAJOR && scale_layout != PQG_COL_MAJOR_TMA &&
        scale_layout != PQG_UE8M0_PACKED && scale_layout != PQG_UE8M0_TILED_128x4)
        return PQG_ERR_INVALID_ARG;
    if (group <= 0) return PQG_ERR_INVALID_ARG;
    if (scale_fmt == PQG_SCALE_E4M3) {
        // NVFP4: blocks of 16, byte scales, no packed words
        if (group != 16 || scale_layout == PQG_UE8M0_PACKED) return PQG_ERR_UNSUPPORTED;
    } else {
        // G in {32, 64, 128}, or one group per row (per-token, K <= 16384)
        const bool per_token = group == K && K % 16 == 0 && K <= kMaxPerTokenK;
        if (group != 32 && group != 64 && group != 128 && !per_token) return PQG_ERR_UNSUPPORTED;
        if ((scale_layout == PQG_UE8M0_PACKED || scale_layout == PQG_UE8M0_TILED_128x4) &&
            scale_fmt != PQG_SCALE_UE8M0)
            return PQG_ERR_UNSUPPORTED;
    }
    if (num_experts < 1 || num_experts > static_cast<int64_t>(pqg::kMaxExperts))
        return PQG_ERR_INVALID_ARG;
    if (M < 0 || K <= 0 || K % group != 0) return PQG_ERR_INVALID_ARG;
    // 2K-byte (4K fused) rows must fit the 32-bit row stride; strips per expert
    // must fit a 32-bit index.
    if (K > (int64_t{1} << 28)) return PQG_ERR_INVALID_ARG;
    const int64_t segs = (K + pqg::kStripElems - 1) / pqg::kStripElems;
    if (M > 0 && M >= (int64_t{1} << 31) / (segs * num_experts)) return PQG_ERR_INVALID_ARG;
    if (M * K > (int64_t{1} << 40) / num_experts) return PQG_ERR_INVALID_ARG;

    const int64_t ng = K / group;
    const int64_t elem = scale_fmt == PQG_SCALE_FP32 ? 4 : 1;
    if (scale_layout == PQG_ROW_MAJOR)
        *plane = M * ng * elem;
    else if (scale_layout == PQG_COL_MAJOR_TMA)
        *plane = ng * padded_rows(M) * elem;
    else if (scale_layout == PQG_UE8M0_PACKED)
        *plane = (ng + 3) / 4 * padded_rows(M) * 4;
    else
        *plane = (M + 127) / 128 * ((ng + 3) / 4) * 512;
    return PQG_OK;
}

bool overlaps(const void *a, int64_t na, const void *b, int64_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(nb) && b0 < a0 + static_cast<uintptr_t>(na);
}

}  // namespace

namespace pqg {
// magic and shift of div_segs (pqg_kernel.cuh): l = ceil(log2 segs),
// magic = ceil(2^(31 + l) / segs), shift = l - 1; segs == 1 gives magic 0.
void segs_divider(uint32_t segs, uint32_t *magic, uint32_t *shift) {
    if (segs <= 1u) {
        *magic = 0u;
        *shift = 0u;
        return;
    }
    uint32_t l = 0;
    while ((1ull << l) < segs) ++l;
    *magic = static_cast<uint32_t>(((1ull << (31u + l)) + segs - 1u) / segs);
    *shift = l - 1u;
}

int sm_count(int device) {
    if (device < 0 || device >= kMaxDevices) device = 0;
    int n = g_sm_count[device].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
            n <= 0)
            n = 1;
        g_sm_count[device].store(n, std::memory_order_relaxed);
    }
    return n;
}
}  // namespace pqg

namespace {

// Varlen (grouped-contiguous) segments: E + 1 row offsets and E token counts
// (or none), all on the device.
struct Segments {
    const int32_t *indptr;
    const int32_t *lens;
};

// Validation and launch shared by pqg_quant, pqg_quant_nvfp4 and
// pqg_quant_varlen (seg.indptr != nullptr: M packed rows in num_experts
// segments, one scale plane).
int quant_impl(const void *in, void *out, void *scales, const float *global_scale, int64_t M,
               int64_t num_experts, int64_t K, int group, int in_dtype, int out_dtype,
               int scale_fmt, int scale_layout, int fuse_silu_mul, const int32_t *masked_m,
               int64_t expected_m, pqg_stream_t stream, Segments seg = {nullptr, nullptr}) {
    const bool varlen = seg.indptr != nullptr;
    if (in_dtype != PQG_BF16 && in_dtype != PQG_FP16) return PQG_ERR_INVALID_ARG;
    if (out_dtype != PQG_E4M3 && out_dtype != PQG_INT8 && out_dtype != PQG_E2M1)
        return PQG_ERR_INVALID_ARG;
    if (varlen && (num_experts < 1 || num_experts > static_cast<int64_t>(pqg::kMaxExperts)))
        return PQG_ERR_INVALID_ARG;
    // a varlen call is one buffer of M rows: its geometry is that of one expert
    const int64_t planes = varlen ? 1 : num_experts;
    int64_t plane = 0;
    const int st = check_geometry(planes, M, K, group, scale_fmt, scale_layout, &plane);
    if (st != PQG_OK) return st;
    const bool nvfp4 = scale_fmt == PQG_SCALE_E4M3;
    if (scale_fmt == PQG_SCALE_UE8M0 && out_dtype == PQG_INT8) return PQG_ERR_UNSUPPORTED;
    if (out_dtype == PQG_E2M1 && !nvfp4 &&
        (scale_fmt != PQG_SCALE_UE8M0 || (group != 32 && group != 64 && group != 128)))
        return PQG_ERR_UNSUPPORTED;  // MXFP4: UE8M0 scales, groups of 32/64/128
    if (M == 0) return PQG_OK;

    if (in == nullptr || out == nullptr || scales == nullptr) return PQG_ERR_INVALID_ARG;
    if (nvfp4 && global_scale == nullptr) return PQG_ERR_INVALID_ARG;
    if (!aligned(in, 32) || !aligned(out, 16)) return PQG_ERR_ALIGNMENT;
    if (nvfp4 && !aligned(global_scale, 4)) return PQG_ERR_ALIGNMENT;
    if (scale_fmt == PQG_SCALE_FP32 || scale_layout == PQG_UE8M0_PACKED ||
        scale_layout == PQG_UE8M0_TILED_128x4) {
        if (!aligned(scales, 4)) return PQG_ERR_ALIGNMENT;  // word stores
    }
    if (masked_m != nullptr && !aligned(masked_m, 4)) return PQG_ERR_ALIGNMENT;
    if (varlen && (!aligned(seg.indptr, 4) || (seg.lens != nullptr && !aligned(seg.lens, 4))))
        return PQG_ERR_ALIGNMENT;

    const int64_t in_row_bytes = K * 2 * (fuse_silu_mul ? 2 : 1);
    const int64_t in_bytes = planes * M * in_row_bytes;
    const int64_t out_row_bytes = out_dtype == PQG_E2M1 ? K / 2 : K;
    const int64_t out_bytes = planes * M * out_row_bytes;
    if (overlaps(in, in_bytes, out, out_bytes) || overlaps(in, in_bytes, scales, plane * planes) ||
        overlaps(out, out_bytes, scales, plane * planes))
        return PQG_ERR_INVALID_ARG;
    if (varlen) {
        // the segment tables are read by every CTA: no output may overwrite them
        const int64_t ib = 4 * (num_experts + 1), lb = seg.lens != nullptr ? 4 * num_experts : 0;
        if (overlaps(seg.indptr, ib, out, out_bytes) || overlaps(seg.indptr, ib, scales, plane) ||
            overlaps(seg.lens, lb, out, out_bytes) || overlaps(seg.lens, lb, scales, plane))
            return PQG_ERR_INVALID_ARG;
    }

    pqg::LaunchArgs a;
    a.p.in = static_cast<const uint8_t *>(in);
    a.p.out = static_cast<uint8_t *>(out);
    a.p.scales = static_cast<uint8_t *>(scales);
    a.p.masked_m = varlen ? nullptr : masked_m;
    a.p.seg_indptr = seg.indptr;
    a.p.seg_lens = seg.lens;
    a.p.gscale = global_scale;
    // varlen segments address the one packed buffer by their own row offsets
    a.p.in_expert_bytes = varlen ? 0 : M * in_row_bytes;
    a.p.out_expert_bytes = varlen ? 0 : M * out_row_bytes;
    a.p.out_row_bytes = static_cast<uint32_t>(out_row_bytes);
    a.p.scale_expert_bytes = varlen ? 0 : plane;
    a.p.M = static_cast<uint32_t>(M);
    a.p.K = static_cast<uint32_t>(K);
    a.p.in_row_bytes = static_cast<uint32_t>(in_row_bytes);
    a.p.ng = static_cast<uint32_t>(K / group);
    a.p.segs = static_cast<uint32_t>((K + pqg::kStripElems - 1) / pqg::kStripElems);
    pqg::segs_divider(a.p.segs, &a.p.segs_magic, &a.p.segs_shift);
    a.p.mpad = static_cast<uint32_t>(padded_rows(M));
    a.p.layout = static_cast<uint32_t>(scale_layout);
    a.p.experts = static_cast<uint32_t>(num_experts);
    // rows the grid is sized for: every expert's expected_m when masked, or
    // (varlen) num_experts * expected_m tokens, at most the M packed rows
    int64_t grid_total = num_experts * M;
    if (varlen)
        grid_total = (expected_m > 0 && expected_m <= M) ? std::min(M, num_experts * expected_m)
                                                         : M;
    else if (masked_m != nullptr && expected_m > 0 && expected_m < M)
        grid_total = num_experts * expected_m;
    if (grid_total < 1) grid_total = 1;
    a.expected_strips = static_cast<uint64_t>(grid_total) * a.p.segs;
    a.expected_rows = static_cast<uint64_t>(grid_total);
    a.group = group;
    a.kind = nvfp4                            ? pqg::Kind::E2M1_E4M3
             : out_dtype == PQG_E2M1          ? pqg::Kind::E2M1_UE8M0
             : scale_fmt == PQG_SCALE_UE8M0 ? pqg::Kind::E4M3_UE8M0
             : out_dtype == PQG_INT8        ? pqg::Kind::INT8_FP32
                                            : pqg::Kind::E4M3_FP32;
    a.disp = varlen ? pqg::kVarlen : num_experts > 1 ? pqg::kMasked : pqg::kFlat;
    // Small fused masked calls (decode: a few rows per expert, at most 32
    // experts) load each expert's first expected_m rows without waiting for
    // masked_m (pqg_kernel.cuh, kMaskedSpec); rows past masked_m are read there
    // but never written.
    a.p.spec = 0;
    a.p.spec_magic = 0;
    a.p.spec_shift = 0;
    if (a.disp == pqg::kMasked && masked_m != nullptr && fuse_silu_mul != 0 && num_experts <= 32 &&
        expected_m >= 1 && expected_m <= kMaxSpecRows) {
        a.disp = pqg::kMaskedSpec;
        a.p.spec = static_cast<uint32_t>(std::min(expected_m, M));
        pqg::segs_divider(a.p.spec * a.p.segs, &a.p.spec_magic, &a.p.spec_shift);
    }
    a.fused = fuse_silu_mul != 0;
    a.pdl = g_pdl.load(std::memory_order_relaxed) != 0;
    a.stream = reinterpret_cast<cudaStream_t>(stream);

    const cudaError_t err = in_dtype == PQG_BF16 ? pqg::launch_bf16(a) : pqg::launch_fp16(a);
    if (err != cudaSuccess) {
        g_last_cuda_error = static_cast<int>(err);
        (void)cudaGetLastError();  // the error is reported here; do not leave it sticky
        return PQG_ERR_CUDA;
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PQG_OK;
}

}  // namespace

extern "C" {

int64_t pqg_scales_bytes(int64_t num_experts, int64_t M, int64_t K, int group, int scale_fmt,
                         int scale_layout) {
    int64_t plane = 0;
    const int st = check_geometry(num_experts, M, K, group, scale_fmt, scale_layout, &plane);
    if (st != PQG_OK) return st;
    return plane * num_experts;
}

int pqg_quant(const void *in, void *out, void *scales, int64_t M, int64_t num_experts, int64_t K,
              int group, int in_dtype, int out_dtype, int scale_fmt, int scale_layout,
              int fuse_silu_mul, const int32_t *masked_m, int64_t expected_m,
              pqg_stream_t stream) {
    if (scale_fmt == PQG_SCALE_E4M3) return PQG_ERR_UNSUPPORTED;  // pqg_quant_nvfp4
    return quant_impl(in, out, scales, nullptr, M, num_experts, K, group, in_dtype, out_dtype,
                      scale_fmt, scale_layout, fuse_silu_mul, masked_m, expected_m, stream);
}

int pqg_quant_nvfp4(const void *in, void *out, void *scales, const float *global_scale,
                    int64_t M, int64_t num_experts, int64_t K, int in_dtype, int scale_layout,
                    int fuse_silu_mul, const int32_t *masked_m, int64_t expected_m,
                    pqg_stream_t stream) {
    return quant_impl(in, out, scales, global_scale, M, num_experts, K, 16, in_dtype, PQG_E2M1,
                      PQG_SCALE_E4M3, scale_layout, fuse_silu_mul, masked_m, expected_m,
                      stream);
}

int pqg_quant_varlen(const void *in, void *out, void *scales, const float *global_scale,
                     int64_t M, int64_t num_experts, int64_t K, int group, int in_dtype,
                     int out_dtype, int scale_fmt, int scale_layout, int fuse_silu_mul,
                     const int32_t *seg_indptr, const int32_t *seg_lens, int64_t expected_m,
                     pqg_stream_t stream) {
    if (seg_indptr == nullptr) return PQG_ERR_INVALID_ARG;
    if ((scale_fmt == PQG_SCALE_E4M3) != (global_scale != nullptr)) return PQG_ERR_INVALID_ARG;
    return quant_impl(in, out, scales, global_scale, M, num_experts, K, group, in_dtype,
                      out_dtype, scale_fmt, scale_layout, fuse_silu_mul, nullptr, expected_m,
                      stream, Segments{seg_indptr, seg_lens});
}

const char *pqg_status_string(int status) {
    switch (status) {
        case PQG_OK: return "ok";
        case PQG_ERR_INVALID_ARG: return "invalid argument";
        case PQG_ERR_UNSUPPORTED: return "unsupported combination of arguments";
        case PQG_ERR_ALIGNMENT: return "pointer misaligned";
        case PQG_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

int pqg_last_cuda_error(void) { return g_last_cuda_error; }

int pqg_set_pdl(int enable) { return g_pdl.exchange(enable != 0 ? 1 : 0); }

uint64_t pqg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *pqg_version(void) { return "pqg 0.1.0 sm_100a"; }

}  // extern "C"
