// Fused SiLU-and-mul quantization with the input staged in shared memory.
//
// The fused prologue (sglang PR #30924 report, 实现拆解 item 1: silu_and_mul
// fused into the quantization) costs about twice the instructions per byte of
// a plain call: two MUFU operations per element (exp2 and reciprocal) and the
// extra multiplies.  A warp that holds its strip's gate and up halves in
// registers has no load in flight while it computes, so the kernel needs many
// warps, and the registers of a second strip in flight cost warps again.
//
// Here the warp copies the gate and up halves of a later strip into shared
// memory with asynchronous 16-byte copies (cp.async, one commit group per
// strip) before it computes the current strip from shared memory.  The copies
// of STAGES - 1 strips stay in flight while the warp computes, without holding
// registers.  Lane i copies the 16-byte chunks i and 32 + i of each 1 KB half,
// so every copy instruction of the warp reads 512 contiguous bytes (whole
// 32-byte sectors, each fetched once); after cp.async.wait_group (a hardware
// wait on the lane's own copies) a warp barrier makes every lane's chunks
// visible, and lane j reads its chunks 2j and 2j + 1.  Chunk c sits at
// position c ^ ((c >> 3) & 1) of its half, so that the eight lanes of each
// quarter-warp phase, reading chunks 2j (or 2j + 1), and the copies of eight
// consecutive chunks, each touch eight different 16-byte bank groups.
//
// Strips follow the strip kernel's block-cyclic order (blocks of WARPS
// strips; CTA c takes blocks c, c + grid, ...; warp w takes strip w of each
// block), in one resident wave so that every warp has a run of strips to
// pipeline.  The arithmetic and the stores are those of the strip kernel
// (quantize_strip), so results are bit-identical to it.
#pragma once

#include "pqg_kernel.cuh"

namespace pqg {

constexpr uint32_t kPipeStageBytes = 2u * kStripBytes;   // gate and up of one strip

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void lds128(uint32_t addr, uint32_t *r) {
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__host__ __device__ constexpr uint32_t pipe_smem_bytes(int warps, int stages) {
    return static_cast<uint32_t>(warps * stages) * kPipeStageBytes;
}

// Flat fused dispatch (one expert, M rows of [gate | up]).
template <typename In, int G, Kind KIND, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32)
    fused_pipe_kernel(const __grid_constant__ Params p) {
    static_assert(STAGES >= 2, "at least one strip in flight while computing");
    extern __shared__ __align__(128) uint8_t stage_smem[];
    __shared__ float nv[KIND == Kind::E2M1_E4M3 ? kNvTable : 1];

    wait_for_producer();                        // before the first global access
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    if constexpr (KIND == Kind::E2M1_E4M3) build_nvfp4_table(p, nv);

    const uint32_t total = p.M * p.segs;
    const uint32_t stage0 = static_cast<uint32_t>(__cvta_generic_to_shared(stage_smem)) +
                            warp * STAGES * kPipeStageBytes;   // this warp's stages
    const uint64_t half = static_cast<uint64_t>(p.K) * 2u;   // up starts K elements in

    // the k-th strip of this warp
    auto strip_of = [&](uint32_t k) { return (blockIdx.x + k * gridDim.x) * WARPS + warp; };
    // swizzled byte offset of 16-byte chunk c (0..63) within a 1 KB half
    auto pos = [](uint32_t c) { return (c ^ ((c >> 3) & 1u)) * 16u; };
    // copy chunks lane and 32 + lane of strip k's gate and up halves into its
    // stage; one commit group per strip, empty past the end.  Chunks past a
    // ragged row's end are not copied (their lanes store nothing).
    auto issue = [&](uint32_t k) {
        const uint32_t s = strip_of(k);
        if (s < total) {
            const uint32_t row = s / p.segs;
            const uint32_t col0 = (s - row * p.segs) * kStripElems;   // first element
            const uint8_t *src = p.in + static_cast<uint64_t>(row) * p.in_row_bytes +
                                 static_cast<uint64_t>(col0) * 2u;
            const uint32_t dst = stage0 + (k % STAGES) * kPipeStageBytes;
#pragma unroll
            for (uint32_t c = lane; c < 64u; c += 32u) {
                if (col0 + c * 8u < p.K) {          // 8 elements per chunk
                    cp_async16(dst + pos(c), src + c * 16u);
                    cp_async16(dst + kStripBytes + pos(c), src + half + c * 16u);
                }
            }
        }
        cp_async_commit();
    };

#pragma unroll
    for (uint32_t k = 0; k + 1 < STAGES; ++k) issue(k);
    for (uint32_t k = 0; strip_of(k) < total; ++k) {
        __syncwarp();                           // every lane is done with iteration k - 1's stage
        issue(k + STAGES - 1);                  // ... which strip k + STAGES - 1 now refills
        cp_async_wait<STAGES - 1>();            // this lane's copies of strip k have landed
        __syncwarp();                           // and so have every other lane's
        const uint32_t s = strip_of(k);
        const uint32_t row = s / p.segs;
        const uint32_t col = (s - row * p.segs) * kStripElems + lane * 16u;
        const uint32_t a = stage0 + (k % STAGES) * kPipeStageBytes;
        uint32_t x[8], u[8];
        lds128(a + pos(2u * lane), x);
        lds128(a + pos(2u * lane + 1u), x + 4);
        lds128(a + kStripBytes + pos(2u * lane), u);
        lds128(a + kStripBytes + pos(2u * lane + 1u), u + 4);
        quantize_strip<In, G, KIND, true>(x, u, 0u, row, col, p, lane, nv);
    }
    cp_async_wait<0>();                         // nothing left in flight at exit
    release_dependents();
}

}  // namespace pqg
