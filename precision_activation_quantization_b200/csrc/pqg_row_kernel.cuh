// Per-token quantization (one group per row, G = K) for sm_100a.
//
// The TeleFuser "tf-kernel 安装与使用" page (使用示例) shows the per-token form
// of the operation, tf_per_token_quant_fp8(x, x_q, x_scale): one fp32 scale per
// row ([M, 1]) and E4M3 codes into caller-allocated outputs.  The arithmetic is
// the per-group rule with the group widened to the whole row.
//
// A row is shared by WPR warps (1, 2, 4 or 8, chosen at launch so that a
// thread holds at most SLOTS 16-element slots).  Lanes read consecutive
// 32-byte slots, so a warp's loads cover 1 KB contiguous.  The row absmax is a
// warp xor-reduction, then (WPR > 1) one exchange through shared memory behind
// a named barrier of the row's own warps.  The partials are double-buffered by
// iteration parity, so one barrier per row iteration is enough.  Values stay in
// registers between the reduction and the quantization, so every input byte is
// read once.  Rows come from the same expert table as the strip kernel
// (counting rows instead of strips), so flat, batched, masked and varlen
// dispatch and the fused SiLU-and-mul all work unchanged.
#pragma once

#include "pqg_kernel.cuh"

namespace pqg {

constexpr int kRowThreads = 256;  // 8 warps per CTA

// Rows ahead of the current one that each row's warps prefetch into L2 (0:
// none).  One row ahead, by the row's first warp, took [8192, 7168] from 30.59
// to 29.60 us; with each warp prefetching its own share, 29.13 us.
#ifndef PQG_PREFETCH_ROW
#define PQG_PREFETCH_ROW 1
#endif


// The scale of row `row` of expert e.  One group per row: row-major,
// column-major and packed all put it at element / word `row` of the expert's
// plane; the tiled layout has one tile column.
template <Kind KIND>
__device__ __forceinline__ void store_row_scale(const Params &p, uint32_t e, uint32_t row,
                                                const GroupScale &gs) {
    uint8_t *sc = p.scales + e * p.scale_expert_bytes;
    if (p.layout == kPacked)
        reinterpret_cast<uint32_t *>(sc)[row] = gs.e8;  // bytes 1..3 are 0
    else if (p.layout == kTiled128x4)
        store_tiled(sc, row, 0u, 1u, gs.e8);
    else if constexpr (is_ue8m0(KIND))
        sc[row] = static_cast<uint8_t>(gs.e8);
    else
        reinterpret_cast<float *>(sc)[row] = gs.s;
}

template <typename In, Kind KIND, bool FUSED, int SLOTS, bool VARLEN>
__global__ void __launch_bounds__(kRowThreads)
    row_quant_kernel(const __grid_constant__ Params p) {
    static_assert(!is_e2m1(KIND), "per-token E2M1 is not offered");
    extern __shared__ __align__(16) uint32_t smem_prefix[];
    __shared__ float partial[2][kRowThreads / 32];

    wait_for_producer();                        // before the first global access
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    // p.segs is 1 for this kernel: the table counts rows
    const ExpertTable t = make_table<VARLEN>(p, smem_prefix, lane);

    const uint32_t wpr = p.items;               // warps per row: 1, 2, 4 or 8
    const uint32_t rows_per_iter = (kRowThreads / 32) / wpr;
    const uint32_t sub = warp / wpr;            // this warp's row within the iteration
    const uint32_t wr = warp - sub * wpr;       // warp index within the row
    const uint32_t tpr = wpr * 32u;             // threads per row
    const uint32_t tid = wr * 32u + lane;       // thread index within the row
    const uint32_t nslots = p.K / 16u;          // 16-element slots per row

    uint32_t parity = 0;
    for (uint32_t base = blockIdx.x * rows_per_iter; base < t.total;
         base += gridDim.x * rows_per_iter, parity ^= 1u) {
        const uint32_t r = base + sub;          // warp-uniform
        const bool live = r < t.total;
        Span sp = locate<VARLEN>(t, p.experts, live ? r : 0u);
        const uint32_t row = sp.base + ((live ? r : 0u) - sp.start);   // varlen: packed row
        const uint8_t *src = p.in + sp.e * p.in_expert_bytes +
                             static_cast<uint64_t>(row) * p.in_row_bytes;

        // -- loads, then widen (and fuse) into registers -----------------------
        uint32_t x[SLOTS][8];
        uint32_t u[SLOTS][FUSED ? 8 : 1];
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) {
            const uint32_t slot = tid + j * tpr;
            if (live && slot < nslots) {
                load32B(src + slot * 32u, x[j]);
                if constexpr (FUSED) load32B(src + static_cast<uint64_t>(p.K) * 2u + slot * 32u, u[j]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    x[j][i] = 0u;
                    if constexpr (FUSED) u[j][i] = 0u;
                }
            }
        }
#if PQG_PREFETCH_ROW
        // bring a row these warps take later into L2 while this one is
        // reduced and encoded: every warp of the row issues one bulk prefetch of
        // its share of the row (16-byte multiples)
        {
            const uint32_t rn = r + PQG_PREFETCH_ROW * gridDim.x * rows_per_iter;
            if (rn < t.total) {                     // warp-uniform
                const Span sn = locate<VARLEN>(t, p.experts, rn);
                const uint32_t rown = sn.base + (rn - sn.start);
                const uint32_t chunk = ((p.in_row_bytes + wpr - 1u) / wpr + 15u) & ~15u;
                const uint32_t lo = min(wr * chunk, p.in_row_bytes);
                const uint32_t hi = min(lo + chunk, p.in_row_bytes);
                if (lane == 0 && hi > lo)
                    prefetch_l2(p.in + sn.e * p.in_expert_bytes +
                                    static_cast<uint64_t>(rown) * p.in_row_bytes + lo,
                                hi - lo);
            }
        }
#endif
        // Fused rows keep silu(gate) * up in registers; plain rows keep the raw
        // 16-bit values (half the registers) and take the absmax on their
        // magnitude bits, widening only to quantize.
        float v[FUSED ? SLOTS : 1][16];
        float amax = 0.0f;
        if constexpr (FUSED) {
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 y = silu_mul_pair<In>(x[j][i], u[j][i]);
                    v[j][2 * i] = y.x;
                    v[j][2 * i + 1] = y.y;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[j][i]));
            }
        } else {
            uint32_t ab = 0;
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) ab = max(ab, absmax_bits16(x[j]));
            amax = bits16_to_float<In>(ab);
        }

        // -- row absmax: warp, then across the row's warps ---------------------
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (wpr > 1) {
            if (lane == 0) partial[parity][warp] = amax;
            // only this row's warps meet: named barrier 1 + sub (0 belongs to
            // __syncthreads) over wpr warps, so the CTA's rows do not wait on
            // one another (measured 31.25 -> 30.29 us at K = 7168)
            asm volatile("bar.sync %0, %1;" ::"r"(1u + sub), "r"(wpr * 32u) : "memory");
            for (uint32_t w = 0; w < wpr; ++w) amax = fmaxf(amax, partial[parity][sub * wpr + w]);
        }

        // -- scale, codes, stores ----------------------------------------------
        const GroupScale gs = make_scale<KIND>(amax);
        if (live) {
            uint8_t *dst = p.out + sp.e * p.out_expert_bytes + static_cast<uint64_t>(row) * p.K;
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) {
                const uint32_t slot = tid + j * tpr;
                if (slot < nslots) {
                    uint32_t w[4];
                    if constexpr (FUSED) {
                        encode16<KIND>(v[j], gs, w);
                    } else {
                        float vj[16];
#pragma unroll
                        for (int i = 0; i < 8; ++i) widen2<In>(x[j][i], vj[2 * i], vj[2 * i + 1]);
                        encode16<KIND>(vj, gs, w);
                    }
                    store16B(dst + slot * 16u, w[0], w[1], w[2], w[3]);
                }
            }
            if (tid == 0) store_row_scale<KIND>(p, sp.e, row, gs);
        }
    }
    release_dependents();
}

}  // namespace pqg
