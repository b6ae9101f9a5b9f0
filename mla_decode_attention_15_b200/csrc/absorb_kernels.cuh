// Absorbed projections on either side of the decode (GQLA technical summary,
// "Caminho MQA-Absorvido": the up-projections are absorbed into the query and
// output projections, so every head attends to the latent cache directly):
//
//   q_out[t][h] = [ q_in[t][h][0:128] . W_UK[h] (512) | q_in[t][h][128:192] ]
//   out[t][h]   =   o[t][h][0:512] . W_UV[h]   (128)
//
// as tcgen05 GEMMs in the decode's transposed orientation: the weight's output
// dimension fills the MMA's M, the few tokens fill N.  The unit of work is a
// 128 x 128 tile of one head's weight (output columns x K rows, MN-major A)
// against 64 tokens (K-major B):
//   absorb_q: one CTA per tile -- the 4 tiles of W_UK[h] are its 4
//             output-column chunks (K = 128), 4 h CTAs of 49 KB;
//   absorb_o: one CTA per head -- the 4 tiles of W_UV[h] are K chunks
//             (K = 512) streamed through a 2-stage ring into one TMEM
//             accumulator, 96 KB per CTA so that two fit an SM.
// One thread prefetches the head's weight into L2 before the dependency wait
// (programmatic dependent launch: the fetch overlaps the previous kernel),
// then loads both operands by TMA and issues the MMAs; four warps read the
// accumulator back from TMEM.  (Splitting absorb_o's K over a 4-CTA cluster
// with a distributed-shared-memory reduction was measured slower.)
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kProjTokens = 64;      // tokens per CTA (MMA N)
constexpr int kProjThreads = 128;    // 4 warps: TMEM lanes 0..127
constexpr int kProjTile = 128;       // output columns (MMA M) and K rows per CTA
constexpr int kProjOStages = 2;      // absorb_o: K-chunk ring depth
constexpr int kProjNope = 128, kProjLatent = 512, kProjRope = 64, kProjVHead = 128;
constexpr uint64_t kProjWaitNs = 1000000000ull;  // 1 s per wait

struct ProjParams {
    __nv_bfloat16* out;            // absorb_q: [T][h][576]; absorb_o: [T][h][128]
    const __nv_bfloat16* rope_in;  // absorb_q: q_in [T][h][192] (its RoPE part is copied)
    int32_t* status;               // optional device status word
    int T, heads;
};

__device__ __forceinline__ bool proj_wait(uint32_t bar, uint32_t parity, int32_t* status) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kProjWaitNs) {
            if (status) atomicOr(status, MLA_STATUS_TIMEOUT);
            return false;
        }
    }
    return true;
}

// kKind 0: absorb_q; kKind 1: absorb_o.
template <int kKind>
struct ProjShape {
    static constexpr int kInW = kKind == 0 ? kProjNope + kProjRope : kProjLatent;    // input row
    static constexpr int kOutW = kKind == 0 ? kProjLatent + kProjRope : kProjVHead;  // output row
    static constexpr int kGridX = kKind == 0 ? kProjLatent / kProjTile : 1;  // CTAs per head
    static constexpr int kKChunks = kKind == 0 ? 1 : kProjLatent / kProjTile;  // K tiles per CTA
    static constexpr int kStages = kKind == 0 ? 1 : kProjOStages;
    static constexpr int kABlockBytes = kProjTile * 128;     // 64 output columns x 128 K rows
    static constexpr int kABytes = 2 * kABlockBytes;         // 32 KB: one weight tile
    static constexpr int kBBoxBytes = kProjTokens * 128;     // 64 tokens x 64 K columns
    static constexpr int kBBytes = 2 * kBBoxBytes;           // 16 KB: the tile's input rows
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = kStages * kStageBytes;    // full[kStages], empty[kStages], done
    static constexpr int kTmemCols = kProjTokens;
    static constexpr int kSmem = kBarOff + 8 * (2 * kStages + 1) + 16 + 1024;  // + TMEM slot, alignment
    static_assert(kProjLatent % kProjTile == 0 && kProjVHead == kProjTile, "128 x 128 weight tiles");
};

template <int kKind>
__global__ void __launch_bounds__(kProjThreads)
    mla_absorb_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                      const ProjParams p) {
    using P = ProjShape<kKind>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int ocol = kProjTile * blockIdx.x;  // first output column of the CTA (absorb_q chunks)
    const int h = blockIdx.y;
    const int t0 = blockIdx.z * kProjTokens;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t s0 = smem_addr(smem);
    const uint32_t bar = s0 + P::kBarOff;  // full[st] at bar + 8 st, empty[st] after them
    const uint32_t bar_done = bar + 8 * (2 * P::kStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kBarOff + 8 * (2 * P::kStages + 1));

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * P::kStages + 1; ++i) mbar_init(bar + 8 * i, 1);
        fence_mbar_init();
        prefetch_tensormap(&w_map);
        prefetch_tensormap(&x_map);
        // The weight does not come from the previous kernel: start its fetch now.
        for (int kc = 0; kc < P::kKChunks; ++kc) {
            tma_prefetch_3d(&w_map, ocol, kProjTile * kc, h);
            tma_prefetch_3d(&w_map, ocol + 64, kProjTile * kc, h);
        }
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), P::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();  // the input rows may come from the previous kernel

    bool ok = true;
    if (threadIdx.x == 0) {
        const uint64_t pol = l2_policy_evict_normal();
        // K chunk kc -> stage kc % kStages: weight rows kc*128.., two 64-column
        // blocks (rows of 128 B, 8-row groups 1 KB apart, swizzled), and the
        // input rows' K columns kc*128..; rows past T read as zero.
        auto load = [&](int kc) {
            const int st = kc % P::kStages;
            const uint32_t a_s = s0 + st * P::kStageBytes, b_s = a_s + P::kABytes;
            const uint32_t full = bar + 8 * st;
            mbar_arrive_expect_tx(full, P::kStageBytes);
            tma_load_3d_hint(a_s, &w_map, full, ocol, kProjTile * kc, h, pol);
            tma_load_3d_hint(a_s + P::kABlockBytes, &w_map, full, ocol + 64, kProjTile * kc, h, pol);
            tma_load_3d_hint(b_s, &x_map, full, kProjTile * kc, h, t0, pol);
            tma_load_3d_hint(b_s + P::kBBoxBytes, &x_map, full, kProjTile * kc + 64, h, t0, pol);
        };
        constexpr uint32_t idesc = idesc_bf16_f32(kProjTile, kProjTokens, 1, 0);
        for (int kc = 0; kc < P::kStages && kc < P::kKChunks; ++kc) load(kc);
        // MMAs of chunk kc, then the refill of its stage with chunk kc +
        // kStages once those MMAs have read it.
#pragma unroll 1
        for (int kc = 0; kc < P::kKChunks && ok; ++kc) {
            const int st = kc % P::kStages;
            ok = proj_wait(bar + 8 * st, (kc / P::kStages) & 1, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a_s = s0 + st * P::kStageBytes, b_s = a_s + P::kABytes;
            // A MN-major: the two 64-column atoms LBO apart, 8-row K groups 1 KB apart.
            const uint64_t a0 = smem_desc(a_s, P::kABlockBytes, 1024, kSwizzle128);
            // B K-major: 8-token groups 1 KB apart, 64 K per 128-byte swizzled row.
            const uint64_t b0 = smem_desc(b_s, 16, 1024, kSwizzle128);
#pragma unroll
            for (int ks = 0; ks < kProjTile / 16; ++ks) {
                const uint64_t a = a0 + ((ks * 2048) >> 4);  // 16 K rows of 128 B
                const uint64_t b = b0 + (((ks >> 2) * P::kBBoxBytes + (ks & 3) * 32) >> 4);
                umma_f16(tmem, a, b, idesc, (kc > 0 || ks > 0) ? 1u : 0u);
            }
            if (kc + P::kStages < P::kKChunks) {
                const uint32_t empty = bar + 8 * (P::kStages + st);
                umma_commit(empty);
                ok = proj_wait(empty, (kc / P::kStages) & 1, p.status);
                if (ok) load(kc + P::kStages);
            }
        }
        if (ok) umma_commit(bar_done);
    }
    // The RoPE part of the query passes through unchanged (absorb_q, first
    // chunk): 64 tokens x 64 columns of this head, 16 bytes per access.
    if constexpr (kKind == 0) {
        if (blockIdx.x == 0) {
            for (int i = threadIdx.x; i < kProjTokens * (kProjRope / 8); i += kProjThreads) {
                const int tt = i / (kProjRope / 8), c8 = i - tt * (kProjRope / 8);
                const int t = t0 + tt;
                if (t < p.T) {
                    const uint4 v = *reinterpret_cast<const uint4*>(
                        p.rope_in + ((size_t)t * p.heads + h) * P::kInW + kProjNope + 8 * c8);
                    *reinterpret_cast<uint4*>(p.out + ((size_t)t * p.heads + h) * P::kOutW + kProjLatent +
                                              8 * c8) = v;
                }
            }
        }
    }
    ok = __syncthreads_and(ok);
    if (ok) ok = __all_sync(0xffffffffu, proj_wait(bar_done, 0, p.status));
    if (ok) {
        tc_fence_after();
        // Thread = TMEM lane = output column; 64 token columns.
        const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
        const int m = ocol + 32 * warp + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < kProjTokens; c0 += 16) {
            float v[16];
            tmem_ld_x16(tmem + lane_base + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int t = t0 + c0 + c;
                if (t < p.T) p.out[((size_t)t * p.heads + h) * P::kOutW + m] = __float2bfloat16_rn(v[c]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, P::kTmemCols);
    }
}

}  // namespace mla
