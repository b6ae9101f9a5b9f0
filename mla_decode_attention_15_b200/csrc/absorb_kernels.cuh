// Absorbed projections on either side of the decode (GQLA technical summary,
// "Caminho MQA-Absorvido": the up-projections are absorbed into the query and
// output projections, so every head attends to the latent cache directly):
//
//   q_out[t][h] = [ q_in[t][h][0:128] . W_UK[h] (512) | q_in[t][h][128:192] ]
//   out[t][h]   =   o[t][h][0:512] . W_UV[h]   (128)
//
// as tcgen05 GEMMs in the decode's transposed orientation: the weight's output
// dimension fills the MMA's M, the few tokens fill N.  One CTA per (128 output
// columns, head, 64-token tile): one thread loads that slice of the head's
// weight (MN-major A: 32 KB for the query side, 128 KB for the output side) and
// the tile's input rows (K-major B) by TMA and issues the MMAs; four warps read
// the accumulator back from TMEM and write bf16 rows.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kProjTokens = 64;      // tokens per CTA (MMA N)
constexpr int kProjThreads = 128;    // 4 warps: TMEM lanes 0..127
constexpr int kProjNope = 128, kProjLatent = 512, kProjRope = 64, kProjVHead = 128;
constexpr uint64_t kProjWaitNs = 1000000000ull;  // 1 s per wait

struct ProjParams {
    __nv_bfloat16* out;            // absorb_q: [T][h][576]; absorb_o: [T][h][128]
    const __nv_bfloat16* rope_in;  // absorb_q: q_in [T][h][192] (its RoPE part is copied)
    int32_t* status;               // optional device status word (MLA_STATUS_TIMEOUT)
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

// kKind 0: absorb_q (A = W_UK[h]^T: M 512 in 4 CTAs of 128, K 128; B = q_nope^T)
// kKind 1: absorb_o (A = W_UV[h]^T: M 128, K 512; B = o^T)
template <int kKind>
struct ProjShape {
    static constexpr int kM = kKind == 0 ? kProjLatent : kProjVHead;  // output width
    static constexpr int kK = kKind == 0 ? kProjNope : kProjLatent;   // contraction
    static constexpr int kChunks = kM / 128;                           // CTAs along M
    static constexpr int kInW = kKind == 0 ? kProjNope + kProjRope : kProjLatent;  // input row
    static constexpr int kOutW = kKind == 0 ? kProjLatent + kProjRope : kProjVHead;
    static constexpr int kABlockBytes = kK * 128;                      // 64 M columns x kK rows
    static constexpr int kABytes = 2 * kABlockBytes;                   // one M chunk of 128
    static constexpr int kBBoxes = kK / 64;                            // B: 64-column boxes
    static constexpr int kBBoxBytes = kProjTokens * 128;               // 64 token rows of 128 B
    static constexpr int kBBytes = kBBoxes * kBBoxBytes;
    static constexpr int kWBoxRows = kK <= 256 ? kK : 256;             // TMA box rows of the weight
    static constexpr int kWBoxesPerBlock = kK / kWBoxRows;
    static constexpr int kTmemCols = kProjTokens;
    static constexpr int kSmem = kABytes + kBBytes + 64 + 1024;        // + barriers, tmem slot, align
};

template <int kKind>
__global__ void __launch_bounds__(kProjThreads)
    mla_absorb_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                      const ProjParams p) {
    using P = ProjShape<kKind>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int ch = blockIdx.x;  // output columns 128 ch .. 128 ch + 127
    const int h = blockIdx.y;
    const int t0 = blockIdx.z * kProjTokens;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t a_s = smem_addr(smem);
    const uint32_t b_s = a_s + P::kABytes;
    const uint32_t bar_full = b_s + P::kBBytes;
    const uint32_t bar_done = bar_full + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kABytes + P::kBBytes + 16);

    if (threadIdx.x == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), P::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&w_map);
        prefetch_tensormap(&x_map);
        const uint64_t pol = l2_policy_evict_normal();
        mbar_arrive_expect_tx(bar_full, P::kABytes + P::kBBytes);
        // Weight of head h: the two 64-column blocks of this chunk, all K rows
        // (rows of 128 B, 8-row groups 1 KB apart, swizzled).
        for (int mb = 0; mb < 2; ++mb)
            for (int r = 0; r < P::kWBoxesPerBlock; ++r)
                tma_load_3d_hint(a_s + mb * P::kABlockBytes + r * P::kWBoxRows * 128, &w_map, bar_full,
                                 128 * ch + 64 * mb, r * P::kWBoxRows, h, pol);
        // Input rows of the tile; rows past T read as zero.
        for (int c = 0; c < P::kBBoxes; ++c)
            tma_load_3d_hint(b_s + c * P::kBBoxBytes, &x_map, bar_full, 64 * c, h, t0, pol);
        ok = proj_wait(bar_full, 0, p.status);
        if (ok) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, kProjTokens, 1, 0);
            // A MN-major: the two 64-column atoms LBO apart, 8-row K groups 1 KB apart.
            const uint64_t a0 = smem_desc(a_s, P::kABlockBytes, 1024, kSwizzle128);
            // B K-major: 8-token groups 1 KB apart, 64 K per 128-byte swizzled row.
            const uint64_t b0 = smem_desc(b_s, 16, 1024, kSwizzle128);
#pragma unroll 1
            for (int ks = 0; ks < P::kK / 16; ++ks) {
                const uint64_t a = a0 + ((ks * 2048) >> 4);  // 16 K rows of 128 B
                const uint64_t b = b0 + (((ks >> 2) * P::kBBoxBytes + (ks & 3) * 32) >> 4);
                umma_f16(tmem, a, b, idesc, ks > 0 ? 1u : 0u);
            }
            umma_commit(bar_done);
        }
    }
    // The RoPE part of the query passes through unchanged (absorb_q, first
    // chunk): 64 tokens x 64 columns of this head, 16 bytes per access.
    if constexpr (kKind == 0) {
        if (ch == 0) {
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
        // Thread = TMEM lane = output column m; 64 token columns.
        const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
        const int m = 128 * ch + 32 * warp + lane;
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
