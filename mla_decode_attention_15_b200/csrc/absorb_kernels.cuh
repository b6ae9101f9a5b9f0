// Absorbed projections on either side of the decode (GQLA technical summary,
// "Caminho MQA-Absorvido": the up-projections are absorbed into the query and
// output projections, so every head attends to the latent cache directly):
//
//   q_out[t][h] = [ q_in[t][h][0:128] . W_UK[h] (512) | q_in[t][h][128:192] ]
//   out[t][h]   =   o[t][h][0:512] . W_UV[h]   (128)
//
// as tcgen05 GEMMs in the decode's transposed orientation: the weight's output
// dimension fills the MMA's M, the few tokens fill N.  Every CTA takes one
// 128 x 128 tile of one head's weight (output columns x K rows, MN-major A)
// and 64 tokens (K-major B), so both projections spread over 4 h CTAs:
//   absorb_q: the 4 tiles of W_UK[h] are 4 output-column chunks (K = 128);
//   absorb_o: the 4 tiles of W_UV[h] are 4 K chunks (K = 512), run as one
//             cluster of 4 CTAs whose fp32 partial products are summed
//             through distributed shared memory, each CTA finishing 16 tokens.
// One thread prefetches the weight tile into L2 before the dependency wait
// (programmatic dependent launch: the fetch overlaps the previous kernel),
// then loads both operands by TMA and issues the MMAs; four warps read the
// accumulator back from TMEM.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kProjTokens = 64;      // tokens per CTA (MMA N)
constexpr int kProjThreads = 128;    // 4 warps: TMEM lanes 0..127
constexpr int kProjTile = 128;       // output columns (MMA M) and K rows per CTA
constexpr int kProjSplitK = 4;       // absorb_o: K = 512 over a cluster of 4
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
    static constexpr int kGridX = 4;  // absorb_q: output chunks; absorb_o: K chunks (the cluster)
    static constexpr int kABlockBytes = kProjTile * 128;     // 64 output columns x 128 K rows
    static constexpr int kABytes = 2 * kABlockBytes;         // 32 KB
    static constexpr int kBBoxBytes = kProjTokens * 128;     // 64 tokens x 64 K columns
    static constexpr int kBBytes = 2 * kBBoxBytes;           // 16 KB
    static constexpr int kRedBytes = kProjTokens * kProjTile * 4;  // fp32 partials (absorb_o)
    static constexpr int kTmemCols = kProjTokens;
    static constexpr int kSmem = kABytes + kBBytes + 64 + 1024;  // + barriers, TMEM slot, alignment
    static_assert(kKind == 0 ? kProjLatent == kGridX * kProjTile : kProjLatent == kProjSplitK * kProjTile);
    static_assert(kRedBytes <= kABytes, "partials reuse the weight tile's shared memory");
};

template <int kKind>
__global__ void __launch_bounds__(kProjThreads)
    mla_absorb_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                      const ProjParams p) {
    using P = ProjShape<kKind>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int ocol = kKind == 0 ? kProjTile * blockIdx.x : 0;  // first output column of the tile
    const int krow = kKind == 0 ? 0 : kProjTile * blockIdx.x;  // first K row of the tile
    const int h = blockIdx.y;
    const int t0 = blockIdx.z * kProjTokens;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t a_s = smem_addr(smem);
    const uint32_t b_s = a_s + P::kABytes;
    const uint32_t bar_full = b_s + P::kBBytes;
    const uint32_t bar_done = bar_full + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kABytes + P::kBBytes + 16);

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_done, 1);
        fence_mbar_init();
        prefetch_tensormap(&w_map);
        prefetch_tensormap(&x_map);
        // The weight does not come from the previous kernel: start its fetch now.
        tma_prefetch_3d(&w_map, ocol, krow, h);
        tma_prefetch_3d(&w_map, ocol + 64, krow, h);
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
        mbar_arrive_expect_tx(bar_full, P::kABytes + P::kBBytes);
        // Weight: two 64-column blocks of 128 K rows (rows of 128 B, 8-row
        // groups 1 KB apart, swizzled).
        tma_load_3d_hint(a_s, &w_map, bar_full, ocol, krow, h, pol);
        tma_load_3d_hint(a_s + P::kABlockBytes, &w_map, bar_full, ocol + 64, krow, h, pol);
        // Input rows of the tile, K columns krow .. krow + 127; rows past T read as zero.
        tma_load_3d_hint(b_s, &x_map, bar_full, krow, h, t0, pol);
        tma_load_3d_hint(b_s + P::kBBoxBytes, &x_map, bar_full, krow + 64, h, t0, pol);
        ok = proj_wait(bar_full, 0, p.status);
        if (ok) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(kProjTile, kProjTokens, 1, 0);
            // A MN-major: the two 64-column atoms LBO apart, 8-row K groups 1 KB apart.
            const uint64_t a0 = smem_desc(a_s, P::kABlockBytes, 1024, kSwizzle128);
            // B K-major: 8-token groups 1 KB apart, 64 K per 128-byte swizzled row.
            const uint64_t b0 = smem_desc(b_s, 16, 1024, kSwizzle128);
#pragma unroll
            for (int ks = 0; ks < kProjTile / 16; ++ks) {
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
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    const int m = 32 * warp + lane;  // this thread's TMEM lane = output column within the tile
    if constexpr (kKind == 0) {
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kProjTokens; c0 += 16) {
                float v[16];
                tmem_ld_x16(tmem + lane_base + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int t = t0 + c0 + c;
                    if (t < p.T)
                        p.out[((size_t)t * p.heads + h) * P::kOutW + ocol + m] = __float2bfloat16_rn(v[c]);
                }
            }
        }
    } else {
        // Partial product over this CTA's 128 K rows -> shared memory as
        // [token][column] fp32, in place of the weight tile (the MMAs that
        // read it have completed).
        float* red = reinterpret_cast<float*>(smem);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kProjTokens; c0 += 16) {
                float v[16];
                tmem_ld_x16(tmem + lane_base + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) red[(c0 + c) * kProjTile + m] = v[c];
            }
        }
        cluster_sync_all();
        // CTA r of the cluster sums the 4 partials of tokens 16 r .. 16 r + 15;
        // all 64 remote loads are issued before the first sum.
        constexpr int kPer = kProjTokens / kProjSplitK;
        const int r = static_cast<int>(cluster_ctarank());
        const uint32_t local = smem_addr(red + r * kPer * kProjTile + m);
        float part[kProjSplitK][kPer];
#pragma unroll
        for (int q = 0; q < kProjSplitK; ++q) {
            const uint32_t remote = cluster_map(local, q);
#pragma unroll
            for (int i = 0; i < kPer; ++i) part[q][i] = ld_cluster_f32(remote + i * kProjTile * 4);
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const float acc = (part[0][i] + part[1][i]) + (part[2][i] + part[3][i]);
            const int t = t0 + r * kPer + i;
            if (t < p.T) p.out[((size_t)t * p.heads + h) * P::kOutW + m] = __float2bfloat16_rn(acc);
        }
        cluster_sync_all();  // no CTA leaves while another still reads its partials
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, P::kTmemCols);
    }
}

}  // namespace mla
