// Merge of the decode results of R ranks that each attended to a disjoint
// part of every request's KV pages (split-KV across GPUs).  With rank i's
// normalised output O_i and log-sum-exp lse_i of one query row:
//
//   L* = log sum_i exp(lse_i),   O = sum_i exp(lse_i - L*) O_i,   LSE = L*
//
// the same LSE-weighted merge the in-GPU combine applies to split partials;
// a rank whose part of the request is empty (or fully masked) has
// lse_i = -inf and weight 0; a row with every lse_i = -inf gives O = 0,
// LSE = -inf.  One warp per query row; each lane owns 8 consecutive output
// columns per 256-column stripe, read as one 16-byte load per rank (bf16
// partials) or two (fp32 partials: the ranks' results before any bf16
// rounding, so that the merged row is rounded once, as inside one GPU).
#pragma once

#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>

namespace mla {

constexpr int kRankCombineWarps = 8;  // query rows per CTA
constexpr int kRankCombineMaxRanks = 64;

struct RankCombineParams {
    const void* o_parts;           // [R][B][s_q][h][d_v], bf16 or fp32
    const float* lse_parts;        // [R][B][h][s_q]
    __nv_bfloat16* out;            // [B][s_q][h][d_v]
    float* lse;                    // [B][h][s_q]
    int R, B, s_q, h;
};

// 8 consecutive partial values as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(h2[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}
__device__ __forceinline__ void load8(const float* src, float (&f)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 b = *reinterpret_cast<const float4*>(src + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <int kDv, typename TIn>
__global__ void __launch_bounds__(32 * kRankCombineWarps) mla_rank_combine_kernel(const RankCombineParams p) {
    constexpr int kChunks = kDv / 8;                    // 16-byte chunks of one row
    constexpr int kPerLane = (kChunks + 31) / 32;       // chunks per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long rows = (long)p.B * p.s_q * p.h;
    const long row = (long)blockIdx.x * kRankCombineWarps + warp;  // (b * s_q + s) * h + head
    if (row >= rows) return;
    const int head = static_cast<int>(row % p.h);
    const long bs = row / p.h;
    const int s = static_cast<int>(bs % p.s_q);
    const long b = bs / p.s_q;
    const long lrow = (b * p.h + head) * p.s_q + s;  // LSE index
    // lse of every rank: lane i holds ranks i, i + 32, ...
    float mx = -INFINITY;
    for (int r = lane; r < p.R; r += 32) mx = fmaxf(mx, p.lse_parts[(long)r * rows + lrow]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float acc[kPerLane][8];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    float lstar = -INFINITY;
    if (mx != -INFINITY) {  // uniform across the warp
        float sum = 0.f;
        for (int r = lane; r < p.R; r += 32) sum += expf(p.lse_parts[(long)r * rows + lrow] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        lstar = mx + logf(sum);
        for (int r = 0; r < p.R; ++r) {
            const float w = expf(p.lse_parts[(long)r * rows + lrow] - lstar);
            if (w == 0.f) continue;  // uniform: every lane reads the same lse
            const TIn* src = static_cast<const TIn*>(p.o_parts) + ((long)r * rows + row) * kDv;
#pragma unroll
            for (int j = 0; j < kPerLane; ++j) {
                const int c = lane + 32 * j;
                if (c < kChunks) {
                    float f[8];
                    load8(src + 8 * c, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[j][e] = fmaf(w, f[e], acc[j][e]);
                }
            }
        }
    }
    __nv_bfloat16* dst = p.out + row * kDv;
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
        const int c = lane + 32 * j;
        if (c < kChunks) {
            uint4 v;
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(acc[j][2 * e], acc[j][2 * e + 1]);
            *reinterpret_cast<uint4*>(dst + 8 * c) = v;
        }
    }
    if (lane == 0) p.lse[lrow] = lstar;
}

}  // namespace mla
