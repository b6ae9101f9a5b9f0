// Split-KV work partitioning for the persistent decode kernel.
//
// Work units: request b, head group g ("bg" = b * Hg + g) owns
//   units(bg) = P_b + kItemOverhead   (P_b = ceil(L_b / 2^shift) token blocks of
//                                       2^shift tokens; 0 if P_b == 0)
// The one-CTA kernels walk 64-token pages (shift 6).  The CTA-pair kernel walks
// steps of 128 tokens (shift 7, two pages per step), and builds its plan over
// requests alone (Hg = 1 in the plan): each work range is then walked by the
// request's head groups side by side, one cluster per group, so that the
// groups read each page at about the same time and the repeats hit L2.
// "Page" below means one such block.
// The overhead stands for the per-item cost that does not scale with pages:
// loading Q, filling the pipeline, the epilogue.  Units are laid out in bg
// order and cut into G equal contiguous ranges of T units; CTA k owns
// [k*T, (k+1)*T).  A unit position u inside bg maps to page
// clamp(u - start(bg) - overhead, 0, P_b), so a CTA's range is a list of
// (bg, page range) items; only its first and last item can be partial, and a
// bg covered by more than one CTA is "split": each piece writes an fp32
// partial that the combine kernel merges by LSE weight.
//
// The pages describe no scheduler; this greedy contiguous partition is the
// plainest one that balances ragged lengths across the SMs.
#pragma once

#include <cstdint>

#include "mla_decode.h"

namespace mla {

constexpr int kPage = 64;
constexpr int kPageShift = 6;      // one-CTA kernels: units of one 64-token page
constexpr int kStepShift = 7;      // CTA-pair kernel: units of two pages
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kItemOverhead = 1;   // units charged per (request, head group)
// Smallest range worth its own CTA.  Measured on B200 (graph-replayed steps):
// with 1 instead of 2, bs1 x 1K (16 pages) spreads over 9 CTAs instead of 6 and
// its decode kernel takes 16.4 instead of 18.4 us; no other workload changed.
// (Dropping the per-item overhead unit instead cost the ragged 16-head
// workload 4 us.)
#ifndef MLA_MIN_PAGES_PER_CTA
#define MLA_MIN_PAGES_PER_CTA 1
#endif
constexpr int kMinPagesPerCta = MLA_MIN_PAGES_PER_CTA;

// ---- schedule buffer layout (int32 words) ----
constexpr int kSchedMagic = 0x4D4C4144;  // 'MLAD'
constexpr int kHdrWords = 16;
enum HdrField {
    kHdrMagic = 0,
    kHdrG = 1,
    kHdrBG = 2,
    kHdrHg = 3,
    kHdrNG = 4,
    kHdrSlots = 5,
    kHdrT = 6,
    kHdrStatus = 7,
    kHdrW = 8,
    kHdrBatch = 9,
    kHdrMaxBlocks = 10,
    kHdrShift = 11,    // log2 of the tokens per unit (6 or 7)
    kHdrShareHg = 12,  // head groups that walk every work range side by side (1: none)
};
constexpr int kMetaWords = 8;  // per CTA: begin_bg, begin_page, end_bg, end_page, first_split
enum MetaField { kMetaBeginBg = 0, kMetaBeginPage = 1, kMetaEndBg = 2, kMetaEndPage = 3, kMetaFirstSplit = 4 };
constexpr int kBgWords = 2;  // per bg: slot of split 0 (or the pair plans' slot base), num_splits

__host__ __device__ inline int64_t meta_offset_words() { return kHdrWords; }
__host__ __device__ inline int64_t bg_offset_words(int G) { return kHdrWords + (int64_t)kMetaWords * G; }
__host__ __device__ inline int64_t prefix_offset_words(int G, int BG) {
    return bg_offset_words(G) + (int64_t)kBgWords * BG;
}
__host__ __device__ inline int64_t schedule_words(int G, int BG) {
    return prefix_offset_words(G, BG) + BG + 1;
}

// Head grouping: N = heads * s_q query columns per request.  Up to 64
// columns go in one group of 16, 32 or 64 (the one-CTA kernel's MMA N); wider
// requests are cut into groups of 128 columns for the CTA-pair kernel.
struct Grouping {
    int N;   // heads * s_q
    int NG;  // columns per group: 16, 32, 64, or 128 (CTA pair)
    int Hg;  // groups per request
};
__host__ __device__ inline Grouping make_grouping(int heads, int s_q) {
    Grouping gr;
    gr.N = heads * s_q;
    if (gr.N <= 16) {
        gr.NG = 16;
        gr.Hg = 1;
    } else if (gr.N <= 32) {
        gr.NG = 32;
        gr.Hg = 1;
    } else if (gr.N <= 64) {
        gr.NG = 64;
        gr.Hg = 1;
    } else {
        gr.NG = 128;
        gr.Hg = (gr.N + 127) / 128;
    }
    return gr;
}

// Cached length clamped to what the block table can address.
__host__ __device__ inline int clamp_seqlen(int L, int max_blocks) {
    int64_t cap = (int64_t)max_blocks * kPage;
    if (L < 0) return 0;
    if ((int64_t)L > cap) return (int)cap;
    return L;
}
__host__ __device__ inline bool seqlen_in_range(int L, int max_blocks) {
    return L >= 0 && (int64_t)L <= (int64_t)max_blocks * kPage;
}
__host__ __device__ inline int pages_of(int L) { return (L + kPage - 1) / kPage; }
// blocks of 2^shift tokens covering L tokens
__host__ __device__ inline int blocks_of(int L, int shift) { return (L + (1 << shift) - 1) >> shift; }
__host__ __device__ inline int64_t units_of(int P) { return P > 0 ? (int64_t)P + kItemOverhead : 0; }

__host__ __device__ inline int64_t units_per_cta(int64_t W, int G) {
    int64_t T = (W + G - 1) / (G > 0 ? G : 1);
    int64_t lo = kMinPagesPerCta + kItemOverhead;
    return T < lo ? lo : T;
}

// Largest bg in [0, BG) with prefix[bg] <= u (prefix non-decreasing, prefix[0] == 0).
__host__ __device__ inline int find_bg(const int32_t* prefix, int BG, int64_t u) {
    int lo = 0, hi = BG - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Blocks of request-group bg (of its length clamped to the block table),
// read back from the unit prefix: its units are P + kItemOverhead, or 0 when
// P == 0.  No access to the lengths.
__host__ __device__ inline int pages_in_prefix(const int32_t* prefix, int bg) {
    const int units = prefix[bg + 1] - prefix[bg];
    return units > 0 ? units - kItemOverhead : 0;
}

// (bg, page) position of unit u; u >= W maps to (BG, 0).
__host__ __device__ inline void locate_unit(const int32_t* prefix, int BG, int64_t W, int64_t u, int* bg_out,
                                            int* page_out) {
    if (u >= W) {
        *bg_out = BG;
        *page_out = 0;
        return;
    }
    int bg = find_bg(prefix, BG, u);
    int P = pages_in_prefix(prefix, bg);
    int64_t p = u - (int64_t)prefix[bg] - kItemOverhead;
    if (p < 0) p = 0;
    if (p > P) p = P;
    *bg_out = bg;
    *page_out = (int)p;
}

// First / last CTA that owns a page of bg (P > 0).
__host__ __device__ inline int first_cta_of(const int32_t* prefix, int bg, int64_t T) {
    return (int)(((int64_t)prefix[bg] + kItemOverhead) / T);
}
__host__ __device__ inline int last_cta_of(const int32_t* prefix, int bg, int P, int64_t T) {
    return (int)(((int64_t)prefix[bg] + kItemOverhead + P - 1) / T);
}

__host__ __device__ inline int num_splits_of(const int32_t* prefix, int bg, int P, int64_t T) {
    return P > 0 ? last_cta_of(prefix, bg, P, T) - first_cta_of(prefix, bg, T) + 1 : 0;
}

// Work range of CTA k: units [k*T, min((k+1)*T, W)).
__host__ __device__ inline void cta_meta(const int32_t* prefix, int BG, int64_t W, int64_t T, int k,
                                         int32_t* meta) {
    int64_t u0 = (int64_t)k * T;
    int64_t u1 = u0 + T;
    if (u0 > W) u0 = W;
    if (u1 > W) u1 = W;
    int bb, bp, eb, ep;
    locate_unit(prefix, BG, W, u0, &bb, &bp);
    locate_unit(prefix, BG, W, u1, &eb, &ep);
    int first_split = 0;
    if (bb < BG) {
        int P = pages_in_prefix(prefix, bb);
        if (P > 0) {
            first_split = k - first_cta_of(prefix, bb, T);
            if (first_split < 0) first_split = 0;
        }
    }
    meta[kMetaBeginBg] = bb;
    meta[kMetaBeginPage] = bp;
    meta[kMetaEndBg] = eb;
    meta[kMetaEndPage] = ep;
    meta[kMetaFirstSplit] = first_split;
    meta[5] = meta[6] = meta[7] = 0;
}

// Upper bound of partial slots: every CTA has at most two partial items.
__host__ __device__ inline int64_t max_slots(int G) { return 2 * (int64_t)G; }

// ---- partial-output slots of the one-CTA kernels ----
// CTA k writes the partial of its first work item to slot 2k and that of its
// last item (when that is another, split request-group) to slot 2k + 1, so a
// CTA places its partials without knowing any other CTA's split count.  A
// request-group whose first page is on CTA c0 and that is split ns ways then
// keeps split i >= 1 in slot 2 (c0 + i), since it opens each later CTA's
// range, and split 0 in slot 2 c0 if it also opens c0's range, else 2 c0 + 1.
// (CTA-pair plans, whose head groups share each range, number their slots
// (base + split) * groups + group, with base a running count over requests.)
__host__ __device__ inline int cta_slot(int k, bool first_item) { return 2 * k + (first_item ? 0 : 1); }
__host__ __device__ inline int first_split_slot(const int32_t* prefix, int bg, int64_t T) {
    const int c0 = first_cta_of(prefix, bg, T);
    return cta_slot(c0, (int64_t)c0 * T >= (int64_t)prefix[bg]);
}
__host__ __device__ inline int64_t split_slot(int slot0, int i) {
    return i == 0 ? (int64_t)slot0 : 2 * ((int64_t)(slot0 >> 1) + i);
}

}  // namespace mla
