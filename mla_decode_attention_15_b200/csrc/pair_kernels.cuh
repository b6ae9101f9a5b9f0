// CTA-pair decode kernel for wide query groups (h * s_q > 64 query columns per
// request), sm_100a.
//
// The method is the one of decode_kernels.cuh (absorbed-MQA MLA decode, a
// 576-wide latent row is the key and its first 512 columns the value;
// FlashMLA-ETAP technical summary, "Mecanismo Central"; GQLA summary,
// "Caminho MQA-Absorvido"), at a shape the one-CTA kernel serves badly: with
// 128 and more query columns per request the decode is bound by the tensor
// pipe (GQLA summary, same section: ~242 FLOP/B at s_q 1 and 128 heads), and
// the one-CTA kernel's MMAs (N <= 64 query columns, M = 64 tokens) run at a
// third to two thirds of the per-SM rate.  On B200 a tcgen05.mma costs the
// pipe about 48 cycles up to a size, so the number of MMAs per unit of work
// decides the rate; a pair of SMs issuing .cta_group::2 MMAs doubles M.
//
// A work item is (request, 128 query columns) on a cluster of two CTAs; CTA r
// owns query columns [64 r, 64 r + 64) of the item.  Per step of 128 tokens
// (two pages: CTA 0 loads the first, CTA 1 the second):
//
//   GEMM1  S = Q K^T     pair MMA M = 128 query columns (64 from each CTA's
//                        Q), N = 128 tokens (each CTA supplies its page's
//                        rows), K = 576: 36 MMAs.  Each CTA's TMEM receives
//                        its own 64 columns x all 128 tokens (measured layout:
//                        lanes 0-63 the first 64 tokens, lanes 64-127 the
//                        next 64, in N/2 = 64 TMEM columns).
//   softmax              per CTA, over its own columns only: every score of
//                        a column is in this CTA, so nothing crosses the pair.
//   GEMM2  O = P V       pair MMA M = 128 query columns (P from each CTA),
//                        N = 256 value columns (each CTA supplies 128 of them
//                        for all 128 tokens), K = 16 tokens: 2 x 8 MMAs.
//                        Each CTA's TMEM holds O for its own 64 columns and
//                        all 512 value columns, so the lazy rescale and the
//                        epilogue stay inside the CTA.
//
// This is the pages' order of the two contractions, not transposed: the
// transposition put the long KV axis in M because a few query columns were
// too narrow for the MMA; here 128 columns fill M by themselves.
//
// Roles per CTA (12 warps): warp 0 loads Q and the pages for GEMM1 (a ring
// of 9 boxes of 64 tokens x 64 columns), warp 3 loads the value columns for
// GEMM2 (a ring of 4 slots of 128 columns x 64 tokens), warp 1 of CTA 0
// issues every MMA of the pair, warp 2 allocates TMEM, warps 4-11 run the
// softmax and the epilogue.  Each CTA loads into its own shared memory; the
// copies of both CTAs complete on CTA 0's "full" barriers (.cta_group::2
// loads), which CTA 0 arms for the bytes of both, so the issuer needs no
// software relay.  Signals from CTA 1's threads to CTA 0 (S read, P written,
// O read) are relaxed remote arrives (see sm100_ptx.cuh for why not release).
// Every wait is bounded (1 s); on expiry the CTA raises MLA_STATUS_TIMEOUT,
// leaves its loops, drains its own copies and MMAs, and both CTAs meet
// (bounded) before releasing TMEM and exiting, so neither touches the other's
// shared memory after it is gone.
#pragma once

#include "decode_kernels.cuh"

namespace mla {

// Ring slots hold several boxes under one pair of barriers: measured on
// B200 (148 CTAs, one issuing thread each), 8 KB tensor boxes reach ~7 TB/s
// from L2 when every box has its own barrier round trip, and ~19 TB/s when
// the 9 boxes of a page share one.  The round trips, not the bytes, bound a
// ring of single boxes.
struct PairSmem {
    static constexpr int kBoxBytes = 8192;                      // 64 rows x 64 bf16 columns, 128-B swizzle
    static constexpr int kQOff = 0;                             // Q of this CTA's 64 columns: 9 boxes
    static constexpr int kGBoxesPerSlot = 3;                    // GEMM1 ring: 3 boxes of the page per slot
    static constexpr int kGSlotsPerStep = 9 / kGBoxesPerSlot;
    static constexpr int kGSlots = 3;                           // one step of lookahead
    static constexpr int kGSlotBytes = kGBoxesPerSlot * kBoxBytes;
    static constexpr int kGOff = kQOff + 9 * kBoxBytes;
    static constexpr int kVSlots = 2;                           // GEMM2 ring: one slot per page of a step
    static constexpr int kVSlotBytes = 4 * kBoxBytes;           // 2 value chunks x 128 columns x 64 tokens
    static constexpr int kVOff = kGOff + kGSlots * kGSlotBytes;
    static constexpr int kPOff = kVOff + kVSlots * kVSlotBytes; // P: 64 rows x 128 tokens (2 K blocks)
    static constexpr int kPBytes = 2 * kBoxBytes;
    static constexpr int kRedOff = kPOff + kPBytes;             // float [2][64][4]
    static constexpr int kBarOff = kRedOff + 2 * 64 * 4 * 4;
    static constexpr int kNumBars = 56;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;     // tmem base, abort flag
    static constexpr int kBytes = kMiscOff + 16;
    // TMEM (512 columns allocated for the pair): S double-buffered (64
    // columns each), O as two chunks of 256 value columns (128 TMEM columns
    // each: lanes 0-63 the first 128 values, lanes 64-127 the next 128).
    static constexpr int kSCol = 0;
    static constexpr int kOCol = 128;
    static constexpr int kTmemCols = 512;
    static_assert(kBytes <= 227 * 1024, "shared memory budget");
    static_assert(kGOff % 1024 == 0 && kVOff % 1024 == 0 && kPOff % 1024 == 0, "swizzle atoms need 1 KB alignment");
};

enum PairBar {
    pQFull = 0, pQEmpty,
    pGFull0,
    pGEmpty0 = pGFull0 + PairSmem::kGSlots,
    pVFull0 = pGEmpty0 + PairSmem::kGSlots,
    pVEmpty0 = pVFull0 + PairSmem::kVSlots,
    pSFull0 = pVEmpty0 + PairSmem::kVSlots, pSFull1,
    pSEmpty0, pSEmpty1,
    pPFull, pPEmpty, pOEmpty,
    pRed0, pRed1, pSum, pSumRead,
    pExit, pMmaDone,
    pBarCount
};
static_assert(pBarCount <= PairSmem::kNumBars, "barrier slots");

constexpr int kPairThreads = 384;
constexpr int kPairSoftmaxWarp0 = 4;
constexpr int kPairSoftmaxThreads = 256;
constexpr int kPairArrivals = 16;  // softmax warps of both CTAs, one elected lane each
constexpr int kPairCols = 128;     // query columns of a work item
constexpr uint16_t kPairMask = 0x3;

// CTA 1's copies may still be in flight when its producer gives up (they
// complete on CTA 0's barriers, which CTA 1 cannot wait on): it lets them
// land for this long before the pair meets to exit.
constexpr uint64_t kPeerDrainNs = 100000;

__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < ns) {
    }
}

// ---- work walk: ranges of (request, step) shared by the request's groups ----
struct PairItem {
    int b, g, s0, s1, L, P, slot;
    bool unsplit;
};

struct PairIter {
    int b, begin_b, begin_s, end_b, end_s, first_split;

    __device__ void init(const int32_t* meta) {
        begin_b = ld_nc_after_wait(meta + kMetaBeginBg);
        begin_s = ld_nc_after_wait(meta + kMetaBeginPage);
        end_b = ld_nc_after_wait(meta + kMetaEndBg);
        end_s = ld_nc_after_wait(meta + kMetaEndPage);
        first_split = ld_nc_after_wait(meta + kMetaFirstSplit);
        b = begin_b;
    }

    // p.BG = requests (the plan's rows); p.Hg = head groups walking each range.
    __device__ bool next(const FwdParams& p, const int32_t* bginfo, int g, PairItem& it) {
        while (b <= end_b && b < p.BG) {
            const int cur = b++;
            const int L = clamp_seqlen(__ldg(p.seqlens + cur), p.max_blocks);
            const int S = blocks_of(L, kStepShift);
            const int s0 = (cur == begin_b) ? begin_s : 0;
            int s1 = (cur == end_b) ? end_s : S;
            if (s1 > S) s1 = S;
            if (s0 >= s1) continue;
            it.b = cur;
            it.g = g;
            it.s0 = s0;
            it.s1 = s1;
            it.L = L;
            it.P = pages_of(L);
            it.unsplit = (s0 == 0 && s1 == S);
            it.slot = -1;
            if (!it.unsplit) {
                const int s = ld_nc_after_wait(bginfo + kBgWords * cur) + ((cur == begin_b) ? first_split : 0);
                const int slot = s * p.Hg + g;
                it.slot = (s >= 0 && slot < p.slots_cap) ? slot : -1;
            }
            return true;
        }
        return false;
    }
};

// Physical page of logical page `page` of request b; a page past the request
// (the second page of an odd final step) reads the step's first page
// instead: its tokens are masked, but the MMA still reads the slot, whose
// contents must be finite.
__device__ __forceinline__ int pair_page(const FwdParams& p, const int32_t* bt, const PairItem& it, int page,
                                         int step) {
    int ph = __ldg(bt + (page < it.P ? page : 2 * step));
    if ((unsigned)ph >= (unsigned)p.num_blocks) {
        atomicOr(p.status, MLA_STATUS_BAD_BLOCK_TABLE);
        ph = 0;
    }
    return ph;
}

// ---- producers ----
// Warp 0: Q of each item (after the item's first step of boxes, so that those
// flow while the previous item finishes), then the 9 boxes of this CTA's page
// of every step.  Each CTA loads into its own shared memory; the copies
// complete on CTA 0's barrier, which CTA 0 arms for both CTAs' bytes.
__device__ void pair_gproducer(const CUtensorMap* kv_map, const CUtensorMap* q_map, const FwdParams& p,
                               const int32_t* meta, const int32_t* bginfo, int g, uint32_t rank, uint8_t* smem,
                               const Ctl& ctl) {
    using L = PairSmem;
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    const uint32_t g_s = smem_addr(smem + L::kGOff);
    const uint32_t q_s = smem_addr(smem + L::kQOff);
    const uint64_t policy = l2_policy_evict_normal();
    PairIter it;
    it.init(meta);
    PairItem item;
    uint32_t g_it = 0, q_it = 0;
    uint32_t issued[L::kGSlots] = {};
    bool stall = p.test_stall != 0 && rank == 0;
    bool ok = true;
    const bool lead = rank == 0;
    auto full_of = [&](int bar) { return mapa_shared(bar0 + 8 * bar, 0); };
    MLA_TRACE_DECL(0);
    while (ok && it.next(p, bginfo, g, item)) {
        const int32_t* bt = p.block_table + (size_t)item.b * p.max_blocks;
        for (int j = item.s0; ok && j < item.s1; ++j) {
            MLA_TRACE_EV(kTrProdIssue);
            const int phys = pair_page(p, bt, item, 2 * j + (int)rank, j);
#pragma unroll 1
            for (int t = 0; t < L::kGSlotsPerStep; ++t) {
                const int gs = g_it % L::kGSlots;
                ok = wait_bounded(bar0 + 8 * (pGEmpty0 + gs), ((g_it / L::kGSlots) & 1) ^ 1, ctl);
                if (!ok) break;
                MLA_TRACE_EV(kTrBoxEmpty);
                if (stall) {  // test hook: this slot is never loaded, so its wait runs out
                    stall = false;
                    ++g_it;
                    continue;
                }
                if (lead) mbar_arrive_expect_tx(bar0 + 8 * (pGFull0 + gs), 2 * L::kGSlotBytes);
                const uint32_t full = full_of(pGFull0 + gs);
#pragma unroll
                for (int u = 0; u < L::kGBoxesPerSlot; ++u) {
                    const int c = t * L::kGBoxesPerSlot + u;
                    tma_load_3d_pair(g_s + gs * L::kGSlotBytes + u * L::kBoxBytes, kv_map, full, 64 * c, 0, phys,
                                     policy);
                }
                MLA_TRACE_EV(kTrBoxIssued);
                ++issued[gs];
                ++g_it;
            }
            if (ok && j == item.s0) {
                ok = wait_bounded(bar0 + 8 * pQEmpty, (q_it & 1) ^ 1, ctl);
                if (!ok) break;
                if (lead) mbar_arrive_expect_tx(bar0 + 8 * pQFull, 2 * 9 * L::kBoxBytes);
                const int row0 = item.b * p.N + item.g * kPairCols + 64 * (int)rank;
#pragma unroll 1
                for (int c = 0; c < 9; ++c)
                    tma_load_2d_pair(q_s + c * L::kBoxBytes, q_map, full_of(pQFull), 64 * c, row0);
                ++q_it;
            }
        }
    }
    if (!ok) {  // let the copies already issued land before the CTA exits
        if (lead) {
            for (int k = 0; k < L::kGSlots; ++k)
                if (issued[k] > 0) wait_drain(bar0 + 8 * (pGFull0 + k), (issued[k] - 1) & 1);
            if (q_it > 0) wait_drain(bar0 + 8 * pQFull, (q_it - 1) & 1);
        } else {
            spin_ns(kPeerDrainNs);
        }
    }
}

// Warp 3: the value columns this CTA supplies to GEMM2 (rank 0: values
// 256c + [0, 128), rank 1: 256c + [128, 256) of chunk c), for both pages of
// every step, as slots of 2 boxes in the order GEMM2 reads them.
__device__ void pair_vproducer(const CUtensorMap* kv_map, const FwdParams& p, const int32_t* meta,
                               const int32_t* bginfo, int g, uint32_t rank, uint8_t* smem, const Ctl& ctl) {
    using L = PairSmem;
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    const uint32_t v_s = smem_addr(smem + L::kVOff);
    const uint64_t policy = l2_policy_evict_normal();
    PairIter it;
    it.init(meta);
    PairItem item;
    uint32_t v_it = 0;
    uint32_t issued[L::kVSlots] = {};
    bool ok = true;
    const bool lead = rank == 0;
    MLA_TRACE_DECL(2);
    while (ok && it.next(p, bginfo, g, item)) {
        const int32_t* bt = p.block_table + (size_t)item.b * p.max_blocks;
        for (int j = item.s0; ok && j < item.s1; ++j) {
            MLA_TRACE_EV(kTrItem);
#pragma unroll 1
            for (int pi = 0; pi < 2; ++pi) {
                const int phys = pair_page(p, bt, item, 2 * j + pi, j);
                const int vs = v_it % L::kVSlots;
                ok = wait_bounded(bar0 + 8 * (pVEmpty0 + vs), ((v_it / L::kVSlots) & 1) ^ 1, ctl);
                if (!ok) break;
                if (lead) mbar_arrive_expect_tx(bar0 + 8 * (pVFull0 + vs), 2 * L::kVSlotBytes);
                const uint32_t full = mapa_shared(bar0 + 8 * (pVFull0 + vs), 0);
                const uint32_t dst = v_s + vs * L::kVSlotBytes;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {  // chunk ch: boxes 4 ch + 2 rank, +1 (128 value columns)
                    const int col = 64 * (4 * ch + 2 * (int)rank);
                    tma_load_3d_pair(dst + ch * 2 * L::kBoxBytes, kv_map, full, col, 0, phys, policy);
                    tma_load_3d_pair(dst + ch * 2 * L::kBoxBytes + L::kBoxBytes, kv_map, full, col + 64, 0, phys,
                                     policy);
                }
                ++issued[vs];
                ++v_it;
            }
        }
    }
    if (!ok) {
        if (lead) {
            for (int k = 0; k < L::kVSlots; ++k)
                if (issued[k] > 0) wait_drain(bar0 + 8 * (pVFull0 + k), (issued[k] - 1) & 1);
        } else {
            spin_ns(kPeerDrainNs);
        }
    }
}

// ---- the issuer (one thread of CTA 0) ----
// Order of issue: for each step t, GEMM1 of t (after Q, for an item's first
// step), then GEMM2 of step t - 1: the softmax of a step overlaps GEMM1 of
// the next.  GEMM2 of an item's last step follows GEMM1 of the next item's
// first step.  Every wait is on a barrier of this CTA: the copies of both
// CTAs complete on it, and CTA 1's threads arrive on it remotely.
__device__ void pair_issuer(const FwdParams& p, const int32_t* meta, const int32_t* bginfo, int g, uint8_t* smem,
                            uint32_t tmem, const Ctl& ctl) {
    using L = PairSmem;
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    const uint32_t q_s = smem_addr(smem + L::kQOff);
    const uint32_t g_s = smem_addr(smem + L::kGOff);
    const uint32_t v_s = smem_addr(smem + L::kVOff);
    const uint32_t p_s = smem_addr(smem + L::kPOff);
    constexpr uint32_t kIdesc1 = idesc_bf16_f32(128, 128, 0, 0);  // S = Q K^T: K-major A and B
    constexpr uint32_t kIdesc2 = idesc_bf16_f32(128, 256, 0, 1);  // O = P V: K-major P, MN-major V
    const uint64_t qd0 = smem_desc(q_s, 16, 1024, kSwizzle128);
    const uint64_t gd0 = smem_desc(g_s, 16, 1024, kSwizzle128);
    const uint64_t pd0 = smem_desc(p_s, 16, 1024, kSwizzle128);
    const uint64_t vd0 = smem_desc(v_s, L::kBoxBytes, 1024, kSwizzle128);
    PairIter it;
    it.init(meta);
    PairItem item;
    uint32_t g_it = 0, v_it = 0, s_it = 0, item_it = 0, q_it = 0;
    bool ok = true;
    // the deferred GEMM2: its step, and whether that step starts an item
    bool pend = false, pend_first = false;
    uint32_t pend_s = 0, pend_item = 0;
    MLA_TRACE_DECL(1);
    auto gemm2 = [&]() -> bool {
        if (!wait_bounded(bar0 + 8 * pPFull, pend_s & 1, ctl)) return false;
        MLA_TRACE_EV(kTrMmaPFull);
        if (pend_first && !wait_bounded(bar0 + 8 * pOEmpty, (pend_item & 1) ^ 1, ctl)) return false;
#pragma unroll 1
        for (int pi = 0; pi < 2; ++pi) {  // the step's two pages
            const int vs = v_it % L::kVSlots;
            if (!wait_bounded(bar0 + 8 * (pVFull0 + vs), (v_it / L::kVSlots) & 1, ctl)) return false;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t a = pd0 + ((pi * L::kBoxBytes + k * 32) >> 4);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const uint64_t b = vd0 + ((vs * L::kVSlotBytes + ch * 2 * L::kBoxBytes + k * 2048) >> 4);
                    umma_f16_pair(tmem + L::kOCol + 128 * ch, a, b, kIdesc2, (pend_first && pi == 0 && k == 0) ? 0u : 1u);
                }
            }
            umma_commit_pair_mc(bar0 + 8 * (pVEmpty0 + vs), kPairMask);
            ++v_it;
        }
        umma_commit_pair_mc(bar0 + 8 * pPEmpty, kPairMask);
        MLA_TRACE_EV(kTrMmaG2Issued);
        return true;
    };
    while (ok && it.next(p, bginfo, g, item)) {
        for (int j = item.s0; ok && j < item.s1; ++j) {
            if (j == item.s0) {
                ok = wait_bounded(bar0 + 8 * pQFull, q_it & 1, ctl);
                if (!ok) break;
            }
            const int sb = s_it & 1;
            MLA_TRACE_EV(kTrMmaKvFull);
            ok = wait_bounded(bar0 + 8 * (pSEmpty0 + sb), ((s_it >> 1) & 1) ^ 1, ctl);
            if (!ok) break;
#pragma unroll 1
            for (int t = 0; t < L::kGSlotsPerStep; ++t) {
                const int gs = g_it % L::kGSlots;
                ok = wait_bounded(bar0 + 8 * (pGFull0 + gs), (g_it / L::kGSlots) & 1, ctl);
                if (!ok) break;
                MLA_TRACE_EV(kTrBoxFull);
                tc_fence_after();
#pragma unroll
                for (int u = 0; u < L::kGBoxesPerSlot; ++u) {
                    const int c = t * L::kGBoxesPerSlot + u;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16_pair(tmem + L::kSCol + 64 * sb, qd0 + ((c * L::kBoxBytes + k * 32) >> 4),
                                      gd0 + ((gs * L::kGSlotBytes + u * L::kBoxBytes + k * 32) >> 4), kIdesc1,
                                      (c | k) ? 1u : 0u);
                }
                umma_commit_pair_mc(bar0 + 8 * (pGEmpty0 + gs), kPairMask);
                ++g_it;
            }
            if (!ok) break;
            umma_commit_pair_mc(bar0 + 8 * (pSFull0 + sb), kPairMask);
            if (j == item.s1 - 1) umma_commit_pair_mc(bar0 + 8 * pQEmpty, kPairMask);
            MLA_TRACE_EV(kTrMmaG1Issued);
            if (pend) {
                ok = gemm2();
                if (!ok) break;
            }
            pend = true;
            pend_first = (j == item.s0);
            pend_s = s_it;
            pend_item = item_it;
            ++s_it;
        }
        if (!ok) break;
        ++q_it;
        ++item_it;
    }
    if (ok && pend) ok = gemm2();
    // Drain before the pair meets to release TMEM: the barrier completes when
    // every MMA this thread issued (into both CTAs) is done.
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar0 + 8 * pMmaDone)
                 : "memory");
    wait_drain(bar0 + 8 * pMmaDone, 0);
}

// ---- softmax and epilogue (warps 4-11 of each CTA) ----
// Thread layout: warp w reads TMEM lane quadrant q = w % 4 and token half
// h = (w - 4) / 4 of each page.  Lane L = 32 q + lane of S holds query column
// c = L % 64 of this CTA, page (L / 64) of the step; the thread takes its 32
// tokens 64 (L / 64) + 32 h + [0, 32).  The four threads of a column share
// page maxima through shared memory; each keeps the running max m (log2
// units, lazy: moved only when a page max exceeds it by 2^8) and its own part
// of the row sum.  O of column c: lane c holds values 256 k + [0, 128), lane
// 64 + c values 256 k + [128, 256), chunk k in TMEM columns 128 k + [0, 128);
// the thread with token half h rescales and writes chunk h of its lane.
__device__ void pair_softmax(const FwdParams& p, const int32_t* meta, const int32_t* bginfo, int g, uint32_t rank,
                             uint8_t* smem, uint32_t tmem, const Ctl& ctl) {
    using L = PairSmem;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int h = (warp - kPairSoftmaxWarp0) >> 2;
    const int Ln = 32 * q + lane;
    const int c = Ln & 63;
    const int pi = Ln >> 6;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);
    uint8_t* prow = smem + L::kPOff + pi * L::kBoxBytes + (c >> 3) * 1024 + (c & 7) * 128;
    // one arrival per warp on CTA 0's barrier (a local arrive in CTA 0)
    auto arrive_leader = [&](int bar) {
        __syncwarp();
        if (lane == 0) {
            if (rank == 0) mbar_arrive(bar0 + 8 * bar);
            else mbar_arrive_remote(mapa_shared(bar0 + 8 * bar, 0));
        }
    };
    PairIter it;
    it.init(meta);
    PairItem item;
    uint32_t s_it = 0, item_it = 0;
    bool ok = true;
#ifdef MLA_TRACE
    Tracer tracer_(3, threadIdx.x == 32 * kPairSoftmaxWarp0);
#endif
    while (ok && it.next(p, bginfo, g, item)) {
        const int gc = item.g * kPairCols + 64 * (int)rank + c;  // query column of the request
        int lvis = 0;
        if (gc < p.N) lvis = (p.causal && p.s_q > 1) ? item.L - p.s_q + 1 + gc / p.heads : item.L;
        float m = -INFINITY;  // running max, log2 units
        float l = 0.f;        // this thread's part of the row sum, relative to m
        for (int j = item.s0; j < item.s1; ++j) {
            const int sb = s_it & 1;
            const int par = s_it & 1;
            ok = wait_warp(bar0 + 8 * (pSFull0 + sb), (s_it >> 1) & 1, ctl);
            if (!ok) break;
            MLA_TRACE_EV(kTrSmSFull);
            tc_fence_after();
            float x[32];
            tmem_ld_x32(tmem + lane_base + L::kSCol + 64 * sb + 32 * h, x);
            tmem_ld_wait();
            tc_fence_before();
            arrive_leader(pSEmpty0 + sb);
            const int t0 = j * 128 + 64 * pi + 32 * h;
            float mloc = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = (t0 + i < lvis) ? x[i] * p.scale_log2 : -INFINITY;
                mloc = fmaxf(mloc, x[i]);
            }
            float* rb = red + par * 256;
            rb[c * 4 + 2 * pi + h] = mloc;
            mbar_arrive(bar0 + 8 * (pRed0 + par));
            // speculative P with the running max; stands unless the max moves
            float e[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) e[i] = (x[i] == -INFINITY) ? 0.f : ex2_approx(x[i] - m);
            ok = wait_warp(bar0 + 8 * (pRed0 + par), (s_it >> 1) & 1, ctl);
            if (!ok) break;
            MLA_TRACE_EV(kTrSmXchg);
            const float4 r4 = *reinterpret_cast<const float4*>(rb + c * 4);
            const float pm = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
            const bool grow = pm > m + kRescaleLog2;  // false while the column has seen nothing
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m - pm);  // 0 when m is -inf
                m = pm;
#pragma unroll
                for (int i = 0; i < 32; ++i) e[i] = (x[i] == -INFINITY) ? 0.f : ex2_approx(x[i] - m);
            }
            float se = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) se += e[i];
            l = l * alpha + se;
            // GEMM2 of the previous step is done: P is free, O is stable.
            ok = wait_warp(bar0 + 8 * pPEmpty, (s_it & 1) ^ 1, ctl);
            if (!ok) break;
            MLA_TRACE_EV(kTrSmMaxDone);
            if (__any_sync(kFullMask, grow && j > item.s0)) {
                tc_fence_after();
                const float a = (grow && j > item.s0) ? alpha : 1.f;
#pragma unroll 1
                for (int blk = 0; blk < 4; ++blk) {
                    float o[32];
                    const uint32_t ta = tmem + lane_base + L::kOCol + 128 * h + 32 * blk;
                    tmem_ld_x32(ta, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; i += 16) {
                        float v[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u) v[u] = o[i + u] * a;
                        tmem_st_x16(ta + i, v);
                    }
                }
                tmem_st_wait();
            }
            // P row c, K block pi, tokens 32h + [0, 32): 64 bytes = 4 swizzled chunks
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(e[8 * cc + 2 * u], e[8 * cc + 2 * u + 1]);
                    w[u] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                *reinterpret_cast<uint4*>(prow + (((4 * h + cc) ^ (c & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            arrive_leader(pPFull);
            MLA_TRACE_EV(kTrSmPDone);
            ++s_it;
        }
        if (!ok) break;
        // ---- epilogue: the item's last GEMM2, row sums, O / l and LSE ----
        const uint32_t last = s_it - 1;
        ok = wait_warp(bar0 + 8 * pPEmpty, last & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        float* sb4 = red + ((last & 1) ^ 1) * 256;  // the other page-max buffer; see pSumRead below
        sb4[c * 4 + 2 * pi + h] = l;
        mbar_arrive(bar0 + 8 * pSum);
        ok = wait_warp(bar0 + 8 * pSum, item_it & 1, ctl);
        if (!ok) break;
        const float4 s4 = *reinterpret_cast<const float4*>(sb4 + c * 4);
        const float lsum = (s4.x + s4.y) + (s4.z + s4.w);
        // every thread has read the sums before the next item's first step
        // writes page maxima into the same buffer
        mbar_arrive(bar0 + 8 * pSumRead);
        const float inv = lsum > 0.f ? rcp_approx(lsum) : 0.f;
        if (pi == 0 && h == 0 && gc < p.N) {
            const float lse = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
            if (item.unsplit) {
                const int sq = gc / p.heads;
                const int head = gc - sq * p.heads;
                p.lse[((size_t)item.b * p.heads + head) * p.s_q + sq] = lse;
            } else if (item.slot >= 0) {
                p.lpart[(size_t)item.slot * kPairCols + 64 * rank + c] = lse;
            }
        }
        const int d0 = 256 * h + 128 * pi;  // value columns of this thread's chunk of O
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            float o[32];
            tmem_ld_x32(tmem + lane_base + L::kOCol + 128 * h + 32 * blk, o);
            tmem_ld_wait();
            const int d = d0 + 32 * blk;
            if (!item.unsplit) {
                if (item.slot >= 0) {
                    float* dst = p.opart + ((size_t)item.slot * kPairCols + 64 * rank + c) * kDv + d;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + i) =
                            make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
                }
            } else if (gc < p.N) {
                const size_t row = (size_t)item.b * p.N + gc;
                if (p.out_f32) {
                    float* dst = static_cast<float*>(p.out) + row * kDv + d;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + i) =
                            make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
                } else {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + row * kDv + d;
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[i + 2 * u] * inv, o[i + 2 * u + 1] * inv);
                            w[u] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
        if (!item.unsplit && item.slot < 0 && threadIdx.x == 32 * kPairSoftmaxWarp0)
            atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
        ok = wait_warp(bar0 + 8 * pSumRead, item_it & 1, ctl);
        if (!ok) break;
        tc_fence_before();
        arrive_leader(pOEmpty);
        ++item_it;
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    mla_decode_pair_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                           const FwdParams p) {
    using L = PairSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    griddep_wait();
    griddep_launch_dependents();
    // Both CTAs of the cluster read the same header and take the same exits.
    const int32_t* hdr = p.sched;
    const int cluster = blockIdx.x >> 1;
    auto h = [&](int i) { return ld_nc_after_wait(hdr + i); };
    if (h(kHdrMagic) != kSchedMagic || h(kHdrG) != p.G || h(kHdrBG) != p.BG || h(kHdrHg) != 1 ||
        h(kHdrNG) != kPairCols || h(kHdrShift) != kStepShift || h(kHdrShareHg) != p.Hg) {
        if (threadIdx.x == 0 && rank == 0) atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
        return;
    }
    if ((smem_addr(smem_raw) & 1023u) != 0) {  // the layout has no slack to realign the base
        if (threadIdx.x == 0) atomicOr(p.status, MLA_STATUS_SMEM_ALIGN);
        return;
    }
    const int range = cluster / p.Hg;
    const int g = cluster - range * p.Hg;
    const bool idle = range >= p.G;  // clusters past the last range have no work
    const int32_t* meta = hdr + kHdrWords + (size_t)(idle ? 0 : range) * kMetaWords;
    const int32_t* bginfo = hdr + bg_offset_words(p.G);
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    if (threadIdx.x == 0) {
        for (int i = 0; i < pBarCount; ++i) {
            uint32_t count = 1;
            if (i == pSEmpty0 || i == pSEmpty1 || i == pPFull || i == pOEmpty) count = kPairArrivals;
            if (i == pRed0 || i == pRed1 || i == pSum || i == pSumRead) count = kPairSoftmaxThreads;
            mbar_init(bar0 + 8 * i, count);
        }
        *abort_flag = idle ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(smem_addr(tmem_slot), L::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl ctl{abort_flag, p.status};
    if (!idle) {
        if (warp == 0) {
            if (lane == 0) {
                prefetch_tensormap(&kv_map);
                prefetch_tensormap(&q_map);
                pair_gproducer(&kv_map, &q_map, p, meta, bginfo, g, rank, smem, ctl);
            }
        } else if (warp == 1) {
            if (lane == 0 && rank == 0) pair_issuer(p, meta, bginfo, g, smem, tmem, ctl);
        } else if (warp == 3) {
            if (lane == 0) pair_vproducer(&kv_map, p, meta, bginfo, g, rank, smem, ctl);
        } else if (warp >= kPairSoftmaxWarp0) {
            pair_softmax(p, meta, bginfo, g, rank, smem, tmem, ctl);
        }
    }
    // The pair meets before TMEM is released and before either CTA exits, so
    // that no MMA, copy or remote arrive touches a CTA that is gone.
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_remote(mapa_shared(bar0 + 8 * pExit, rank ^ 1u));
        wait_drain(bar0 + 8 * pExit, 0);
    }
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, L::kTmemCols);
    }
}

}  // namespace mla
