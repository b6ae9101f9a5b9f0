// sm_100a kernels of absorbed-MQA MLA decode in the transposed ("ETAP") order.
//
// Method (FlashMLA-ETAP technical summary, gist.science pt 2506.01969,
// "Mecanismo Central"): instead of S = Q K^T, softmax over keys, O = P V,
// compute S^T = K Q^T, P^T = softmax(S^T) along the KV axis and
// O = (V^T P^T)^T, so the long KV axis is the MMA M dimension and the few
// query columns (heads x new tokens) are N.  The cache is the absorbed-MQA
// latent cache of the GQLA summary (gist.science pt 2605.15250, "Caminho
// MQA-Absorvido"): one 576-wide row per token, key = whole row, value = the
// first 512 columns.  "Detalhes de Implementação" of the FlashMLA-ETAP summary
// describes a producer/consumer split inside one CTA on Hopper; here the roles
// are re-cut for Blackwell:
//
//   warp 0        TMA producer: Q of the work item, then every 64-token page
//                 gathered through the block table (9 boxes of 64x64 bf16,
//                 128-byte swizzle) into a 2-stage ring of 72 KB stages.
//   warps 1, 2    one thread each issues GEMM1  S^T[64 x N] = K[64 x 576] . Q^T
//                 (M = 64 tokens, K-major A and B) into TMEM; the two issuers
//                 take alternate 64-column boxes into separate accumulators,
//                 which the softmax adds up.
//   warp 3 (, 4)  one thread per warp issues GEMM2  O^T[512 x N] += V^T[512 x 64] . P^T
//                 (4 x M = 128 d_v chunks, MN-major A and B; with two issuers each
//                 takes two chunks); V^T is the same shared-memory page read
//                 through a second (MN-major) descriptor.  Separate issuers let
//                 GEMM2 of page j start as soon as P^T(j) is ready,
//                 independently of when page j+1 lands.
//   last 4 warps  softmax over the KV axis (one TMEM lane = one token), lazy
//                 rescale of O^T in TMEM, P^T to shared memory as bf16, and the
//                 epilogue (O = O^T / l transposed back, LSE), either final or
//                 as an fp32 partial of a split request.
//
// Every wait on an mbarrier is bounded: after kWaitLimitNs the waiting role
// raises MLA_STATUS_TIMEOUT and a CTA-wide abort flag, all roles leave their
// loops, in-flight copies and MMAs are drained (again with a limit) and TMEM
// is released before the CTA exits.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr uint32_t kFullMask = 0xffffffffu;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
// Warps: TMA producer, G1<NG>::kIssuers GEMM1 issuers, G2Issuers<NG> GEMM2 issuers,
// then the 4 softmax warps.  The softmax of NG = 32 needs more than the 224
// registers per thread a ninth warp would leave, so it keeps one GEMM2 issuer.
// A small tcgen05.mma (N <= 64, M = 64 or 128) occupies the tensor pipe for
// about 50 cycles whatever its size, so the 52 MMAs of a 16-column page keep
// the pipe busy for most of a page's HBM time, and the page rate follows the
// time GEMM1 and GEMM2 take to issue.  Issued from several threads (each into
// its own accumulator) they complete sooner; measured on B200 at bs16 x 64K,
// decode kernel per launch: GEMM1 from 1 / 2 / 3 threads 247.3 / 214.5 /
// 204.3 us, and 4 GEMM2 threads (one per d_v chunk) with a one-page L2
// prefetch 203.1 us.  32- and 64-column groups keep 2 + 1 issuers: their
// softmax needs the registers a larger CTA would take away.
// Cache shapes.  ShapeMla (absorbed MQA, the main path): a 576-wide row
// (512 latent + 64 RoPE) is the key and its first 512 columns the value.
// ShapeGqa (the GQLA summary's "Caminho GQA"): per token, g groups of
// 128-wide keys, then g groups of 128-wide values, then one shared 64-wide
// RoPE key; a work item reads its group's key (2 boxes of 64 columns), the
// RoPE key and its group's value.  Stage box kRopeBox is read by GEMM1 only,
// so the softmax writes the page's P^T over it.
struct ShapeMla {
    static constexpr int kDqk = 576, kDv = 512;
    static constexpr int kKBoxes = 9;      // K (and Q) boxes of 64 columns
    static constexpr int kStageBoxes = 9;  // boxes loaded per page
    static constexpr int kRopeBox = 8;
    static constexpr int kVChunks = 4;     // d_v / 128: GEMM2 chunks of 128 rows
    static constexpr bool kPrefetchL2 = true;  // a page is one contiguous 72 KB block
    static constexpr int kStages = 2;          // 72 KB page stages
    static constexpr bool kOneRun = true;      // a group's query columns are NG consecutive rows
    __host__ __device__ static constexpr int k_box(int c) { return c; }
    // first stage box of d_v chunk ch; the chunk's second box follows 8 KB on
    __host__ __device__ static constexpr int v_box(int ch) { return 2 * ch; }
    // cache column of stage box c for KV group kg of kv_groups
    __host__ __device__ static constexpr int col(int c, int, int) { return 64 * c; }
    __host__ __device__ static constexpr int row_width(int) { return kDqk; }
};
struct ShapeGqa {
    static constexpr int kDh = 128, kDrope = 64;
    static constexpr int kDqk = kDh + kDrope, kDv = kDh;
    static constexpr int kKBoxes = 3;      // K_g (2 boxes) + the RoPE key
    static constexpr int kStageBoxes = 5;  // K_g, K_g, RoPE, V_g, V_g
    static constexpr int kRopeBox = 2;
    static constexpr int kVChunks = 1;
    static constexpr bool kPrefetchL2 = false;  // a group's boxes are strided across the page
    static constexpr int kStages = 4;           // 40 KB page stages
    static constexpr bool kOneRun = false;     // one run of 16 heads per new token
    __host__ __device__ static constexpr int k_box(int c) { return c; }
    __host__ __device__ static constexpr int v_box(int) { return 3; }
    __host__ __device__ static constexpr int col(int c, int kg, int kv_groups) {
        return c < 2 ? kg * kDh + 64 * c : c == 2 ? 2 * kv_groups * kDh : kv_groups * kDh + kg * kDh + 64 * (c - 3);
    }
    __host__ __device__ static constexpr int row_width(int kv_groups) { return 2 * kv_groups * kDh + kDrope; }
};

template <int NG>
struct G1 {
    static constexpr int kIssuers = NG == 16 ? 3 : 2;  // GEMM1 issuer threads = S^T accumulators
};
// 64-column groups run 8 softmax warps: two column groups of 32 columns,
// each the 4 warps that reach the four TMEM lane quadrants.  Their 384
// threads leave 168 registers per thread at launch; warpgroup 0 (producer and
// issuers) gives registers back with setmaxnreg so that the softmax
// warpgroups can hold the per-column state of 32 columns.  (Measured on B200
// at bs32 x s_q 2 x 128 heads: a 16-warp layout with 4 GEMM2 issuers and
// 32-register issuers is slower, 648 vs 626 us per launch; a third GEMM1
// accumulator does not fit TMEM at 64 columns.)
template <int NG, class S = ShapeMla>
struct FwdWarps {
    static constexpr int kG2Issuers = NG == 16 && S::kVChunks >= 4 ? 4 : 1;  // 4: one per d_v chunk
    static constexpr int kFirstG2 = 1 + G1<NG>::kIssuers;
    static constexpr int kFirstSoftmax = kFirstG2 + kG2Issuers;
    // softmax column groups: 64-column MLA groups, and 32-column GQA groups
    // (whose 40 KB pages leave the softmax as the serial step)
    static constexpr int kColGroups = NG == 64 || (NG == 32 && S::kVChunks == 1) ? 2 : 1;
    static constexpr int kGroupCols = NG / kColGroups;     // query columns per group
    static constexpr int kSoftmaxThreads = 128 * kColGroups;
    static constexpr int kThreads = 32 * kFirstSoftmax + kSoftmaxThreads;
    static constexpr bool kSplitRegs = NG == 64;
    static constexpr int kRegsLaunch = 65536 / kThreads / 8 * 8;
    static constexpr int kRegsIssue = 56;                   // warpgroup 0 after setmaxnreg.dec
    static constexpr int kRegsSoftmax = 224;                // softmax warpgroups after setmaxnreg.inc
    static_assert(!kSplitRegs || kFirstSoftmax % 4 == 0, "setmaxnreg works on whole warpgroups");
    static_assert(!kSplitRegs || kRegsIssue * 32 * kFirstSoftmax + kRegsSoftmax * kSoftmaxThreads <=
                                     kRegsLaunch * kThreads,
                  "register split exceeds the launch allocation");
};
// P as two bf16 terms.  GEMM2 takes bf16 operands, and rounding P to bf16
// costs up to 2^-9 of each weight, which shows in the fp32 result of peaked
// rows (one token far above the rest).  Where the query group is at most 32
// columns wide, the softmax writes P = hi + lo (hi = bf16(P), lo = bf16(P -
// hi), together within 2^-17 of P) as 2 x NG columns of P^T, and GEMM2
// accumulates both halves of O^T in one MMA of N = 2 x NG: an MMA of N <= 64
// occupies the tensor pipe as long as one of N = 16, so the second term costs
// no MMA time.  The epilogue adds the halves.  64-column groups (N = 128 would
// double GEMM2's pipe time and O^T would need all of TMEM) keep one bf16 term;
// so does the GQA shape.
template <int NG, class S>
struct PSplit {
    static constexpr bool kOn = NG <= 32 && S::kVChunks == 4;
    static constexpr int kNP = kOn ? 2 * NG : NG;  // P^T columns = GEMM2 N = O^T columns per d_v chunk
};
// Rescale O only when the running max grows by > 2^8.  Measured on B200
// (bs16 x 64K decode kernel): an exact running max (rescale on any growth)
// costs 6% (202.2 -> 214.4 us); with O normalised by the sum of the
// bf16-rounded P the lazy max loses no accuracy on peaked rows.
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.693147180559945309f;
// GEMM1 (S^T = K Q^T, K = 576) accumulates into one TMEM accumulator per
// issuer; the softmax adds them.

// L2 prefetch of whole pages ahead of the shared-memory loads
// (cp.async.bulk.prefetch.L2, one 72 KB page per instruction).  With only two
// 72 KB stages per SM the refill then sees L2 rather than HBM latency.
// Measured on B200 at bs16 x 64K (decode kernel per launch): no prefetch
// 228.9 us, 1 page ahead 212.5, 2 pages 214.6, 4 pages 218.5, 8 pages 271.7.
// Short work items gain nothing and lose a little, so only items of at least
// kPrefetchMinPages pages prefetch.
// Measured as well: prefetching every page of an item into L2 when the item
// starts, on steps whose pages fit L2 (bs16 x 4K: 30.8 -> 35-37 us; 1 x 1K:
// 16.5 -> 18.4 us): the bulk prefetches delay the page loads behind them.
constexpr int kPrefetchPages = 1;
constexpr int kPrefetchMinPages = 16;

// Optional timeline tracing (build with -DMLA_TRACE): each role of each CTA
// stamps %globaltimer at pipeline events into a device buffer that the host
// copies out with mla_decode_trace_fetch().  Compiled out by default.
#ifdef MLA_TRACE
constexpr int kTraceCtas = 160;
constexpr int kTraceRoles = 4;
constexpr int kTraceCap = 1024;
__device__ unsigned long long g_mla_trace[kTraceCtas][kTraceRoles][kTraceCap];
__device__ unsigned int g_mla_trace_count[kTraceCtas][kTraceRoles];
enum TraceTag : unsigned {
    kTrProdIssue = 1,   // producer: stage free, page loads issued
    kTrMmaKvFull = 2,   // gemm1 issuer: page landed in shared memory
    kTrMmaPFull = 3,    // gemm2 issuer: P^T ready, GEMM2 about to issue
    kTrSmSFull = 4,     // softmax: S^T ready in TMEM
    kTrSmPDone = 5,     // softmax: P^T written (and O rescaled)
    kTrSmEpi0 = 6,      // softmax: epilogue start (last GEMM2 done)
    kTrSmEpi1 = 7,      // softmax: epilogue end
    kTrItem = 8,        // any role: new work item
    kTrSmMaxDone = 9,   // softmax: page column maxima written (before the exchange)
    kTrSmXchg = 10,     // softmax: exchange complete
    kTrSmPStored = 11,  // softmax: P^T stored
    kTrSmEpiSum = 12,   // softmax: row sums exchanged (epilogue)
    kTrSmEpiOut = 13,   // softmax: outputs written (epilogue)
    kTrSmEpiLse = 14,   // softmax: LSE written (epilogue)
    kTrMmaG1Issued = 15,  // gemm1 issuer: MMAs issued and committed
    kTrMmaG2Issued = 16,  // gemm2 issuer: MMAs issued and committed
    kTrBoxIssued = 17,    // CTA-pair producer: one GEMM1 box load issued
    kTrBoxFull = 18,      // CTA-pair issuer: one GEMM1 box seen full
    kTrBoxEmpty = 19,     // CTA-pair producer: one GEMM1 slot seen empty
};
struct Tracer {
    int cta, role;
    unsigned n;
    bool on;
    __device__ Tracer(int r, bool enabled = true) : cta(blockIdx.x), role(r), n(0), on(enabled) {}
    __device__ void ev(unsigned tag) {
        if (on && cta < kTraceCtas && n < kTraceCap)
            g_mla_trace[cta][role][n] = (static_cast<unsigned long long>(tag) << 56) |
                                        (stamp_timer_ns() & 0x00FFFFFFFFFFFFFFull);
        ++n;
    }
    __device__ ~Tracer() {
        if (on && cta < kTraceCtas) g_mla_trace_count[cta][role] = n;
    }
};
#define MLA_TRACE_DECL(role) Tracer tracer_(role)
#define MLA_TRACE_EV(tag) tracer_.ev(tag)
// Kernel-level stamps: per decode CTA [entry, plan readable, setup done, -,
// TMEM released, GEMM1 / GEMM2 / softmax role returned];
// for the whole step [schedule entry, schedule exit, first combine entry,
// first combine past its wait, last combine exit] (min / max over blocks).
__device__ unsigned long long g_mla_trace_k[kTraceCtas][8];
__device__ unsigned long long g_mla_trace_step[8];
__device__ unsigned long long g_mla_trace_comb[64][64];  // combine CTA (bg, column) exit
#define MLA_TRACE_K(slot) MLA_TRACE_K_BY(slot, 0)
#define MLA_TRACE_K_BY(slot, thread)                                           \
    do {                                                                       \
        if (threadIdx.x == (thread) && blockIdx.x < kTraceCtas)                \
            g_mla_trace_k[blockIdx.x][slot] = stamp_timer_ns();                \
    } while (0)
#define MLA_TRACE_STEP_MIN(slot) \
    do { if (threadIdx.x == 0) atomicMin(&g_mla_trace_step[slot], stamp_timer_ns()); } while (0)
#define MLA_TRACE_STEP_MAX(slot) \
    do { if (threadIdx.x == 0) atomicMax(&g_mla_trace_step[slot], stamp_timer_ns()); } while (0)
#else
#define MLA_TRACE_DECL(role)
#define MLA_TRACE_EV(tag)
#define MLA_TRACE_K(slot)
#define MLA_TRACE_K_BY(slot, thread)
#define MLA_TRACE_STEP_MIN(slot)
#define MLA_TRACE_STEP_MAX(slot)
#endif

struct FwdParams {
    const int32_t* sched;
    // Non-null: the kernel builds the plan itself from the lengths and writes
    // it here (the schedule buffer); null: it reads the plan in `sched`.
    int32_t* plan_out;
    const int32_t* block_table;
    const int32_t* seqlens;
    const uint8_t* kv;  // page pool base (for L2 prefetch)
    void* out;          // bf16 rows, or fp32 rows when out_f32
    float* lse;
    float* opart;  // [slots][NG][512]
    float* lpart;  // [slots][NG]
    int32_t* status;
    int s_q, heads, N, num_blocks, max_blocks, causal;
    int G, BG, Hg, slots_cap;  // plan ranges, plan rows, head groups per plan row, partial slots
    // One-CTA kernels: CTAs walking each plan range side by side, one per
    // head group (1: none; >1: the plan has one row per request and CTA c
    // walks range c / share for head group c % share).
    int share;
    int out_f32;       // MLA_FLAG_FP32_OUT: final rows are written as fp32
    float scale_log2;  // softmax_scale * log2(e)
    int test_stall;    // MLA_FLAG_TEST_STALL: leave the first page unloaded
    // Query columns of a work item: runs of run_rows consecutive rows, run r
    // at row offset r * run_stride + g * run_rows (one run for MLA groups;
    // one run per new token for GQA groups).  kv_groups: GQA groups.
    int run_rows, run_stride, kv_groups;
};
// Query column (in [0, N)) of column q of group g.
__device__ __forceinline__ int item_col(int run_rows, int run_stride, int g, int q) {
    const int r = q / run_rows;
    return r * run_stride + g * run_rows + (q - r * run_rows);
}
// The same for a kernel instance: a cache shape whose groups are one run of
// NG rows maps at compile time, without the division.
template <int NG, class S>
__device__ __forceinline__ int group_col(const FwdParams& p, int g, int q) {
    if constexpr (S::kOneRun) return g * NG + q;
    else return item_col(p.run_rows, p.run_stride, g, q);
}

struct CombineParams {
    const int32_t* sched;
    const float* opart;
    const float* lpart;
    void* out;  // bf16 rows, or fp32 rows when out_f32
    float* lse;
    int32_t* status;
    int s_q, heads, N, NG, Hg, G, BG, slots_cap;  // Hg, BG: head groups per request, request-groups
    int run_rows, run_stride;
    int out_f32;
    // The plan's own shape: plan_BG work items per plan row of bginfo, and
    // share = head groups that walked each work range side by side (1: the
    // plan has one row per request-group; else one row per request, and split
    // i of group g sits in slot (base + i) * share + g).
    int plan_BG, plan_Hg, shift, share;
    int plan_in_decode;  // the decode kernel built the plan (read it only after the wait)
};

// ------------------------------------------------------------------ layout
constexpr int kMaxStages = 4;
template <int NG, class S = ShapeMla>
struct FwdSmem {
    static constexpr int kStages = S::kStages;
    static constexpr int kBoxCols = 64;
    static constexpr int kBoxBytes = kPage * kBoxCols * 2;    // 8 KB: 64 tokens x 64 cols
    static constexpr int kBoxes = S::kStageBoxes;             // boxes per page (9 for MLA)
    static constexpr int kStageBytes = kBoxes * kBoxBytes;    // 72 KB: one MLA page
    static constexpr int kQBoxBytes = NG * 128;               // NG rows x 64 cols
    static constexpr int kQBytes = S::kKBoxes * kQBoxBytes;
    static constexpr int kNP = PSplit<NG, S>::kNP;            // P^T columns (hi and lo halves when split)
    static constexpr int kPBytes = kPage * kNP * 2;           // P^T of one page, bf16
    // P^T of a page is written over the page's own RoPE box (box 8): only
    // GEMM1 reads that box, S^T is complete before the softmax writes P^T, and
    // the stage is refilled only after the page's GEMM2 has read P^T.  So P^T
    // is double-buffered with the stages at no cost in shared memory.
    static constexpr int kPInStage = S::kRopeBox * kBoxBytes;
    static_assert(kPBytes <= kBoxBytes, "P^T fits the RoPE box");
    static constexpr int kKvOff = 0;
    static constexpr int kQOff = kKvOff + kStages * kStageBytes;
    // 64-column groups: Q^T takes 72 KB, so the epilogue stores straight from
    // registers (no staging tile).
    // output rows (query columns) per staging pass; column-grouped softmax
    // warps store from registers instead
    static constexpr int kOutRows = FwdWarps<NG, S>::kColGroups > 1 ? 0 : 16;
    static constexpr int kOutOff = kQOff + kQBytes;           // staging: [16][d_v] fp32 (or bf16)
    static constexpr int kOutBytes = kOutRows * S::kDv * 4;
    // float [2][NG][4]: page maxima of the 4 lane quadrants, double-buffered
    // by page; the epilogue's row sums use the buffer of the item's last page.
    static constexpr int kRedOff = kOutOff + kOutBytes;
    static constexpr int kSumQOff = kRedOff + 2 * NG * 4 * 4;  // float [NG][4]: sums of the bf16 P
    static constexpr int kVoteOff = kSumQOff + NG * 4 * 4;     // uint32 [2][8]: per-warp growth votes
    static constexpr int kBarOff = kVoteOff + 2 * 8 * 4;
    static constexpr int kNumBars = 32;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem base, abort flag
    static constexpr int kPlanMetaOff = kMiscOff + 16;         // this CTA's plan row + 4 words, when built in the kernel
    static constexpr int kBytes = kPlanMetaOff + (kMetaWords + 8) * 4;
    // largest plan (request-groups) the kernel builds itself: prefix + scan state in one stage
    static constexpr int kInlinePlanMaxBG = kStageBytes / 4 - 48;  // prefix (BG + 1) + 32 warp totals
    // Slack to align the base to 1 KB where it fits; without it the kernel
    // checks that the dynamic shared memory base is 1 KB aligned.
    static constexpr int kAlignSlack = kBytes + 1024 <= 227 * 1024 ? 1024 : 0;
    static constexpr int kAlloc = kBytes + kAlignSlack;
    // TMEM columns: S^T buffer i, chain c at kSCol + (i*G1<NG>::kIssuers + c)*NG;
    // O^T d_v chunk c at kOCol + c*kNP (hi half, then the lo half when split).
    static constexpr int kSCol = 0;
    static constexpr int kOCol = 2 * G1<NG>::kIssuers * NG;
    static constexpr int kTmemUsed = kOCol + S::kVChunks * kNP;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
    static_assert(kTmemUsed <= 512, "TMEM budget");
    static_assert(kQOff % 1024 == 0 && kStageBytes % 1024 == 0 && kPInStage % 1024 == 0,
                  "swizzle atoms need 1 KB alignment");
    static_assert(kBytes <= 227 * 1024, "shared memory budget");
    static_assert(kStages >= 2 && kStages <= kMaxStages, "stage count");
    static_assert(!PSplit<NG, S>::kOn || kOutRows > 0, "split P is summed by the staged epilogue");
};

enum Bar {
    kQFull = 0, kQEmpty,
    kSFull0, kSFull1, kSEmpty0, kSEmpty1, kPFull0, kPFull1, kPEmpty0, kPEmpty1,
    kOEmpty, kMmaDone, kRedFull0, kRedFull1, kSumFull, kMmaDone2, kOutStaged, kOutFree, kMaxFull,
    kKvFull0,                             // kMaxStages "page landed" barriers
    kKvEmpty0 = kKvFull0 + kMaxStages,    // kMaxStages "stage free" barriers
    kBarCount = kKvEmpty0 + kMaxStages
};
static_assert(kBarCount <= FwdSmem<16>::kNumBars, "barrier slots");

// ------------------------------------------------------------------ waits
struct Ctl {
    volatile int* abort_flag;
    int32_t* status;
};

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const Ctl& c) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*c.abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *c.abort_flag = 1;
            atomicOr(c.status, MLA_STATUS_TIMEOUT);
            return false;
        }
    }
}

// All 32 lanes wait; the outcome is made warp-uniform so that the warp keeps
// executing .sync.aligned instructions together.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const Ctl& c) {
    const bool ok = wait_bounded(bar, parity, c);
    return __all_sync(kFullMask, ok);
}

// Teardown wait: ignores the abort flag, bounded by time only.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// ------------------------------------------------------------------ work walk
struct Item {
    int bg, b, g, p0, p1, P, L, slot;
    bool unsplit;
};

struct WorkIter {
    int bg, begin_bg, begin_page, end_bg, end_page;
    int range, group;  // plan range of this CTA; its head group when ranges are shared

    // meta: this CTA's row of the plan, in the schedule buffer or (plan built
    // by the kernel itself) in shared memory.
    __device__ void init(const int32_t* meta, const FwdParams& p) {
        begin_bg = meta[kMetaBeginBg];
        begin_page = meta[kMetaBeginPage];
        end_bg = meta[kMetaEndBg];
        end_page = meta[kMetaEndPage];
        bg = begin_bg;
        range = blockIdx.x / p.share;
        group = blockIdx.x - range * p.share;
    }

    __device__ bool next(const FwdParams& p, Item& it) {
        while (bg <= end_bg && bg < p.BG) {
            const int cur = bg++;
            const int b = cur / p.Hg;
            const int L = clamp_seqlen(__ldg(p.seqlens + b), p.max_blocks);
            const int P = pages_of(L);
            const int p0 = (cur == begin_bg) ? begin_page : 0;
            int p1 = (cur == end_bg) ? end_page : P;
            if (p1 > P) p1 = P;
            if (p0 >= p1) continue;
            it.bg = cur;
            it.b = b;
            it.g = p.share > 1 ? group : cur - b * p.Hg;
            it.p0 = p0;
            it.p1 = p1;
            it.P = P;
            it.L = L;
            it.unsplit = (p0 == 0 && p1 == P);
            it.slot = -1;
            if (!it.unsplit) {
                // first item of the range: slot 2k; last item: slot 2k + 1 (see
                // cta_slot), times the groups sharing the range, plus this group
                const int s = cta_slot(range, cur == begin_bg) * p.share + group;
                it.slot = s < p.slots_cap ? s : -1;
            }
            return true;
        }
        return false;
    }
};

// ------------------------------------------------------------------ helpers
// ---- half-column layout of the softmax warps ----
// tcgen05.ld.16x64b reads the 16 lanes of an M=64 accumulator quadrant with
// all 32 threads.  Measured thread mapping on B200: thread t holds lane
// (token) t/4 + 8*(t&1) and the columns of parity (t>>1)&1, one per register
// (column parity + 2*i in register i).  So each thread owns one token and
// half of the NG query columns ("own" columns).
__device__ __forceinline__ int half_token(int lane) { return (lane >> 2) + 8 * (lane & 1); }
__device__ __forceinline__ int half_parity(int lane) { return (lane >> 1) & 1; }

__host__ __device__ constexpr int half_off(int step) { return step == 0 ? 16 : step == 1 ? 8 : step == 2 ? 4 : 1; }

// Transpose-reduce over the 16 threads that share a column parity (lane bits
// 4, 3, 2 and 0; bit 1 is the parity).  Each transposing step keeps half of
// the thread's W columns and folds in its partner's copy of them; when one
// column is left the remaining partner bits are reduced plainly.
template <int W, int S, bool kMax>
struct HalfReduce {
    __device__ __forceinline__ static float run(float* v, int lane) {
        constexpr int OFF = half_off(S);
        constexpr int H = W / 2;
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const float send = upper ? v[i] : v[i + H];
            const float keep = upper ? v[i + H] : v[i];
            const float got = __shfl_xor_sync(kFullMask, send, OFF);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
        return HalfReduce<H, S + 1, kMax>::run(v, lane);
    }
};
template <int S, bool kMax>
struct HalfReduce<1, S, kMax> {
    __device__ __forceinline__ static float run(float* v, int) {
        float x = v[0];
#pragma unroll
        for (int s = S; s < 4; ++s) {
            const float got = __shfl_xor_sync(kFullMask, x, half_off(s));
            x = kMax ? fmaxf(x, got) : x + got;
        }
        return x;
    }
};
// Own-column index i (column = parity + 2*i) the thread holds after HalfReduce,
// and whether it is the one thread of its pair that writes the result.
template <int NG>
__device__ __forceinline__ int half_reduced_index(int lane) {
    return NG == 16 ? ((lane >> 2) & 7) : ((((lane >> 2) & 7) << 1) | (lane & 1));
}
template <int NG>
__device__ __forceinline__ bool half_reduced_writer(int lane) {
    return NG == 32 || (lane & 1) == 0;
}
// P^T (and so O^T) columns are stored parity-major: position q holds query
// column 2q for q < NG/2 and column 2(q - NG/2) + 1 above.
__host__ __device__ constexpr int pos_to_col(int q, int NG) { return q < NG / 2 ? 2 * q : 2 * (q - NG / 2) + 1; }

// 16 lanes x NG/2 own columns of one accumulator (16x64b.x8 or .x16).
template <int NG>
__device__ __forceinline__ void tmem_load_half(uint32_t taddr, float (&v)[NG / 2]) {
    uint32_t r[NG / 2];
    if constexpr (NG == 16) {
        asm volatile("tcgen05.ld.sync.aligned.16x64b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                       "=r"(r[7])
                     : "r"(taddr));
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.16x64b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
              "=r"(r[15])
            : "r"(taddr));
    }
#pragma unroll
    for (int i = 0; i < NG / 2; ++i) v[i] = __uint_as_float(r[i]);
}

template <int NG>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float (&v)[NG]) {
#pragma unroll
    for (int c = 0; c < NG; c += 16) {
        float t[16];
        tmem_ld_x16(taddr + c, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c + i] = t[i];
    }
}
template <int NG>
__device__ __forceinline__ void tmem_store_cols(uint32_t taddr, const float (&v)[NG]) {
#pragma unroll
    for (int c = 0; c < NG; c += 16) {
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) t[i] = v[c + i];
        tmem_st_x16(taddr + c, t);
    }
}

// ------------------------------------------------------------------ roles
// L2 policy of the page loads: pages that other CTAs read too (the head
// groups of a plan row) stay normal, the rest are evicted first.  (Marking the
// pages of shared GQA ranges normal too measured no better: 0.827 against
// 0.844 of the copy bandwidth.)
__device__ __forceinline__ uint64_t page_policy(const FwdParams& p) {
    return p.Hg > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
}

// Page j of item into stage st: its block-table entry, then the stage's boxes
// on the stage's "landed" barrier.
template <int NG, class S>
__device__ __forceinline__ void issue_page(const CUtensorMap* kv_map, const FwdParams& p, const Item& item, int j,
                                           int st, uint8_t* smem, uint64_t policy) {
    using L = FwdSmem<NG, S>;
    const int32_t* bt = p.block_table + (size_t)item.b * p.max_blocks;
    int phys = __ldg(bt + j);
    if ((unsigned)phys >= (unsigned)p.num_blocks) {
        atomicOr(p.status, MLA_STATUS_BAD_BLOCK_TABLE);
        phys = 0;
    }
    const uint32_t full = smem_addr(smem + L::kBarOff) + 8 * (kKvFull0 + st);
    mbar_arrive_expect_tx(full, L::kStageBytes);
    const uint32_t dst = smem_addr(smem + L::kKvOff) + st * L::kStageBytes;
#pragma unroll
    for (int c = 0; c < L::kBoxes; ++c)
        tma_load_3d_hint(dst + c * L::kBoxBytes, kv_map, full, S::col(c, item.g, p.kv_groups), 0, phys, policy);
}

// first_page_issued: the kernel already issued the first page of the first
// item into stage 0, before its wait on the previous grid.
template <int NG, class S>
__device__ void run_producer(const CUtensorMap* kv_map, const CUtensorMap* q_map,
                             const FwdParams& p, const int32_t* meta,
                             uint8_t* smem, const Ctl& ctl, bool first_page_issued) {
    using L = FwdSmem<NG, S>;
    const uint32_t q_s = smem_addr(smem + L::kQOff);
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    const uint64_t policy = page_policy(p);
    WorkIter it;
    it.init(meta, p);
    Item item;
    uint32_t kv_it = 0, q_it = 0;
    uint32_t issued[kMaxStages] = {};  // pages loaded per stage (for the abort drain)
    bool stall = p.test_stall != 0;
    bool ok = true;
    MLA_TRACE_DECL(0);
    while (ok && it.next(p, item)) {
        MLA_TRACE_EV(kTrItem);
        ok = wait_bounded(bar0 + 8 * kQEmpty, (q_it & 1) ^ 1, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar0 + 8 * kQFull, L::kQBytes);
        const int run_rows = S::kOneRun ? NG : p.run_rows;
        const int run_stride = S::kOneRun ? 0 : p.run_stride;
#pragma unroll 1
        for (int r = 0; r * run_rows < NG; ++r) {  // runs of query rows (one for MLA groups)
            const int row0 = item.b * p.N + r * run_stride + item.g * run_rows;
#pragma unroll 1
            for (int c = 0; c < S::kKBoxes; ++c)
                tma_load_2d(q_s + c * L::kQBoxBytes + r * run_rows * 128, q_map, bar0 + 8 * kQFull,
                            c * L::kBoxCols, row0);
        }
        ++q_it;
        const int32_t* bt = p.block_table + (size_t)item.b * p.max_blocks;
        const bool prefetch = S::kPrefetchL2 && kPrefetchPages > 0 && item.p1 - item.p0 >= kPrefetchMinPages;
        if (prefetch)
            for (int j = item.p0; j < item.p1 && j < item.p0 + kPrefetchPages; ++j) {
                const int ph = __ldg(bt + j);
                if ((unsigned)ph < (unsigned)p.num_blocks)
                    prefetch_l2_bulk(p.kv + (size_t)ph * L::kStageBytes, L::kStageBytes);
            }
        for (int j = item.p0; j < item.p1; ++j) {
            if (prefetch && j + kPrefetchPages < item.p1) {
                const int ph = __ldg(bt + j + kPrefetchPages);
                if ((unsigned)ph < (unsigned)p.num_blocks)
                    prefetch_l2_bulk(p.kv + (size_t)ph * L::kStageBytes, L::kStageBytes);
            }
            const int st = kv_it % L::kStages;
            ok = wait_bounded(bar0 + 8 * (kKvEmpty0 + st), ((kv_it / L::kStages) & 1) ^ 1, ctl);
            if (!ok) break;
            if (stall) {  // test hook: this page is never loaded, so its GEMM1 wait runs out
                stall = false;
                ++kv_it;
                continue;
            }
            MLA_TRACE_EV(kTrProdIssue);
            if (first_page_issued)  // (kv_it == 0: stage 0)
                first_page_issued = false;
            else
                issue_page<NG, S>(kv_map, p, item, j, st, smem, policy);
#pragma unroll
            for (int k = 0; k < L::kStages; ++k) issued[k] += st == k;
            ++kv_it;
        }
    }
    if (!ok) {
        // Let the copies already issued land before the CTA exits.
#pragma unroll
        for (int k = 0; k < L::kStages; ++k)
            if (issued[k] > 0) wait_drain(bar0 + 8 * (kKvFull0 + k), (issued[k] - 1) & 1);
        if (q_it > 0) wait_drain(bar0 + 8 * kQFull, (q_it - 1) & 1);
    }
}

// GEMM1 issuer: S^T[64 x NG] = K[64 x 576] . Q^T as soon as a page has landed
// and its S^T buffer is free.  K-major A (64 token rows of 128 B per box,
// 8-row groups 1 KB apart) and K-major B (Q^T rows); the 16-wide k-step
// advances 32 B inside the 128-byte swizzle atom.  k-step i accumulates into
// the accumulator of its issuer.
template <int NG, class S>
__device__ void run_gemm1(const FwdParams& p, const int32_t* meta,
                          uint8_t* smem, uint32_t tmem, const Ctl& ctl, int issuer) {
    using L = FwdSmem<NG, S>;
    constexpr uint32_t kIdescS = idesc_bf16_f32(64, NG, 0, 0);
    const uint32_t kv_s = smem_addr(smem + L::kKvOff);
    const uint32_t q_s = smem_addr(smem + L::kQOff);
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    WorkIter it;
    it.init(meta, p);
    Item item;
    uint32_t s_it = 0, q_it = 0;
    bool ok = true;
#ifdef MLA_TRACE
    Tracer tracer_(issuer == 0 ? 1 : 0, issuer == 0);
#endif
    // Descriptors differ only in their start address (bits 0..13, in 16-byte
    // units): build them once and add offsets.
    const uint64_t a_desc0 = smem_desc(kv_s, 16, 1024, kSwizzle128);
    const uint64_t b_desc0 = smem_desc(q_s, 16, 1024, kSwizzle128);
    while (ok && it.next(p, item)) {
        ok = wait_bounded(bar0 + 8 * kQFull, q_it & 1, ctl);
        if (!ok) break;
        for (int j = item.p0; j < item.p1; ++j) {
            const int st = s_it % L::kStages;  // KV stage of the page
            const int sb = s_it & 1;            // S^T buffer
            ok = wait_bounded(bar0 + 8 * (kKvFull0 + st), (s_it / L::kStages) & 1, ctl);
            if (!ok) break;
            MLA_TRACE_EV(kTrMmaKvFull);
            ok = wait_bounded(bar0 + 8 * (kSEmpty0 + sb), ((s_it >> 1) & 1) ^ 1, ctl);
            if (!ok) break;
            tc_fence_after();
            // This issuer's accumulator; it takes boxes issuer, issuer + 2, ...
            const uint32_t d = tmem + L::kSCol + (sb * G1<NG>::kIssuers + issuer) * NG;
            const uint64_t a_st = a_desc0 + ((st * L::kStageBytes) >> 4);
            bool first = true;
#pragma unroll 1
            for (int c = issuer; c < S::kKBoxes; c += G1<NG>::kIssuers) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t a = a_st + ((S::k_box(c) * L::kBoxBytes + k * 32) >> 4);
                    const uint64_t b = b_desc0 + ((c * L::kQBoxBytes + k * 32) >> 4);
                    umma_f16(d, a, b, kIdescS, first ? 0u : 1u);
                    first = false;
                }
            }
            umma_commit(bar0 + 8 * (kSFull0 + sb));
            MLA_TRACE_EV(kTrMmaG1Issued);
            if (j == item.p1 - 1) umma_commit(bar0 + 8 * kQEmpty);
            ++s_it;
        }
        ++q_it;
    }
    // Drain before TMEM is released, on the normal and the abort path alike:
    // every GEMM1 issuer commits (a commit with no MMA outstanding arrives at
    // once), so the barrier completes as soon as all their MMAs are done.
    umma_commit(bar0 + 8 * kMmaDone);
    wait_drain(bar0 + 8 * kMmaDone, 0);
}

// GEMM2 issuer: O^T[512 x NG] += V^T[512 x 64] . P^T as soon as P^T is in
// shared memory.  V^T is the stage's first 8 boxes read MN-major (d_v
// contiguous within a token row; 64 d_v per swizzle atom, next atom = next box
// 8 KB on, 8-token groups 1 KB apart); P^T is MN-major with NG columns per
// token row.  k-outer order keeps consecutive MMAs on different accumulators.
template <int NG, class S>
__device__ void run_gemm2(const FwdParams& p, const int32_t* meta,
                          uint8_t* smem, uint32_t tmem, const Ctl& ctl, int issuer) {
    constexpr int kIssuers = FwdWarps<NG, S>::kG2Issuers;
    constexpr int kChunksPer = S::kVChunks / kIssuers;  // d_v chunks of 128 per issuer
    using L = FwdSmem<NG, S>;
    constexpr int NP = L::kNP;
    constexpr uint32_t kIdescO = idesc_bf16_f32(128, NP, 1, 1);
    constexpr uint32_t kPSwizzle = NP == 16 ? kSwizzle32 : NP == 32 ? kSwizzle64 : kSwizzle128;
    const uint32_t kv_s = smem_addr(smem + L::kKvOff);
    const uint32_t p_s = kv_s + L::kPInStage;  // P^T of stage 0
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    WorkIter it;
    it.init(meta, p);
    Item item;
    uint32_t s_it = 0, item_it = 0;
    bool ok = true;
#ifdef MLA_TRACE
    Tracer tracer_(issuer == 0 ? 2 : 0, issuer == 0);
#endif
    const uint64_t a_desc0 = smem_desc(kv_s, L::kBoxBytes, 1024, kSwizzle128);
    const uint64_t b_desc0 = smem_desc(p_s, L::kPBytes, 8 * NP * 2, kPSwizzle);
    while (ok && it.next(p, item)) {
        for (int j = item.p0; j < item.p1; ++j) {
            const int st = s_it % L::kStages;  // KV stage of the page (holds its P^T)
            const int pb = s_it & 1;            // P^T handoff barriers
            const bool first = (j == item.p0);
            ok = wait_bounded(bar0 + 8 * (kPFull0 + pb), (s_it >> 1) & 1, ctl);
            if (!ok) break;
            if (first) {
                ok = wait_bounded(bar0 + 8 * kOEmpty, (item_it & 1) ^ 1, ctl);
                if (!ok) break;
            }
            MLA_TRACE_EV(kTrMmaPFull);
            tc_fence_after();
            const uint64_t a_st = a_desc0 + ((st * L::kStageBytes) >> 4);
            const uint64_t b_st = b_desc0 + ((st * L::kStageBytes) >> 4);
#pragma unroll
            for (int k = 0; k < kPage / 16; ++k) {
                const uint64_t b = b_st + ((k * 16 * NP * 2) >> 4);
#pragma unroll
                for (int cc = 0; cc < kChunksPer; ++cc) {
                    const int ch = issuer * kChunksPer + cc;
                    const uint64_t a = a_st + ((S::v_box(ch) * L::kBoxBytes + k * 2048) >> 4);
                    umma_f16(tmem + L::kOCol + ch * NP, a, b, kIdescO, (first && k == 0) ? 0u : 1u);
                }
            }
            umma_commit(bar0 + 8 * (kKvEmpty0 + st));
            umma_commit(bar0 + 8 * (kPEmpty0 + pb));
            MLA_TRACE_EV(kTrMmaG2Issued);
            ++s_it;
        }
        if (!ok) break;
        ++item_it;
    }
    // drained as GEMM1's issuers are
    umma_commit(bar0 + 8 * kMmaDone2);
    wait_drain(bar0 + 8 * kMmaDone2, 0);
}

template <int NG, class S>
__device__ void run_softmax(const FwdParams& p, const int32_t* meta,
                            uint8_t* smem, uint32_t tmem, const Ctl& ctl) {
    using L = FwdSmem<NG, S>;
    using Wp = FwdWarps<NG, S>;
    constexpr bool kSplit = PSplit<NG, S>::kOn;           // P^T = [hi | lo] (2 x NG columns)
    constexpr int NP = L::kNP;
    constexpr int NGW = Wp::kGroupCols;                   // query columns of this warp's group
    constexpr int W = NGW / 2;                            // own columns per thread
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wq = warp & 3;                              // TMEM lane quadrant this warp may access
    const int cg = (warp - Wp::kFirstSoftmax) >> 2;       // column group: columns [cg*NGW, cg*NGW + NGW)
    const int c0g = cg * NGW;
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const int gt = threadIdx.x - 32 * Wp::kFirstSoftmax;  // 0 .. kSoftmaxThreads-1
    const int gtg = gt & 127;                             // 0..127 within the column group
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);
    uint32_t* vote = reinterpret_cast<uint32_t*>(smem + L::kVoteOff);  // [2][softmax warps] growth flags
    constexpr int kSoftmaxWarps = Wp::kSoftmaxThreads / 32;
    const int sw = (threadIdx.x >> 5) - Wp::kFirstSoftmax;  // softmax warp index
    uint8_t* pbuf = smem + L::kKvOff + L::kPInStage;     // P^T of stage 0
    float* stage_f32 = reinterpret_cast<float*>(smem + L::kOutOff);
    __nv_bfloat16* stage_bf16 = reinterpret_cast<__nv_bfloat16*>(smem + L::kOutOff);
    // Token row of this thread in the page (M=64 accumulator: token m sits in
    // TMEM lane 32*(m/16) + m%16) and its column parity.
    const int par = half_parity(lane);
    const int row = 16 * wq + half_token(lane);
    const int red_i = half_reduced_index<NGW>(lane);
    const int red_col = c0g + par + 2 * red_i;            // column whose reduction this thread holds
    const bool red_w = half_reduced_writer<NGW>(lane);
    // P^T row: NP bf16 positions; the group owns positions c0g .. c0g+NGW-1,
    // parity-major inside (own columns of parity par at c0g + par*W ..); with
    // a split P the lo terms follow at NG + the same positions.
    constexpr int kChunks = NP * 2 / 16;                  // 16-byte chunks per P^T row
    constexpr int kMyChunks = NGW / 16;                   // chunks of one thread (per term)
    constexpr int kLoChunk = NG * 2 / 16;                 // chunk offset of the lo terms
    const int chunk0 = cg * (NGW / 8) + par * kMyChunks;
    const int swz = ((row * NP * 2) >> 7) & (kChunks - 1);
#ifdef MLA_TRACE
    Tracer tracer_(3);
    const bool tr = (gt == 0);
#define MLA_TRACE_SM(tag) \
    if (tr) tracer_.ev(tag)
#else
#define MLA_TRACE_SM(tag)
#endif

    WorkIter it;
    it.init(meta, p);
    Item item;
    uint32_t s_it = 0, item_it = 0, out_it = 0, max_it = 0;
    bool ok = true;
    while (ok && it.next(p, item)) {
        int lvis[W];                                      // visible length of each own column
#pragma unroll
        for (int i = 0; i < W; ++i) {
            const int gc = group_col<NG, S>(p, item.g, c0g + par + 2 * i);
            int v = 0;
            if (gc < p.N) {
                const int sq = gc / p.heads;
                v = (p.causal && p.s_q > 1) ? item.L - p.s_q + 1 + sq : item.L;
            }
            lvis[i] = v;
        }
        float m_all[NGW];                                 // running max (log2 units), every group column
        // Running row sums, own columns, own token: l_own of the fp32 P (for the
        // LSE) and lq_own of P as rounded to bf16 for GEMM2 (to normalise O, so
        // that numerator and denominator carry the same weights; a dominant
        // token's rounding then cancels in O).
        float l_own[W], lq_own[W];
#pragma unroll
        for (int n = 0; n < NGW; ++n) m_all[n] = -INFINITY;
#pragma unroll
        for (int i = 0; i < W; ++i) l_own[i] = lq_own[i] = 0.f;

        for (int j = item.p0; j < item.p1; ++j) {
            const int sb = s_it & 1;
            ok = wait_warp(bar0 + 8 * (kSFull0 + sb), (s_it >> 1) & 1, ctl);
            if (!ok) break;
            MLA_TRACE_SM(kTrSmSFull);
            tc_fence_after();
            float x[W];
            {
                const uint32_t sbase = tmem + lane_base + L::kSCol + sb * G1<NG>::kIssuers * NG + c0g;
                tmem_load_half<NGW>(sbase, x);
#pragma unroll
                for (int c = 1; c < G1<NG>::kIssuers; ++c) {
                    float y[W];
                    tmem_load_half<NGW>(sbase + c * NG, y);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < W; ++i) x[i] += y[i];
                }
                tmem_ld_wait();
            }
            tc_fence_before();
            mbar_arrive(bar0 + 8 * (kSEmpty0 + sb));

            const int t = j * kPage + row;
#pragma unroll
            for (int i = 0; i < W; ++i) x[i] = (t < lvis[i]) ? x[i] * p.scale_log2 : -INFINITY;

            // Does any column's max grow by more than 2^8 on this page?
            // 16/32-column groups: the warps post exact page maxima per column
            // and meet once through shared memory.  64-column groups: each
            // warp first posts only a one-word vote (any own value above the
            // running max + 2^8); the maxima follow in a second round only if
            // some warp voted.  That halves the common page's softmax work at
            // 64 columns (B200, bs32 x s_q 2 x 128 heads: 626 -> 593 us per
            // launch) but gains nothing at 16 and loses at 32 columns.
            float m_own[W];
#pragma unroll
            for (int i = 0; i < W; ++i) m_own[i] = par ? m_all[2 * i + 1] : m_all[2 * i];
            float* rb = red + (s_it & 1) * NG * 4;
            if constexpr (NG != 64) {
                float xr[W];
#pragma unroll
                for (int i = 0; i < W; ++i) xr[i] = x[i];
                const float wmax = HalfReduce<W, 0, true>::run(xr, lane);
                if (red_w) rb[red_col * 4 + wq] = wmax;
            } else {
                bool grow_l = false;
#pragma unroll
                for (int i = 0; i < W; ++i) grow_l |= x[i] > m_own[i] + kRescaleLog2;
                const uint32_t grow_w = __any_sync(kFullMask, grow_l) ? 1u : 0u;
                if (lane == 0) vote[(s_it & 1) * kSoftmaxWarps + sw] = grow_w;
            }
            MLA_TRACE_SM(kTrSmMaxDone);
            mbar_arrive(bar0 + 8 * (kRedFull0 + (s_it & 1)));

            // Speculative P with the running max, stored before the exchange
            // completes; it stands unless some column's max grew by > 2^8.
            float e[W];
#pragma unroll
            for (int i = 0; i < W; ++i) e[i] = (x[i] == -INFINITY) ? 0.f : ex2_approx(x[i] - m_own[i]);
            const int pb = s_it & 1;                      // P^T handoff barriers
            uint8_t* rowp = pbuf + (s_it % L::kStages) * L::kStageBytes + row * (NP * 2);  // the page's stage
            auto store_p = [&](const float (&ev)[W]) {
                uint32_t packed[W / 2];
                uint32_t packed_lo[kSplit ? W / 2 : 1];
#pragma unroll
                for (int i = 0; i < W; i += 2) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(ev[i], ev[i + 1]);
                    packed[i / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                    if constexpr (kSplit) {
                        // P - hi is exact in fp32 (hi is P rounded to 8 bits), so
                        // lo carries the next 8 bits of P.
                        const float2 hf = __bfloat1622float2(h2);
                        const __nv_bfloat162 l2 = __floats2bfloat162_rn(ev[i] - hf.x, ev[i + 1] - hf.y);
                        packed_lo[i / 2] = *reinterpret_cast<const uint32_t*>(&l2);
                    }
                }
#pragma unroll
                for (int c = 0; c < kMyChunks; ++c) {
                    const int chunk = chunk0 + c;
                    *reinterpret_cast<uint4*>(rowp + ((chunk ^ swz) * 16)) =
                        make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
                }
                if constexpr (kSplit) {
#pragma unroll
                    for (int c = 0; c < kMyChunks; ++c) {
                        const int chunk = kLoChunk + chunk0 + c;
                        *reinterpret_cast<uint4*>(rowp + ((chunk ^ swz) * 16)) = make_uint4(
                            packed_lo[4 * c], packed_lo[4 * c + 1], packed_lo[4 * c + 2], packed_lo[4 * c + 3]);
                    }
                }
            };
            ok = wait_warp(bar0 + 8 * (kPEmpty0 + pb), ((s_it >> 1) & 1) ^ 1, ctl);
            if (!ok) break;
            store_p(e);
            fence_proxy_async_smem();
            MLA_TRACE_SM(kTrSmPStored);

            ok = wait_warp(bar0 + 8 * (kRedFull0 + (s_it & 1)), (s_it >> 1) & 1, ctl);
            if (!ok) break;
            MLA_TRACE_SM(kTrSmXchg);
            bool grow_any = false;
            if constexpr (NG != 64) {
                // The warp's threads cover every column of the group and the
                // group's four warps read the same maxima, so this decision is
                // uniform across the group.
                bool grow = false;
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    const float4 r4 = *reinterpret_cast<const float4*>(rb + (c0g + par + 2 * i) * 4);
                    const float pmax = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                    grow |= pmax > m_own[i] + kRescaleLog2;
                }
                grow_any = __any_sync(kFullMask, grow);
            } else {
                // Every softmax warp reads every vote, so the decision is the
                // same for all of them (the second round's barrier needs all).
                uint32_t votes = 0;
#pragma unroll
                for (int w = 0; w < kSoftmaxWarps; w += 4) {
                    const uint4 f4 = *reinterpret_cast<const uint4*>(vote + (s_it & 1) * kSoftmaxWarps + w);
                    votes |= f4.x | f4.y | f4.z | f4.w;
                }
                grow_any = votes != 0;
                if (grow_any) {
                    float xr[W];
#pragma unroll
                    for (int i = 0; i < W; ++i) xr[i] = x[i];
                    const float wmax = HalfReduce<W, 0, true>::run(xr, lane);
                    if (red_w) rb[red_col * 4 + wq] = wmax;
                    mbar_arrive(bar0 + 8 * kMaxFull);
                    ok = wait_warp(bar0 + 8 * kMaxFull, max_it & 1, ctl);
                    ++max_it;
                    if (!ok) break;
                }
            }
            if (!grow_any) {
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    l_own[i] += e[i];
                    if constexpr (!kSplit) lq_own[i] += bf16_round(e[i]);
                }
            } else {
                // Slow path: the group's exact page maxima are in rb; move the
                // reference max of the grown columns and rescale.
                float alpha[NGW];
                bool scale_any = false;
#pragma unroll
                for (int n = 0; n < NGW; ++n) {
                    const float4 r4 = *reinterpret_cast<const float4*>(rb + (c0g + n) * 4);
                    const float pmax = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                    const float mnew = fmaxf(m_all[n], pmax);
                    if (mnew > m_all[n] + kRescaleLog2) {
                        alpha[n] = ex2_approx(m_all[n] - mnew);
                        m_all[n] = mnew;
                        scale_any = true;
                    } else {
                        alpha[n] = 1.f;
                    }
                }
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    const float a = par ? alpha[2 * i + 1] : alpha[2 * i];
                    const float m = par ? m_all[2 * i + 1] : m_all[2 * i];
                    e[i] = (x[i] == -INFINITY) ? 0.f : ex2_approx(x[i] - m);
                    l_own[i] = l_own[i] * a + e[i];
                    if constexpr (!kSplit) lq_own[i] = lq_own[i] * a + bf16_round(e[i]);
                }
                // scale_any is the same for the group's four warps (same maxima).
                if (scale_any) {
                    store_p(e);
                    fence_proxy_async_smem();
                }
                if (scale_any && j > item.p0) {
                    // O^T already holds earlier pages: wait for the previous
                    // GEMM2, then scale each of the group's columns (positions)
                    // in place.
                    const uint32_t prev = s_it - 1;
                    ok = wait_warp(bar0 + 8 * (kPEmpty0 + (prev & 1)), (prev >> 1) & 1, ctl);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < S::kVChunks * (kSplit ? 2 : 1); ++ch) {  // (chunk, term)
#pragma unroll
                        for (int h = 0; h < NGW; h += 16) {  // 16 positions at a time
                            float o[16];
                            const uint32_t ta = tmem + lane_base + L::kOCol + ch * NG + c0g + h;
                            tmem_ld_x16(ta, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 16; ++q) o[q] *= alpha[pos_to_col(h + q, NGW)];
                            tmem_st_x16(ta, o);
                        }
                    }
                    tmem_st_wait();
                }
            }
            tc_fence_before();
            MLA_TRACE_SM(kTrSmPDone);
            mbar_arrive(bar0 + 8 * (kPFull0 + pb));
            ++s_it;
        }
        if (!ok) break;

        // ---- epilogue: wait for the last GEMM2, reduce l over the tokens ----
        const uint32_t last = s_it - 1;
        ok = wait_warp(bar0 + 8 * (kPEmpty0 + (last & 1)), (last >> 1) & 1, ctl);
        if (!ok) break;
        MLA_TRACE_SM(kTrSmEpi0);
        tc_fence_after();
        // Row sums go through the page-maxima buffer of the last page: every
        // thread has read it (the last GEMM2 waited for all of them), and the
        // next write to it is two pages on, after all threads have left this
        // epilogue.
        float* sred = red + (last & 1) * NG * 4;
        float* sredq = reinterpret_cast<float*>(smem + L::kSumQOff);
        {
            float lr[W];
#pragma unroll
            for (int i = 0; i < W; ++i) lr[i] = l_own[i];
            const float wsum = HalfReduce<W, 0, false>::run(lr, lane);
            if (red_w) sred[red_col * 4 + wq] = wsum;
#pragma unroll
            for (int i = 0; i < W; ++i) lr[i] = lq_own[i];
            const float wsumq = HalfReduce<W, 0, false>::run(lr, lane);
            if (red_w) sredq[red_col * 4 + wq] = wsumq;
        }
        mbar_arrive(bar0 + 8 * kSumFull);
        ok = wait_warp(bar0 + 8 * kSumFull, item_it & 1, ctl);
        if (!ok) break;
        MLA_TRACE_SM(kTrSmEpiSum);
        // l per group column; one thread per column writes its LSE.  The
        // column of thread gtg is picked by a select chain rather than by
        // unrolling the whole LSE computation per column: this code runs once
        // per item, so its size (instruction fetch) matters more than its
        // instruction count.
        float inv[NGW], m_gt = -INFINITY, l_gt = 0.f;
#pragma unroll
        for (int n = 0; n < NGW; ++n) {
            const float4 s4 = *reinterpret_cast<const float4*>(sred + (c0g + n) * 4);
            const float4 q4 = *reinterpret_cast<const float4*>(sredq + (c0g + n) * 4);
            const float ls = (s4.x + s4.y) + (s4.z + s4.w);
            const float lq = (q4.x + q4.y) + (q4.z + q4.w);
            // A split P sums to the fp32 P within 2^-17; one bf16 term is
            // normalised by its own sum, so that a dominant token's rounding
            // cancels between numerator and denominator.
            const float lden = kSplit ? ls : lq;
            inv[n] = lden > 0.f ? rcp_approx(lden) : 0.f;
            m_gt = gtg == n ? m_all[n] : m_gt;
            l_gt = gtg == n ? ls : l_gt;
        }
        {
            const int gc = group_col<NG, S>(p, item.g, c0g + gtg);
            if (gtg < NGW && gc < p.N) {
                const float lse = l_gt > 0.f ? (m_gt + log2f(l_gt)) * kLn2 : -INFINITY;
                if (item.unsplit) {
                    const int sq = gc / p.heads;
                    const int head = gc - sq * p.heads;
                    p.lse[((size_t)item.b * p.heads + head) * p.s_q + sq] = lse;
                } else if (item.slot >= 0) {
                    p.lpart[(size_t)item.slot * NG + c0g + gtg] = lse;
                }
            }
        }
        MLA_TRACE_SM(kTrSmEpiLse);
        if constexpr (L::kOutRows > 0) {
            // O = O^T / l, transposed back through a shared-memory staging tile of
            // 16 query columns x 512 (bf16 final rows or fp32 partial rows), then
            // written by one bulk copy: a request's output rows, and a partial
            // slot, are contiguous in global memory.
#pragma unroll
            for (int ps = 0; ps < NG / L::kOutRows; ++ps) {
                ok = wait_warp(bar0 + 8 * kOutFree, (out_it & 1) ^ 1, ctl);
                if (!ok) break;
                const bool f32 = !item.unsplit || p.out_f32;  // staged as fp32 rows
#pragma unroll 1
                for (int ch = 0; ch < S::kVChunks; ++ch) {
                    // positions 8ps.. hold even columns 16ps + 2i, NG/2 + 8ps.. the odd ones
                    // (and the lo terms of a split P the same, NG further on)
                    float ev[8], od[8];
                    const uint32_t ta = tmem + lane_base + L::kOCol + ch * NP;
                    tmem_ld_x8(ta + 8 * ps, ev);
                    tmem_ld_x8(ta + NG / 2 + 8 * ps, od);
                    if constexpr (kSplit) {
                        float ev2[8], od2[8];
                        tmem_ld_x8(ta + NG + 8 * ps, ev2);
                        tmem_ld_x8(ta + NG + NG / 2 + 8 * ps, od2);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            ev[i] += ev2[i];
                            od[i] += od2[i];
                        }
                    } else {
                        tmem_ld_wait();
                    }
                    const int d = ch * 128 + 32 * wq + lane;  // O^T row (lane) = output column d
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float ve = ev[i] * inv[16 * ps + 2 * i];
                        const float vo = od[i] * inv[16 * ps + 2 * i + 1];
                        if (f32) {
                            stage_f32[(2 * i) * S::kDv + d] = ve;
                            stage_f32[(2 * i + 1) * S::kDv + d] = vo;
                        } else {
                            stage_bf16[(2 * i) * S::kDv + d] = __float2bfloat16_rn(ve);
                            stage_bf16[(2 * i + 1) * S::kDv + d] = __float2bfloat16_rn(vo);
                        }
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(bar0 + 8 * kOutStaged);
                if (gt == 0) {
                    ok = wait_bounded(bar0 + 8 * kOutStaged, out_it & 1, ctl);
                    if (ok) {
                        // first query column of the pass; a pass stays within one run
                        const int c0 = group_col<NG, S>(p, item.g, L::kOutRows * ps);
                        if (!item.unsplit) {
                            if (item.slot >= 0)
                                bulk_store_s2g(p.opart + ((size_t)item.slot * NG + L::kOutRows * ps) * S::kDv,
                                               smem_addr(stage_f32), L::kOutRows * S::kDv * 4);
                        } else {
                            int rows = p.N - c0;
                            rows = rows < L::kOutRows ? rows : L::kOutRows;
                            const size_t row0 = (size_t)item.b * p.N + c0;
                            if (rows > 0) {
                                if (p.out_f32)
                                    bulk_store_s2g(static_cast<float*>(p.out) + row0 * S::kDv, smem_addr(stage_f32),
                                                   rows * S::kDv * 4);
                                else
                                    bulk_store_s2g(static_cast<__nv_bfloat16*>(p.out) + row0 * S::kDv,
                                                   smem_addr(stage_bf16), rows * S::kDv * 2);
                            }
                        }
                        bulk_commit();
                        bulk_wait_read_all();
                    }
                    mbar_arrive(bar0 + 8 * kOutFree);
                }
                ++out_it;
            }
            if (!ok) break;
        } else {
            // No staging room: O = O^T / l straight from registers.  For one
            // query column the 32 lanes of a warp hold 32 consecutive d, so
            // each store instruction writes 64 (bf16) or 128 (fp32) contiguous
            // bytes.
            const bool f32 = !item.unsplit;
#pragma unroll 1
            for (int ch = 0; ch < S::kVChunks; ++ch) {
#pragma unroll
              for (int h = 0; h < NGW; h += 16) {  // 16 positions at a time
                float o[16];
                tmem_ld_x16(tmem + lane_base + L::kOCol + ch * NG + c0g + h, o);
                tmem_ld_wait();
                const int d = ch * 128 + 32 * wq + lane;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int n = pos_to_col(h + q, NGW);          // group column of position h + q
                    const float v = o[q] * inv[n];
                    if (f32) {
                        if (item.slot >= 0) p.opart[((size_t)item.slot * NG + c0g + n) * S::kDv + d] = v;
                    } else {
                        const int gc = group_col<NG, S>(p, item.g, c0g + n);
                        const size_t o = ((size_t)item.b * p.N + gc) * S::kDv + d;
                        if (gc < p.N) {
                            if (p.out_f32)
                                static_cast<float*>(p.out)[o] = v;
                            else
                                static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v);
                        }
                    }
                }
              }
            }
        }
        MLA_TRACE_SM(kTrSmEpiOut);
        if (!item.unsplit && item.slot < 0 && gt == 0) atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
        MLA_TRACE_SM(kTrSmEpi1);
        tc_fence_before();
        mbar_arrive(bar0 + 8 * kOEmpty);
        ++item_it;
    }
    if constexpr (L::kOutRows > 0)
        if (gt == 0) bulk_wait_all();  // output copies complete before the CTA exits
}

// Block-wide inclusive scan of one int per thread (blockDim.x a multiple of
// 32, at most 1024); warp_tot holds 32 ints of shared memory.
__device__ __forceinline__ int block_inclusive_scan(int v, int* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFullMask, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    const int r = v + (warp > 0 ? warp_tot[warp - 1] : 0);
    __syncthreads();
    return r;
}

// The split-KV plan built inside the decode kernel from the lengths alone:
// the same plan mla_decode_schedule_kernel writes (schedule.cuh), without its
// launch.  Two parts.  build_plan_in_cta reads only the lengths, so it runs
// before the wait on the previous grid: the unit prefix over request-groups
// goes to `scratch` (BG + 1 words plus 32 of warp totals, in a page stage
// that no copy has targeted yet), this CTA's range to plan_s[0..7], and W, T
// and the bad-length flag to plan_s[10], [11], [9].  publish_plan_in_cta runs
// after the wait (a combine of the previous call may still read the schedule
// buffer before it) and writes the CTA's share of the plan there, for the
// combine kernel and for inspection: its meta row; the rows of the
// request-groups whose first page it holds (CTA 0 takes those with no pages);
// and CTA 0 the header and the prefix.  The header's status word is left
// alone, so faults accumulate until the next mla_decode_get_schedule clears
// it.  Every thread takes part in both; each ends with a block barrier (three
// in all when BG fits one pass of the CTA's threads), the last one before the
// scratch stage is given to the producer.
constexpr int kPlanSlots = kMetaWords, kPlanBad = kMetaWords + 1, kPlanW = kMetaWords + 2,
              kPlanT = kMetaWords + 3;

__device__ void build_plan_in_cta(const FwdParams& p, int32_t* scratch, int32_t* plan_s) {
    const int nthr = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    // With shared ranges every CTA of range k computes the same plan.
    const int k = blockIdx.x / p.share, G = gridDim.x / p.share, BG = p.BG, Hg = p.Hg, mb = p.max_blocks;
    int32_t* prefix = scratch;
    int32_t* warp_tot = scratch + BG + 1;
    if (tid == 0) {
        plan_s[kPlanSlots] = 0;
        plan_s[kPlanBad] = 0;
    }
    // Unit prefix, one pass of nthr request-groups at a time: a warp scan by
    // shuffles, then every thread adds the totals of the warps before it.
    int carry = 0;
    bool any_bad = false;
    for (int base = 0; base < BG; base += nthr) {
        const int bg = base + tid;
        int v = 0;
        if (bg < BG) {
            const int L = __ldg(p.seqlens + bg / Hg);
            any_bad |= !seqlen_in_range(L, mb);
            v = (int)units_of(blocks_of(clamp_seqlen(L, mb), kPageShift));
        }
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFullMask, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        int before = carry, total = carry;
        for (int w = 0; w < nwarps; ++w) {
            const int t = warp_tot[w];
            before += w < warp ? t : 0;
            total += t;
        }
        if (bg < BG) prefix[bg] = before + x - v;
        carry = total;
        if (base + nthr < BG) __syncthreads();  // warp_tot is reused by the next pass
    }
    const int64_t W = carry;
    if (tid == 0) prefix[BG] = (int)W;
    if (any_bad) plan_s[kPlanBad] = 1;
    __syncthreads();
    if (tid == 0) {
        const int64_t T = units_per_cta(W, G);
        cta_meta(prefix, BG, W, T, k, plan_s);
        plan_s[kPlanW] = (int)W;
        plan_s[kPlanT] = (int)T;
    }
    __syncthreads();
}

__device__ void publish_plan_in_cta(const FwdParams& p, int NG, const int32_t* scratch, int32_t* plan_s) {
    const int nthr = blockDim.x, tid = threadIdx.x, lane = tid & 31;
    const int k = blockIdx.x / p.share, G = gridDim.x / p.share, BG = p.BG, Hg = p.Hg;
    const bool writer = blockIdx.x % p.share == 0;  // group 0 of a shared range writes its rows
    const int32_t* prefix = scratch;
    const int64_t T = plan_s[kPlanT];
    if (tid == 0 && writer) {
        int32_t* row = p.plan_out + kHdrWords + (size_t)k * kMetaWords;
        for (int i = 0; i < kMetaWords; ++i) row[i] = plan_s[i];
    }
    int32_t* bginfo = p.plan_out + bg_offset_words(G);
    int my_slots = 0;
    for (int bg = tid; bg < BG; bg += nthr) {
        const int P = pages_in_prefix(prefix, bg);
        const int ns = num_splits_of(prefix, bg, P, T);
        if (ns > 1) my_slots += ns;
        int owner = P > 0 ? first_cta_of(prefix, bg, T) : 0;
        if (owner > G - 1) owner = G - 1;
        if (owner == k && writer) {
            bginfo[kBgWords * bg] = ns > 1 ? first_split_slot(prefix, bg, T) : 0;
            bginfo[kBgWords * bg + 1] = ns;
        }
    }
    if (blockIdx.x == 0) {
        int32_t* pg = p.plan_out + prefix_offset_words(G, BG);
        for (int i = tid; i <= BG; i += nthr) pg[i] = prefix[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_slots += __shfl_xor_sync(kFullMask, my_slots, o);
        if (lane == 0 && my_slots) atomicAdd(plan_s + kPlanSlots, my_slots);
    }
    __syncthreads();
    if (blockIdx.x == 0 && tid == 0) {
        int32_t* h = p.plan_out;
        h[kHdrMagic] = kSchedMagic;
        h[kHdrG] = G;
        h[kHdrBG] = BG;
        h[kHdrHg] = Hg;
        h[kHdrNG] = NG;
        h[kHdrSlots] = plan_s[kPlanSlots];
        h[kHdrT] = (int)T;
        h[kHdrW] = plan_s[kPlanW];
        h[kHdrBatch] = BG / Hg;
        h[kHdrMaxBlocks] = p.max_blocks;
        h[kHdrShift] = kPageShift;
        h[kHdrShareHg] = p.share;
        for (int i = kHdrShareHg + 1; i < kHdrWords; ++i) h[i] = 0;
        if (plan_s[kPlanBad]) atomicOr(p.status, MLA_STATUS_BAD_SEQLEN);
    }
}

// ------------------------------------------------------------------ kernels
template <int NG, class S>
__global__ void __launch_bounds__(FwdWarps<NG, S>::kThreads, 1)
    mla_decode_fwd_kernel(const __grid_constant__ CUtensorMap kv_map,
                          const __grid_constant__ CUtensorMap q_map, const FwdParams p) {
    using L = FwdSmem<NG, S>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    MLA_TRACE_K(0);
    // The grid after this one (the combine) may launch now: it waits for this
    // grid's end before it reads anything of it.
    griddep_launch_dependents();
    const uint32_t bar0 = smem_addr(smem + L::kBarOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    int32_t* meta_s = reinterpret_cast<int32_t*>(smem + L::kPlanMetaOff);
    // A base that could not be realigned (no slack reserved) is reported after
    // the wait below, with nothing set up.
    bool misaligned = false;
    if constexpr (L::kAlignSlack == 0) misaligned = smem != smem_raw;
    // Setup that reads nothing another grid writes (barriers, TMEM) overlaps
    // the end of the grid before this one.
    if (!misaligned) {
        if (threadIdx.x == 0) {
            for (int i = 0; i < kBarCount; ++i) {
                uint32_t count = 1;
                if (i == kSEmpty0 || i == kSEmpty1 || i == kPFull0 || i == kPFull1 || i == kOEmpty ||
                    i == kRedFull0 || i == kRedFull1 || i == kSumFull || i == kOutStaged || i == kMaxFull)
                    count = FwdWarps<NG, S>::kSoftmaxThreads;
                if (i == kSFull0 || i == kSFull1 || i == kQEmpty || i == kMmaDone) count = G1<NG>::kIssuers;
                if ((i >= kKvEmpty0 && i < kKvEmpty0 + kMaxStages) || i == kPEmpty0 || i == kPEmpty1 ||
                    i == kMmaDone2)
                    count = FwdWarps<NG, S>::kG2Issuers;
                mbar_init(bar0 + 8 * i, count);
            }
            *abort_flag = 0;
            fence_mbar_init();
        }
        if (warp == 1) {
            tmem_alloc(smem_addr(tmem_slot), L::kTmemCols);
            tmem_relinquish();
        }
    }
    // The lengths the plan is built from: into L2 while the grid before this
    // one may still run (a prefetch returns no data, so a later write to the
    // lengths still reaches the loads after the wait).
    if (p.plan_out != nullptr)
        for (int i = 32 * threadIdx.x; i < p.BG / p.Hg; i += 32 * blockDim.x) prefetch_l2_line(p.seqlens + i);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // A plan built here is computed from the lengths alone before the wait
    // below, while the grid before this one (for example the query
    // projection) finishes; the second page stage holds its scratch until the
    // producer's first copy into it, after publish_plan_in_cta.  The lengths
    // must be final when that grid lets its dependents start.
    int32_t* plan_scratch = reinterpret_cast<int32_t*>(smem + L::kKvOff + L::kStageBytes);
    bool first_page_issued = false;
    if (p.plan_out != nullptr && !misaligned) {
        build_plan_in_cta(p, plan_scratch, meta_s);
        // With the range known, the producer thread starts the first page of
        // its first item into stage 0 before the wait as well: the cache and
        // the block table, like the lengths, must be final when the grid
        // before this one lets its dependents start.
        if (threadIdx.x == 0 && p.test_stall == 0) {
            WorkIter it;
            it.init(meta_s, p);
            Item item;
            // (a bad block-table entry is left to the producer, which reports
            // it after the wait: the status word may still be reset before it)
            if (it.next(p, item) &&
                (unsigned)__ldg(p.block_table + (size_t)item.b * p.max_blocks + item.p0) < (unsigned)p.num_blocks) {
                issue_page<NG, S>(&kv_map, p, item, item.p0, 0, smem, page_policy(p));
                first_page_issued = true;
            }
        }
    }
    // Launched as a programmatic dependent: wait until the grid before this
    // one (the schedule kernel, or whatever wrote q) is complete.
    griddep_wait();
    MLA_TRACE_K(1);
    if (misaligned) {
        if (threadIdx.x == 0) atomicOr(p.status, MLA_STATUS_SMEM_ALIGN);
        return;
    }
    const uint32_t tmem = *tmem_slot;
    const int32_t* meta;
    if (p.plan_out != nullptr) {
        publish_plan_in_cta(p, NG, plan_scratch, meta_s);
        meta = meta_s;
    } else {
        const int32_t* hdr = p.sched;
        if (hdr[kHdrMagic] != kSchedMagic || hdr[kHdrG] != p.G ||
            hdr[kHdrBG] != p.BG || hdr[kHdrHg] != p.Hg || hdr[kHdrNG] != NG ||
            hdr[kHdrShift] != kPageShift || hdr[kHdrShareHg] != p.share) {
            if (threadIdx.x == 0) atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
            if (warp == 1) {
                tc_fence_after();
                tmem_dealloc(tmem, L::kTmemCols);
            }
            return;
        }
        meta = hdr + kHdrWords + (size_t)(blockIdx.x / p.share) * kMetaWords;
    }
    const Ctl ctl{abort_flag, p.status};
    MLA_TRACE_K(2);

    if (warp < FwdWarps<NG, S>::kFirstSoftmax) {
        if constexpr (FwdWarps<NG, S>::kSplitRegs) setmaxnreg_dec<FwdWarps<NG, S>::kRegsIssue>();
        if (warp == 0) {
            if (lane == 0) {
                prefetch_tensormap(&kv_map);
                prefetch_tensormap(&q_map);
                run_producer<NG, S>(&kv_map, &q_map, p, meta, smem, ctl, first_page_issued);
            }
        } else if (warp <= G1<NG>::kIssuers) {
            if (lane == 0) run_gemm1<NG, S>(p, meta, smem, tmem, ctl, warp - 1);
            MLA_TRACE_K_BY(5, 32);
        } else {
            if (lane == 0) run_gemm2<NG, S>(p, meta, smem, tmem, ctl, warp - FwdWarps<NG, S>::kFirstG2);
            MLA_TRACE_K_BY(6, (32 * FwdWarps<NG, S>::kFirstG2));
        }
    } else {
        if constexpr (FwdWarps<NG, S>::kSplitRegs) setmaxnreg_inc<FwdWarps<NG, S>::kRegsSoftmax>();
        run_softmax<NG, S>(p, meta, smem, tmem, ctl);
        MLA_TRACE_K_BY(7, (32 * FwdWarps<NG, S>::kFirstSoftmax));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
    MLA_TRACE_K_BY(4, 32);
}

// LSE-weighted merge of split partials; one CTA per (request-group, column),
// four output columns d per thread.  Up to kCombineFast splits, the merge is
// one round of loads after the decode grid completes: each thread reads all
// k partial LSEs and its columns of all k rows and reduces them alone.  With
// more splits the LSEs are read one per thread and reduced across the block
// while the first kCombinePre partial rows are already in flight; further
// rows are read kCombineUnroll at a time.
constexpr int kCombinePre = 8;
constexpr int kCombineUnroll = 8;
// Up to this many splits the merge takes no block reduction.  Measured on
// B200 (graph-replayed steps): at 4 the 128-head workload's ~8,200 combine
// CTAs (2-3 splits each) take 8 us less than with block reductions; at 8 the
// larger arrays cost registers, fewer combine CTAs share an SM, and that
// step is 4 us slower than at 4 (the 16-head workloads were unchanged).
constexpr int kCombineFast = 4;
#ifndef MLA_COMBINE_SLICES
#define MLA_COMBINE_SLICES 8
#endif
// Many splits with few combine CTAs (a short batch over a long context: one
// request over 148 CTAs has ~148 splits in 16 CTAs) make the per-thread chain
// of row loads the step's tail: measured on B200 (graph-replayed, L2 flushed),
// a bs1 x 16K step took 46.5 us against 18.5 us for its decode alone.  When
// the combine grid (one CTA per request-group and column) is smaller than the
// decode grid, the host launches kCombineSlices CTAs per column (grid z).
// Above kCombineSliceMin splits, CTA z then merges the d_v columns
// [z * W, z * W + W) only, W = d_v / kCombineSlices: a row of W floats is
// kLanes = W / 4 threads, so the CTA walks kCombineThreads / kLanes splits side
// by side, each thread group taking every such split after its first, with
// kCombineUnroll rows in flight.  The groups' sums meet in shared memory, in
// group order.  Up to kCombineSliceMin splits, CTA 0 merges the whole row as
// above and the others leave.
constexpr int kCombineSlices = MLA_COMBINE_SLICES;
constexpr int kCombineSliceMin = 16;

template <int kCombineThreads, bool kMax>
__device__ __forceinline__ float combine_block_reduce(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(kFullMask, v, o);
        v = kMax ? fmaxf(v, y) : v + y;
    }
    __syncthreads();  // red[] of an earlier reduction has been read
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    v = red[0];
#pragma unroll
    for (int w = 1; w < kCombineThreads / 32; ++w) v = kMax ? fmaxf(v, red[w]) : v + red[w];
    return v;
}

__device__ __forceinline__ void fma4(float4& acc, float w, const float4& v) {
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
}

template <int kDv, bool kSliced>
__global__ void __launch_bounds__(kDv / 4) mla_decode_combine_kernel(const CombineParams p) {
    constexpr int kCombineThreads = kDv / 4;
    constexpr int kWarps = kCombineThreads / 32;
    // the sliced launch only: a slice row is kLanes threads, kGroups of them per CTA
    constexpr int kLanes = kDv / kCombineSlices / 4;
    constexpr int kGroups = kCombineThreads / (kLanes > 0 ? kLanes : 1);
    constexpr bool kCanSlice = kSliced && kLanes > 0 && kLanes <= 32 && kDv == kCombineSlices * kLanes * 4 &&
                               kCombineThreads == kGroups * kLanes;
    __shared__ float red[kWarps];
    __shared__ float wts[kCombineThreads];
    __shared__ float4 wsum[kGroups > 0 ? kGroups : 1][kLanes > 0 ? kLanes : 1];
    const int bg = blockIdx.x;
    const int n = blockIdx.y;
    // The grid after this one (the output projection, or the next decode) may
    // start its prologue now; it reads nothing of this grid's before its own
    // wait for this grid's completion.
    griddep_launch_dependents();
    // A plan from the schedule kernel may be read before the wait: the decode
    // grid let this grid start only after its own wait on the grid that wrote
    // it.  A plan the decode kernel built itself is complete only after it.
    // What an earlier grid wrote (the plan, the partials) is read with plain
    // loads: a read-only __ldg load may be scheduled above the wait, and one
    // was (a combine that read the header before the decode grid wrote it).
    if (p.plan_in_decode) griddep_wait();
    const int32_t* hdr = p.sched;
    if (hdr[kHdrMagic] != kSchedMagic || hdr[kHdrG] != p.G ||
        hdr[kHdrBG] != p.plan_BG || hdr[kHdrHg] != p.plan_Hg || hdr[kHdrNG] != p.NG ||
        hdr[kHdrShift] != p.shift || hdr[kHdrShareHg] != p.share) {
        if (threadIdx.x == 0 && bg == 0 && n == 0) atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
        return;
    }
    const int b = bg / p.Hg;
    const int g = bg - b * p.Hg;
    // one run (MLA groups): no division
    const int gc = p.run_stride == 0 ? g * p.run_rows + n : item_col(p.run_rows, p.run_stride, g, n);
    if (gc >= p.N) return;
    const int row = p.share > 1 ? b : bg;  // plan row of this request-group
    const int gs = p.share > 1 ? g : 0;
    const int32_t* info = hdr + bg_offset_words(p.G) + (size_t)kBgWords * row;
    const int base = info[0];
    const int k = info[1];
    if (k == 1) return;  // unsplit: the decode kernel wrote the final row
    const bool sliced = kCanSlice && gridDim.z > 1 && k > kCombineSliceMin;
    if (!sliced && blockIdx.z != 0) return;  // CTA 0 of the column merges the whole row
    // Slots of the splits: the one-CTA kernels' fixed slots (split_slot, times
    // the groups sharing a range, plus the group), or the CTA-pair plans'
    // (base + i) * share + group.  In both, split i >= 1 sits at a constant
    // stride from split 1.
    const bool fixed = p.shift == kPageShift;
    if (k > 1 && (base < 0 || (fixed ? split_slot(base, k - 1) * p.share + gs >= p.slots_cap
                                     : ((int64_t)base + k) * p.share > p.slots_cap))) {
        if (threadIdx.x == 0) atomicOr(p.status, MLA_STATUS_BAD_SCHEDULE);
        return;
    }
    const int s = gc / p.heads;
    const int head = gc - s * p.heads;
    const int d0 = threadIdx.x * 4;
    const size_t slot0 = (size_t)base * p.share + gs;
    const size_t slot1 = fixed ? (size_t)split_slot(base, 1) * p.share + gs : slot0 + p.share;
    const size_t sstride = fixed ? 2 * (size_t)p.share : (size_t)p.share;
    auto slot_i = [&](int i) -> size_t { return i == 0 ? slot0 : slot1 + (size_t)(i - 1) * sstride; };
    const float* lp0 = p.lpart + n;
    const float* op0 = p.opart + (size_t)n * kDv + d0;
    auto lse_of = [&](int i) { return lp0[slot_i(i) * p.NG]; };
    auto row_of = [&](int i) { return *reinterpret_cast<const float4*>(op0 + slot_i(i) * p.NG * kDv); };
    MLA_TRACE_STEP_MIN(2);
    if (!p.plan_in_decode) griddep_wait();  // the decode grid's partials are complete and visible
    MLA_TRACE_STEP_MIN(3);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lstar = -INFINITY;
    if (k > 1 && k <= kCombineFast) {
        // Few splits: one round of loads.  Every thread reads the k LSEs (the
        // same words across the block) next to its four columns of each
        // partial row, and reduces them itself.
        float l[kCombineFast];
        float4 v[kCombineFast];
#pragma unroll
        for (int i = 0; i < kCombineFast; ++i)
            if (i < k) {
                l[i] = lse_of(i);
                v[i] = row_of(i);
            }
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kCombineFast; ++i)
            if (i < k) mx = fmaxf(mx, l[i]);
        if (mx != -INFINITY) {
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < kCombineFast; ++i)
                if (i < k) sum += expf(l[i] - mx);
            lstar = mx + logf(sum);
#pragma unroll
            for (int i = 0; i < kCombineFast; ++i)
                if (i < k) fma4(acc, expf(l[i] - lstar), v[i]);
        }
    } else if (sliced) {
        float own = threadIdx.x < k ? lse_of(threadIdx.x) : -INFINITY;
        float mx = own;
        for (int i = threadIdx.x + kCombineThreads; i < k; i += kCombineThreads) mx = fmaxf(mx, lse_of(i));
        mx = combine_block_reduce<kCombineThreads, true>(mx, red);
        if (mx != -INFINITY) {  // uniform across the block
            float sum = 0.f;
            for (int i = threadIdx.x; i < k; i += kCombineThreads)
                sum += expf((i == threadIdx.x ? own : lse_of(i)) - mx);
            sum = combine_block_reduce<kCombineThreads, false>(sum, red);
            lstar = mx + logf(sum);
            const int grp = threadIdx.x / kLanes;
            const float* rs = p.opart + (size_t)n * kDv + blockIdx.z * (kDv / kCombineSlices) + (threadIdx.x % kLanes) * 4;
            auto srow = [&](int i) { return *reinterpret_cast<const float4*>(rs + slot_i(i) * p.NG * kDv); };
            for (int c0 = 0; c0 < k; c0 += kCombineThreads) {
                const int cn = k - c0 < kCombineThreads ? k - c0 : kCombineThreads;
                __syncthreads();  // the previous chunk's weights are consumed
                if (threadIdx.x < cn) wts[threadIdx.x] = expf((c0 == 0 ? own : lse_of(c0 + threadIdx.x)) - lstar);
                __syncthreads();
                int j = grp;
                for (; j + kGroups * (kCombineUnroll - 1) < cn; j += kGroups * kCombineUnroll) {
                    float4 v[kCombineUnroll];
#pragma unroll
                    for (int u = 0; u < kCombineUnroll; ++u) v[u] = srow(c0 + j + kGroups * u);
#pragma unroll
                    for (int u = 0; u < kCombineUnroll; ++u) fma4(acc, wts[j + kGroups * u], v[u]);
                }
                for (; j < cn; j += kGroups) fma4(acc, wts[j], srow(c0 + j));
            }
        }
        wsum[threadIdx.x / kLanes][threadIdx.x % kLanes] = acc;
        __syncthreads();
        if (threadIdx.x < kLanes) {
            acc = wsum[0][threadIdx.x];
#pragma unroll
            for (int w = 1; w < kGroups; ++w) {
                const float4 t = wsum[w][threadIdx.x];
                acc.x += t.x;
                acc.y += t.y;
                acc.z += t.z;
                acc.w += t.w;
            }
        }
    } else if (k > 1) {
        float4 pre[kCombinePre];
#pragma unroll
        for (int i = 0; i < kCombinePre; ++i)
            if (i < k) pre[i] = row_of(i);
        float own = threadIdx.x < k ? lse_of(threadIdx.x) : -INFINITY;
        float mx = own;
        for (int i = threadIdx.x + kCombineThreads; i < k; i += kCombineThreads) mx = fmaxf(mx, lse_of(i));
        mx = combine_block_reduce<kCombineThreads, true>(mx, red);
        if (mx != -INFINITY) {  // uniform across the block
            float sum = 0.f;
            for (int i = threadIdx.x; i < k; i += kCombineThreads)
                sum += expf((i == threadIdx.x ? own : lse_of(i)) - mx);
            sum = combine_block_reduce<kCombineThreads, false>(sum, red);
            lstar = mx + logf(sum);
            for (int c0 = 0; c0 < k; c0 += kCombineThreads) {
                const int cn = k - c0 < kCombineThreads ? k - c0 : kCombineThreads;
                __syncthreads();  // the previous chunk's weights are consumed
                if (threadIdx.x < cn) wts[threadIdx.x] = expf((c0 == 0 ? own : lse_of(c0 + threadIdx.x)) - lstar);
                __syncthreads();
                int i = 0;
                if (c0 == 0) {
#pragma unroll
                    for (int j = 0; j < kCombinePre; ++j)
                        if (j < cn) fma4(acc, wts[j], pre[j]);
                    i = cn < kCombinePre ? cn : kCombinePre;
                }
                for (; i + kCombineUnroll <= cn; i += kCombineUnroll) {
                    float4 v[kCombineUnroll];
#pragma unroll
                    for (int j = 0; j < kCombineUnroll; ++j) v[j] = row_of(c0 + i + j);
#pragma unroll
                    for (int j = 0; j < kCombineUnroll; ++j) fma4(acc, wts[i + j], v[j]);
                }
                for (; i < cn; ++i) fma4(acc, wts[i], row_of(c0 + i));
            }
        }
    }
    const int dcol = sliced ? (int)blockIdx.z * (kDv / kCombineSlices) + (threadIdx.x % kLanes) * 4 : d0;
    const size_t o = (((size_t)b * p.s_q + s) * p.heads + head) * kDv + dcol;
    if (!sliced || threadIdx.x < kLanes) {
        if (p.out_f32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) = acc;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 packed;
            packed.x = *reinterpret_cast<const uint32_t*>(&lo);
            packed.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + o) = packed;
        }
    }
    if (threadIdx.x == 0 && blockIdx.z == 0) p.lse[((size_t)b * p.heads + head) * p.s_q + s] = lstar;
    MLA_TRACE_STEP_MAX(4);
#ifdef MLA_TRACE
    if (threadIdx.x == 0 && bg < 64 && n < 64) g_mla_trace_comb[bg][n] = stamp_timer_ns();
#endif
}


// Builds the persistent-CTA plan on the device (one block of 1024 threads).
// With use_smem the lengths and the unit prefix live in dynamic shared memory
// ((B + BG + 1) int32), so the per-CTA binary searches stay on chip; the
// prefix is also written to the schedule buffer.
__global__ void __launch_bounds__(1024)
    mla_decode_schedule_kernel(const int32_t* __restrict__ seqlens_g, int32_t* __restrict__ sched, int B,
                               int Hg, int NG, int G, int max_blocks, int use_smem, int shift, int share_hg) {
    extern __shared__ int32_t sh[];
    __shared__ int warp_tot[32];
    __shared__ int carry;
    __shared__ int bad_len;
    // The decode kernel that follows may launch now; it waits for this grid
    // to complete before it reads the plan.
    MLA_TRACE_STEP_MIN(0);
    griddep_launch_dependents();
    const int BG = B * Hg;
    int32_t* prefix_g = sched + prefix_offset_words(G, BG);
    int32_t* bginfo = sched + bg_offset_words(G);
    int32_t* meta = sched + kHdrWords;
    const int32_t* seqlens = seqlens_g;
    int32_t* prefix = prefix_g;
    if (threadIdx.x == 0) {
        carry = 0;
        bad_len = 0;
    }
    if (use_smem) {
        for (int i = threadIdx.x; i < B; i += 1024) sh[i] = seqlens_g[i];
        seqlens = sh;
        prefix = sh + B;
    }
    __syncthreads();
    for (int base = 0; base < BG; base += 1024) {
        const int bg = base + threadIdx.x;
        int v = 0;
        if (bg < BG) {
            const int L = seqlens[bg / Hg];
            if (!seqlen_in_range(L, max_blocks)) bad_len = 1;
            v = (int)units_of(blocks_of(clamp_seqlen(L, max_blocks), shift));
        }
        const int incl = block_inclusive_scan(v, warp_tot);
        if (bg < BG) {
            prefix[bg] = carry + incl - v;
            if (use_smem) prefix_g[bg] = carry + incl - v;
        }
        __syncthreads();
        if (threadIdx.x == 1023) carry += incl;
        __syncthreads();
    }
    const int64_t W = carry;
    if (threadIdx.x == 0) {
        prefix[BG] = (int)W;
        prefix_g[BG] = (int)W;
    }
    __syncthreads();
    const int64_t T = units_per_cta(W, G);
    for (int k = threadIdx.x; k < G; k += 1024) cta_meta(prefix, BG, W, T, k, meta + (size_t)k * kMetaWords);
    __syncthreads();
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < BG; base += 1024) {
        const int bg = base + threadIdx.x;
        int ns = 0;
        if (bg < BG) ns = num_splits_of(prefix, bg, pages_in_prefix(prefix, bg), T);
        const int v = ns > 1 ? ns : 0;
        const int incl = block_inclusive_scan(v, warp_tot);
        if (bg < BG) {
            // one-CTA kernels (64-token units): fixed slots; CTA-pair plans: running count
            bginfo[kBgWords * bg] = shift != kPageShift ? carry + incl - v : ns > 1 ? first_split_slot(prefix, bg, T) : 0;
            bginfo[kBgWords * bg + 1] = ns;
        }
        __syncthreads();
        if (threadIdx.x == 1023) carry += incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        sched[kHdrMagic] = kSchedMagic;
        sched[kHdrG] = G;
        sched[kHdrBG] = BG;
        sched[kHdrHg] = Hg;
        sched[kHdrNG] = NG;
        sched[kHdrSlots] = carry;
        sched[kHdrT] = (int)T;
        sched[kHdrStatus] = bad_len ? MLA_STATUS_BAD_SEQLEN : 0;
        sched[kHdrW] = (int)W;
        sched[kHdrBatch] = B;
        sched[kHdrMaxBlocks] = max_blocks;
        sched[kHdrShift] = shift;
        sched[kHdrShareHg] = share_hg;
        for (int i = kHdrShareHg + 1; i < kHdrWords; ++i) sched[i] = 0;
    }
    MLA_TRACE_STEP_MAX(1);
}

}  // namespace mla
