// C ABI of the sm_100a MLA decode library: argument checks, TMA tensor maps,
// launches.  Declarations and their contract: include/mla_decode.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "absorb_kernels.cuh"
#include "decode_kernels.cuh"
#include "pair_kernels.cuh"
#include "rank_combine.cuh"
#include "mla_decode.h"
#include "schedule.cuh"

namespace {

using namespace mla;

constexpr int kAbiVersion = 6;
constexpr int kMaxDevices = 64;
constexpr int32_t kKnownFlags = MLA_FLAG_NO_COMBINE | MLA_FLAG_TEST_STALL | MLA_FLAG_FP32_OUT | MLA_FLAG_INLINE_PLAN;

int validate_dims(const mla_decode_dims* d) {
    if (d == nullptr) return MLA_ERR_INVALID_ARG;
    if (d->batch < 1 || d->s_q < 1 || d->num_heads < 1 || d->num_blocks < 1 ||
        d->max_blocks_per_seq < 1 || d->num_sms < 0 || d->reserved != 0 ||
        (d->flags & ~kKnownFlags) != 0 || (d->causal != 0 && d->causal != 1))
        return MLA_ERR_INVALID_ARG;
    if (d->page_size != kPage || d->d_qk != kDqk || d->d_v != kDv) return MLA_ERR_UNSUPPORTED;
    // One or two new tokens per request (plain decode, or two-token
    // multi-token-prediction decode with the causal rule between them).
    if (d->s_q > 2 || (int64_t)d->num_heads * d->s_q > 256) return MLA_ERR_UNSUPPORTED;
    const Grouping gr = make_grouping(d->num_heads, d->s_q);
    const int64_t BG = (int64_t)d->batch * gr.Hg;
    // Work units and row counts must fit the int32 arithmetic of the kernels.
    if (BG * ((int64_t)d->max_blocks_per_seq + kItemOverhead) >= (int64_t)INT32_MAX) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * gr.N >= (int64_t)INT32_MAX / 2) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * d->max_blocks_per_seq >= (int64_t)INT32_MAX) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

int resolve_ctas(const mla_decode_dims* d, int* G) {
    if (d->num_sms > 0) {
        *G = d->num_sms;
        return MLA_OK;
    }
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    *G = n;
    return MLA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A launch plan.  G and BG are the split-KV plan's own shape: work ranges
// and plan rows (request-groups for the one-CTA kernels; requests for the
// CTA-pair kernel, whose ranges are walked by all head groups side by side).
struct Plan {
    Grouping gr;
    int G;        // work ranges of the plan
    int BG;       // plan rows
    int plan_Hg;  // head groups per plan row (1 for the pair kernel's plan)
    int shift;    // log2 tokens per plan unit
    int share;    // head groups walking each range (1: none)
    int ctas;     // CTAs launched
    bool pair;    // CTA-pair kernel (query groups of 128 columns)
    int64_t slots;
};

// Clusters of the pair kernel that can be resident at once on the current
// device (0 if unknown, e.g. without a device): a persistent grid larger
// than that would run its last clusters as a second wave.
int pair_max_clusters() {
    static int cache[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        cache[dev] = -1;
        if (cudaFuncSetAttribute(mla_decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PairSmem::kBytes) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2);
            cfg.blockDim = dim3(kPairThreads);
            cfg.dynamicSmemBytes = PairSmem::kBytes;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, (void*)mla_decode_pair_kernel, &cfg) == cudaSuccess && n > 0)
                cache[dev] = n;
        }
        cudaGetLastError();
    }
    return cache[dev] > 0 ? cache[dev] : 0;
}

int make_plan(const mla_decode_dims* d, Plan* pl) {
    int rc = validate_dims(d);
    if (rc != MLA_OK) return rc;
    int sms = 0;
    rc = resolve_ctas(d, &sms);
    if (rc != MLA_OK) return rc;
    pl->gr = make_grouping(d->num_heads, d->s_q);
    pl->pair = pl->gr.NG == kPairCols;
    if (pl->pair) {
        // one cluster of two CTAs per pair of SMs; the head groups of a
        // request walk each range side by side on Hg clusters
        int clusters = sms / 2 > 0 ? sms / 2 : 1;
        const int resident = pair_max_clusters();
        if (resident > 0 && clusters > resident) clusters = resident;
        pl->G = clusters / pl->gr.Hg > 0 ? clusters / pl->gr.Hg : 1;
        pl->BG = d->batch;
        pl->plan_Hg = 1;
        pl->shift = kStepShift;
        pl->share = pl->gr.Hg;
        pl->ctas = 2 * pl->G * pl->gr.Hg;
        pl->slots = max_slots(pl->G) * pl->gr.Hg;
    } else {
        pl->G = sms;
        pl->BG = d->batch * pl->gr.Hg;
        pl->plan_Hg = pl->gr.Hg;
        pl->shift = kPageShift;
        pl->share = 1;
        pl->ctas = sms;
        pl->slots = max_slots(pl->G);
    }
    return MLA_OK;
}

size_t workspace_bytes_of(const Plan& pl, int d_v = kDv) {
    const size_t per_slot = (size_t)pl.gr.NG * (d_v + 1) * sizeof(float);
    return (size_t)pl.slots * per_slot;
}

// ---- GQA path: groups of 16 query heads x s_q new tokens, one per KV group ----
constexpr int kGqaHeadsPerGroup = 16;

int validate_gqa(const mla_gqa_dims* d) {
    if (d == nullptr) return MLA_ERR_INVALID_ARG;
    if (d->batch < 1 || d->s_q < 1 || d->num_q_heads < 1 || d->num_kv_groups < 1 || d->num_blocks < 1 ||
        d->max_blocks_per_seq < 1 || d->num_sms < 0 ||
        (d->flags & ~kKnownFlags) != 0 || (d->causal != 0 && d->causal != 1))
        return MLA_ERR_INVALID_ARG;
    if (d->page_size != kPage || d->d_head != ShapeGqa::kDh || d->d_rope != ShapeGqa::kDrope || d->s_q > 2 ||
        (int64_t)d->num_q_heads != (int64_t)kGqaHeadsPerGroup * d->num_kv_groups || d->num_kv_groups > 64)
        return MLA_ERR_UNSUPPORTED;
    const int64_t BG = (int64_t)d->batch * d->num_kv_groups;
    if (BG * ((int64_t)d->max_blocks_per_seq + kItemOverhead) >= (int64_t)INT32_MAX) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * d->num_q_heads * d->s_q >= (int64_t)INT32_MAX / 2) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * d->max_blocks_per_seq >= (int64_t)INT32_MAX) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

int make_plan_gqa(const mla_gqa_dims* d, Plan* pl) {
    int rc = validate_gqa(d);
    if (rc != MLA_OK) return rc;
    mla_decode_dims tmp = {};
    tmp.num_sms = d->num_sms;
    rc = resolve_ctas(&tmp, &pl->G);
    if (rc != MLA_OK) return rc;
    pl->gr.N = d->num_q_heads * d->s_q;
    pl->gr.NG = kGqaHeadsPerGroup * d->s_q;
    pl->gr.Hg = d->num_kv_groups;
    pl->shift = kPageShift;
    pl->pair = false;
    const int sms = pl->G;
    if (d->num_kv_groups > 1 && sms / d->num_kv_groups >= 1) {
        // Shared ranges: the plan has one row per request, and each range is
        // walked by the request's KV groups side by side, one CTA per group,
        // so that the groups read each page's shared RoPE box at about the
        // same time and all but the first read hit L2.
        pl->G = sms / d->num_kv_groups;
        pl->BG = d->batch;
        pl->plan_Hg = 1;
        pl->share = d->num_kv_groups;
    } else {
        pl->BG = d->batch * d->num_kv_groups;
        pl->plan_Hg = pl->gr.Hg;
        pl->share = 1;
    }
    pl->ctas = pl->G * pl->share;
    pl->slots = max_slots(pl->G) * pl->share;
    return MLA_OK;
}

// ---- TMA tensor maps ----
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        else
            cudaGetLastError();
    });
    return fn;
}

// Pool [num_blocks][64][row_width] bf16 viewed as 3-D (col, token, page); box = 64 cols x 64 tokens.
int make_kv_map(CUtensorMap* m, const void* kv, int num_blocks, int row_width = kDqk) {
    auto enc = get_encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)row_width, (cuuint64_t)kPage, (cuuint64_t)num_blocks};
    cuuint64_t strides[2] = {(cuuint64_t)row_width * 2, (cuuint64_t)row_width * 2 * kPage};
    cuuint32_t box[3] = {64, (cuuint32_t)kPage, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Q [B*s_q*h][width] bf16 as 2-D; box = 64 cols x box_rows rows (rows past the end read as zero).
int make_q_map(CUtensorMap* m, const void* q, int rows, int box_rows, int width = kDqk) {
    auto enc = get_encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)width * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

template <int NG, class S>
int ensure_smem_attr() {
    static bool done[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(mla_decode_fwd_kernel<NG, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 FwdSmem<NG, S>::kAlloc) != cudaSuccess)
            return MLA_ERR_CUDA;
        if constexpr (FwdWarps<NG, S>::kSplitRegs) {
            // setmaxnreg.inc waits until the registers it asks for are free in
            // the CTA, so the split must fit the launch allocation exactly as
            // compiled; refuse to launch otherwise.
            using Wp = FwdWarps<NG, S>;
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, mla_decode_fwd_kernel<NG, S>) != cudaSuccess) return MLA_ERR_CUDA;
            if ((long)fa.numRegs * Wp::kThreads < (long)Wp::kRegsIssue * 128 + (long)Wp::kRegsSoftmax * Wp::kSoftmaxThreads)
                return MLA_ERR_UNSUPPORTED;
        }
        done[dev] = true;
    }
    return MLA_OK;
}

int launch_pair(const Plan& pl, const FwdParams& p, const CUtensorMap& kvm, const CUtensorMap& qm,
                cudaStream_t stream) {
    {
        static bool done[kMaxDevices] = {};
        static std::mutex mu;
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            if (cudaFuncSetAttribute(mla_decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     PairSmem::kBytes) != cudaSuccess)
                return MLA_ERR_CUDA;
            done[dev] = true;
        }
    }
    // Clusters of two CTAs (compiled into the kernel), launched as a
    // programmatic dependent of the schedule kernel.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.ctas);
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = PairSmem::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla_decode_pair_kernel, kvm, qm, p) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <int NG, class S>
int launch_fwd(const Plan& pl, const FwdParams& p, const CUtensorMap& kvm, const CUtensorMap& qm,
               cudaStream_t stream) {
    int rc = ensure_smem_attr<NG, S>();
    if (rc != MLA_OK) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.ctas);
    cfg.blockDim = dim3(FwdWarps<NG, S>::kThreads);
    cfg.dynamicSmemBytes = FwdSmem<NG, S>::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla_decode_fwd_kernel<NG, S>, kvm, qm, p) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Query-column layout of the work items, for the kernels' item_col().
struct ColMap {
    int s_q, heads, run_rows, run_stride, batch;
};

template <int kDvT>
int launch_combine(const ColMap& cm, const Plan& pl, const void* schedule, const void* workspace, void* out,
                   float* lse, int32_t flags, bool plan_in_decode, cudaStream_t stream) {
    CombineParams c;
    c.plan_in_decode = plan_in_decode ? 1 : 0;
    c.sched = static_cast<const int32_t*>(schedule);
    c.opart = static_cast<const float*>(workspace);
    c.lpart = c.opart + (size_t)pl.slots * pl.gr.NG * kDvT;
    c.out = out;
    c.out_f32 = (flags & MLA_FLAG_FP32_OUT) ? 1 : 0;
    c.lse = lse;
    c.status = const_cast<int32_t*>(c.sched) + kHdrStatus;
    c.s_q = cm.s_q;
    c.heads = cm.heads;
    c.N = pl.gr.N;
    c.NG = pl.gr.NG;
    c.Hg = pl.gr.Hg;
    c.G = pl.G;
    c.BG = cm.batch * pl.gr.Hg;
    c.slots_cap = (int)pl.slots;
    c.plan_BG = pl.BG;
    c.plan_Hg = pl.plan_Hg;
    c.shift = pl.shift;
    c.share = pl.share;
    c.run_rows = cm.run_rows;
    c.run_stride = cm.run_stride;
    cudaLaunchConfig_t cfg = {};
    // Fewer combine CTAs than decode CTAs: several per column, so that many
    // splits are merged in d_v slices (mla_decode_combine_kernel).
    const bool slices = kDvT == kDv && (int64_t)c.BG * pl.gr.NG < pl.ctas;
    cfg.gridDim = dim3(c.BG, pl.gr.NG, slices ? kCombineSlices : 1);
    cfg.blockDim = dim3(kDvT / 4);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = slices ? cudaLaunchKernelEx(&cfg, mla_decode_combine_kernel<kDvT, true>, c)
                                 : cudaLaunchKernelEx(&cfg, mla_decode_combine_kernel<kDvT, false>, c);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

ColMap mla_colmap(const mla_decode_dims* d, const Plan& pl) {
    return ColMap{d->s_q, d->num_heads, pl.gr.NG, 0, d->batch};
}

// MLA_FLAG_INLINE_PLAN: the one-CTA decode kernel builds the plan itself when
// its unit prefix fits one page stage; otherwise (CTA-pair kernel, or more
// request-groups) the call enqueues the schedule kernel before the decode.
template <class S>
int inline_plan_cap(int NG) {
    return NG == 16 ? FwdSmem<16, S>::kInlinePlanMaxBG
         : NG == 32 ? FwdSmem<32, S>::kInlinePlanMaxBG
                    : FwdSmem<64, S>::kInlinePlanMaxBG;
}
bool plan_in_kernel(int32_t flags, const Plan& pl, bool gqa) {
    if (!(flags & MLA_FLAG_INLINE_PLAN) || pl.pair) return false;
    return pl.BG <= (gqa ? inline_plan_cap<ShapeGqa>(pl.gr.NG) : inline_plan_cap<ShapeMla>(pl.gr.NG));
}

int launch_schedule(const Plan& pl, int batch, int max_blocks, const int32_t* cache_seqlens, void* schedule,
                    cudaStream_t stream) {
    // Lengths and unit prefix in shared memory when they fit the default 48 KB.
    const size_t sh_bytes = ((size_t)batch + pl.BG + 1) * sizeof(int32_t);
    const int use_smem = sh_bytes <= 48 * 1024 ? 1 : 0;
    mla_decode_schedule_kernel<<<1, 1024, use_smem ? sh_bytes : 0, stream>>>(
        cache_seqlens, static_cast<int32_t*>(schedule), batch, pl.plan_Hg, pl.gr.NG, pl.G, max_blocks, use_smem,
        pl.shift, pl.share);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// ---- scratch of the allocation-free entry point ----
// One array per device, in this library's module; allocated by the driver when
// the module is loaded on a device and held until the process exits.
constexpr size_t kNoAllocScratchBytes = MLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_mla_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and cached.
int noalloc_scratch(void** out) {
    static void* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_mla_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return MLA_ERR_CUDA;
        }
        addr[dev] = ptr;
    }
    *out = addr[dev];
    return MLA_OK;
}

// ---- absorbed projections ----
int validate_absorb(const mla_absorb_dims* d) {
    if (d == nullptr) return MLA_ERR_INVALID_ARG;
    if (d->tokens < 1 || d->tokens > 65535 * kProjTokens || d->num_heads < 1 || d->num_heads > 65535)
        return MLA_ERR_INVALID_ARG;
    if (d->d_nope != kProjNope || d->d_rope != kProjRope || d->d_latent != kProjLatent ||
        d->d_v_head != kProjVHead)
        return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

// Per-head weight [h][rows][cols] bf16 as 3-D (col, row, head); box = 64 cols x box_rows rows.
int make_weight_map(CUtensorMap* m, const void* w, int heads, int rows, int cols, int box_rows) {
    auto enc = get_encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)heads};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * rows};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Token rows [T][h][width] bf16 as 3-D (col, head, token); box = 64 cols x 1 head x 64 tokens.
int make_rows_map(CUtensorMap* m, const void* x, int T, int heads, int width) {
    auto enc = get_encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)heads, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)width * 2 * heads};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kProjTokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

template <int kKind>
int launch_absorb(const mla_absorb_dims* d, const void* x, const void* w, void* out, int32_t* status,
                  cudaStream_t stream) {
    using P = ProjShape<kKind>;
    static bool done[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            if (cudaFuncSetAttribute(mla_absorb_kernel<kKind>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     P::kSmem) != cudaSuccess)
                return MLA_ERR_CUDA;
            done[dev] = true;
        }
    }
    CUtensorMap wm, xm;
    int rc = kKind == 0 ? make_weight_map(&wm, w, d->num_heads, kProjNope, kProjLatent, kProjTile)
                        : make_weight_map(&wm, w, d->num_heads, kProjLatent, kProjVHead, kProjTile);
    if (rc != MLA_OK) return rc;
    rc = make_rows_map(&xm, x, d->tokens, d->num_heads, P::kInW);
    if (rc != MLA_OK) return rc;
    ProjParams p;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.rope_in = static_cast<const __nv_bfloat16*>(x);
    p.status = status;
    p.T = d->tokens;
    p.heads = d->num_heads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P::kGridX, d->num_heads, (d->tokens + kProjTokens - 1) / kProjTokens);
    cfg.blockDim = dim3(kProjThreads);
    cfg.dynamicSmemBytes = P::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla_absorb_kernel<kKind>, wm, xm, p) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

// The split-KV plan computed on the host, word for word what the schedule
// kernel writes (schedule.cuh); for inspection and tests.
void host_plan(const Plan& pl, int batch, int mb, const int32_t* seqlens, void* schedule_host) {
    const int G = pl.G, BG = pl.BG, Hg = pl.plan_Hg, sh = pl.shift;
    int32_t* s = static_cast<int32_t*>(schedule_host);
    int32_t* prefix = s + prefix_offset_words(G, BG);
    int32_t* bginfo = s + bg_offset_words(G);
    int bad_len = 0;
    int64_t W = 0;
    for (int bg = 0; bg < BG; ++bg) {
        const int L = seqlens[bg / Hg];
        if (!seqlen_in_range(L, mb)) bad_len = 1;
        prefix[bg] = (int32_t)W;
        W += units_of(blocks_of(clamp_seqlen(L, mb), sh));
    }
    prefix[BG] = (int32_t)W;
    const int64_t T = units_per_cta(W, G);
    for (int k = 0; k < G; ++k) cta_meta(prefix, BG, W, T, k, s + kHdrWords + (size_t)k * kMetaWords);
    int64_t slots = 0;
    for (int bg = 0; bg < BG; ++bg) {
        const int ns = num_splits_of(prefix, bg, pages_in_prefix(prefix, bg), T);
        bginfo[kBgWords * bg] = pl.pair ? (int32_t)slots : ns > 1 ? first_split_slot(prefix, bg, T) : 0;
        bginfo[kBgWords * bg + 1] = ns;
        if (ns > 1) slots += ns;
    }
    std::memset(s, 0, kHdrWords * sizeof(int32_t));
    s[kHdrMagic] = kSchedMagic;
    s[kHdrG] = G;
    s[kHdrBG] = BG;
    s[kHdrHg] = Hg;
    s[kHdrNG] = pl.gr.NG;
    s[kHdrSlots] = (int32_t)slots;
    s[kHdrT] = (int32_t)T;
    s[kHdrStatus] = bad_len ? MLA_STATUS_BAD_SEQLEN : 0;
    s[kHdrW] = (int32_t)W;
    s[kHdrBatch] = batch;
    s[kHdrMaxBlocks] = mb;
    s[kHdrShift] = sh;
    s[kHdrShareHg] = pl.share;
}

extern "C" {

int mla_decode_version(void) { return kAbiVersion; }

const char* mla_decode_strerror(int code) {
    switch (code) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or bad dims)";
        case MLA_ERR_UNSUPPORTED:
            return "unsupported shape (page_size must be 64, d_qk 576, d_v 512, s_q 1 or 2, heads*s_q <= 256)";
        case MLA_ERR_CUDA: return "CUDA runtime or launch error";
        case MLA_ERR_BAD_SCHEDULE: return "schedule buffer does not match these dims";
        case MLA_ERR_SCRATCH_TOO_SMALL:
            return "request needs more than the 24 MiB built-in scratch of mla_decode_fwd_noalloc; "
                   "use mla_decode_fwd with caller-allocated schedule and workspace";
        default: return "unknown error code";
    }
}

size_t mla_decode_schedule_bytes(const mla_decode_dims* dims) {
    Plan pl;
    if (make_plan(dims, &pl) != MLA_OK) return 0;
    return (size_t)schedule_words(pl.G, pl.BG) * sizeof(int32_t);
}

size_t mla_decode_workspace_bytes(const mla_decode_dims* dims) {
    Plan pl;
    if (make_plan(dims, &pl) != MLA_OK) return 0;
    return workspace_bytes_of(pl);
}

int mla_decode_get_schedule(const mla_decode_dims* dims, const int32_t* cache_seqlens, void* schedule,
                            void* stream) {
    Plan pl;
    int rc = make_plan(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(cache_seqlens) || !aligned16(schedule)) return MLA_ERR_INVALID_ARG;
    return launch_schedule(pl, dims->batch, dims->max_blocks_per_seq, cache_seqlens, schedule,
                           static_cast<cudaStream_t>(stream));
}

int mla_decode_get_schedule_host(const mla_decode_dims* dims, const int32_t* seqlens, void* schedule_host) {
    int rc = validate_dims(dims);
    if (rc != MLA_OK) return rc;
    if (dims->num_sms <= 0 || seqlens == nullptr || schedule_host == nullptr) return MLA_ERR_INVALID_ARG;
    Plan pl;
    rc = make_plan(dims, &pl);
    if (rc != MLA_OK) return rc;
    host_plan(pl, dims->batch, dims->max_blocks_per_seq, seqlens, schedule_host);
    return MLA_OK;
}

int mla_decode_fwd(const mla_decode_dims* dims, void* schedule, void* workspace, const void* q,
                   const void* kv_cache, const int32_t* block_table, const int32_t* cache_seqlens,
                   float softmax_scale, void* out, float* lse, void* stream) {
    Plan pl;
    int rc = make_plan(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(schedule) || !aligned16(workspace) || !aligned16(q) || !aligned16(kv_cache) ||
        !aligned16(block_table) || !aligned16(cache_seqlens) || !aligned16(out) || !aligned16(lse))
        return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    CUtensorMap kvm, qm;
    rc = make_kv_map(&kvm, kv_cache, dims->num_blocks);
    if (rc != MLA_OK) return rc;
    // Q boxes: the group's rows (one CTA of a pair loads 64 of its 128)
    rc = make_q_map(&qm, q, dims->batch * pl.gr.N, pl.pair ? kPairCols / 2 : pl.gr.NG);
    if (rc != MLA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool in_kernel = plan_in_kernel(dims->flags, pl, false);
    if ((dims->flags & MLA_FLAG_INLINE_PLAN) && !in_kernel) {
        rc = launch_schedule(pl, dims->batch, dims->max_blocks_per_seq, cache_seqlens, schedule, st);
        if (rc != MLA_OK) return rc;
    }
    FwdParams p;
    p.sched = static_cast<const int32_t*>(schedule);
    p.plan_out = in_kernel ? static_cast<int32_t*>(schedule) : nullptr;
    p.block_table = block_table;
    p.seqlens = cache_seqlens;
    p.kv = static_cast<const uint8_t*>(kv_cache);
    p.out = out;
    p.out_f32 = (dims->flags & MLA_FLAG_FP32_OUT) ? 1 : 0;
    p.lse = lse;
    p.opart = static_cast<float*>(workspace);
    p.lpart = p.opart + (size_t)pl.slots * pl.gr.NG * kDv;
    p.status = const_cast<int32_t*>(p.sched) + kHdrStatus;
    p.s_q = dims->s_q;
    p.heads = dims->num_heads;
    p.N = pl.gr.N;
    p.num_blocks = dims->num_blocks;
    p.max_blocks = dims->max_blocks_per_seq;
    p.causal = dims->causal;
    p.G = pl.G;
    p.BG = pl.BG;
    p.Hg = pl.pair ? pl.share : pl.gr.Hg;  // pair kernel: head groups walking each range
    p.share = 1;
    p.slots_cap = (int)pl.slots;
    p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
    p.test_stall = (dims->flags & MLA_FLAG_TEST_STALL) ? 1 : 0;
    p.run_rows = pl.gr.NG;
    p.run_stride = 0;
    p.kv_groups = 1;
    rc = pl.pair            ? launch_pair(pl, p, kvm, qm, st)
         : pl.gr.NG == 16   ? launch_fwd<16, ShapeMla>(pl, p, kvm, qm, st)
         : pl.gr.NG == 32   ? launch_fwd<32, ShapeMla>(pl, p, kvm, qm, st)
                            : launch_fwd<64, ShapeMla>(pl, p, kvm, qm, st);
    if (rc != MLA_OK) return rc;
    if (dims->flags & MLA_FLAG_NO_COMBINE) return MLA_OK;
    return launch_combine<kDv>(mla_colmap(dims, pl), pl, schedule, workspace, out, lse, dims->flags, in_kernel, st);
}

int mla_decode_combine(const mla_decode_dims* dims, const void* schedule, const void* workspace, void* out,
                       float* lse, void* stream) {
    Plan pl;
    int rc = make_plan(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(schedule) || !aligned16(workspace) || !aligned16(out) || !aligned16(lse))
        return MLA_ERR_INVALID_ARG;
    return launch_combine<kDv>(mla_colmap(dims, pl), pl, schedule, workspace, out, lse, dims->flags,
                               plan_in_kernel(dims->flags, pl, false), static_cast<cudaStream_t>(stream));
}

size_t mla_gqa_decode_schedule_bytes(const mla_gqa_dims* dims) {
    Plan pl;
    if (make_plan_gqa(dims, &pl) != MLA_OK) return 0;
    return (size_t)schedule_words(pl.G, pl.BG) * sizeof(int32_t);
}

size_t mla_gqa_decode_workspace_bytes(const mla_gqa_dims* dims) {
    Plan pl;
    if (make_plan_gqa(dims, &pl) != MLA_OK) return 0;
    return workspace_bytes_of(pl, ShapeGqa::kDv);
}

int mla_gqa_decode_get_schedule(const mla_gqa_dims* dims, const int32_t* cache_seqlens, void* schedule,
                                void* stream) {
    Plan pl;
    int rc = make_plan_gqa(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(cache_seqlens) || !aligned16(schedule)) return MLA_ERR_INVALID_ARG;
    return launch_schedule(pl, dims->batch, dims->max_blocks_per_seq, cache_seqlens, schedule,
                           static_cast<cudaStream_t>(stream));
}

int mla_gqa_decode_get_schedule_host(const mla_gqa_dims* dims, const int32_t* seqlens, void* schedule_host) {
    int rc = validate_gqa(dims);
    if (rc != MLA_OK) return rc;
    if (dims->num_sms <= 0 || seqlens == nullptr || schedule_host == nullptr) return MLA_ERR_INVALID_ARG;
    Plan pl;
    rc = make_plan_gqa(dims, &pl);
    if (rc != MLA_OK) return rc;
    host_plan(pl, dims->batch, dims->max_blocks_per_seq, seqlens, schedule_host);
    return MLA_OK;
}

int mla_gqa_decode_fwd(const mla_gqa_dims* dims, void* schedule, void* workspace, const void* q,
                       const void* kv_cache, const int32_t* block_table, const int32_t* cache_seqlens,
                       float softmax_scale, void* out, float* lse, void* stream) {
    Plan pl;
    int rc = make_plan_gqa(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(schedule) || !aligned16(workspace) || !aligned16(q) || !aligned16(kv_cache) ||
        !aligned16(block_table) || !aligned16(cache_seqlens) || !aligned16(out) || !aligned16(lse))
        return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    CUtensorMap kvm, qm;
    rc = make_kv_map(&kvm, kv_cache, dims->num_blocks, ShapeGqa::row_width(dims->num_kv_groups));
    if (rc != MLA_OK) return rc;
    rc = make_q_map(&qm, q, dims->batch * pl.gr.N, kGqaHeadsPerGroup, ShapeGqa::kDqk);
    if (rc != MLA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool in_kernel = plan_in_kernel(dims->flags, pl, true);
    if ((dims->flags & MLA_FLAG_INLINE_PLAN) && !in_kernel) {
        rc = launch_schedule(pl, dims->batch, dims->max_blocks_per_seq, cache_seqlens, schedule, st);
        if (rc != MLA_OK) return rc;
    }
    FwdParams p;
    p.sched = static_cast<const int32_t*>(schedule);
    p.plan_out = in_kernel ? static_cast<int32_t*>(schedule) : nullptr;
    p.block_table = block_table;
    p.seqlens = cache_seqlens;
    p.kv = static_cast<const uint8_t*>(kv_cache);
    p.out = out;
    p.out_f32 = (dims->flags & MLA_FLAG_FP32_OUT) ? 1 : 0;
    p.lse = lse;
    p.opart = static_cast<float*>(workspace);
    p.lpart = p.opart + (size_t)pl.slots * pl.gr.NG * ShapeGqa::kDv;
    p.status = const_cast<int32_t*>(p.sched) + kHdrStatus;
    p.s_q = dims->s_q;
    p.heads = dims->num_q_heads;
    p.N = pl.gr.N;
    p.num_blocks = dims->num_blocks;
    p.max_blocks = dims->max_blocks_per_seq;
    p.causal = dims->causal;
    p.G = pl.G;
    p.BG = pl.BG;
    p.Hg = pl.plan_Hg;
    p.share = pl.share;
    p.slots_cap = (int)pl.slots;
    p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
    p.test_stall = (dims->flags & MLA_FLAG_TEST_STALL) ? 1 : 0;
    p.run_rows = kGqaHeadsPerGroup;  // one run of 16 heads per new token
    p.run_stride = dims->num_q_heads;
    p.kv_groups = dims->num_kv_groups;
    rc = pl.gr.NG == 16 ? launch_fwd<16, ShapeGqa>(pl, p, kvm, qm, st) : launch_fwd<32, ShapeGqa>(pl, p, kvm, qm, st);
    if (rc != MLA_OK) return rc;
    if (dims->flags & MLA_FLAG_NO_COMBINE) return MLA_OK;
    return launch_combine<ShapeGqa::kDv>(ColMap{dims->s_q, dims->num_q_heads, kGqaHeadsPerGroup, dims->num_q_heads, dims->batch},
                                         pl, schedule, workspace, out, lse, dims->flags, in_kernel, st);
}

int mla_gqa_decode_combine(const mla_gqa_dims* dims, const void* schedule, const void* workspace, void* out,
                           float* lse, void* stream) {
    Plan pl;
    int rc = make_plan_gqa(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (!aligned16(schedule) || !aligned16(workspace) || !aligned16(out) || !aligned16(lse))
        return MLA_ERR_INVALID_ARG;
    return launch_combine<ShapeGqa::kDv>(ColMap{dims->s_q, dims->num_q_heads, kGqaHeadsPerGroup, dims->num_q_heads, dims->batch},
                                         pl, schedule, workspace, out, lse, dims->flags,
                                         plan_in_kernel(dims->flags, pl, true), static_cast<cudaStream_t>(stream));
}

#ifdef MLA_TRACE
// Tracing builds only: copies the per-CTA event buffer (see decode_kernels.cuh)
// and the per-role event counts to host memory.
int mla_decode_trace_fetch(void* events_host, size_t events_bytes, void* counts_host, size_t counts_bytes) {
    if (events_bytes != sizeof(g_mla_trace) || counts_bytes != sizeof(g_mla_trace_count)) return MLA_ERR_INVALID_ARG;
    if (cudaMemcpyFromSymbol(events_host, g_mla_trace, events_bytes) != cudaSuccess ||
        cudaMemcpyFromSymbol(counts_host, g_mla_trace_count, counts_bytes) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}
// Copies the combine CTAs' exit stamps.
int mla_decode_trace_fetch_comb(void* host, size_t bytes) {
    if (bytes != sizeof(g_mla_trace_comb)) return MLA_ERR_INVALID_ARG;
    if (cudaMemcpyFromSymbol(host, g_mla_trace_comb, bytes) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}
// Copies the kernel-level stamps (decode CTAs, then the step's five) and
// resets the step stamps for the next call.
int mla_decode_trace_fetch_k(void* k_host, size_t k_bytes, void* step_host, size_t step_bytes) {
    if (k_bytes != sizeof(g_mla_trace_k) || step_bytes != sizeof(g_mla_trace_step)) return MLA_ERR_INVALID_ARG;
    unsigned long long init[8];
    for (int i = 0; i < 8; ++i) init[i] = (i == 1 || i == 4) ? 0ull : ~0ull;
    if (cudaMemcpyFromSymbol(k_host, g_mla_trace_k, k_bytes) != cudaSuccess ||
        cudaMemcpyFromSymbol(step_host, g_mla_trace_step, step_bytes) != cudaSuccess ||
        cudaMemcpyToSymbol(g_mla_trace_step, init, sizeof(init)) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}
#endif

int mla_decode_fwd_noalloc(const mla_decode_dims* dims, const void* q, const void* kv_cache,
                           const int32_t* block_table, const int32_t* cache_seqlens, float softmax_scale,
                           void* out, float* lse, void* stream) {
    Plan pl;
    int rc = make_plan(dims, &pl);
    if (rc != MLA_OK) return rc;
    if (dims->flags & MLA_FLAG_NO_COMBINE) return MLA_ERR_INVALID_ARG;  // no workspace to combine from later
    if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(block_table) || !aligned16(cache_seqlens) ||
        !aligned16(out) || !aligned16(lse) || !std::isfinite(softmax_scale))
        return MLA_ERR_INVALID_ARG;
    const size_t sched_bytes = ((size_t)schedule_words(pl.G, pl.BG) * sizeof(int32_t) + 255) & ~(size_t)255;
    const size_t ws_bytes = workspace_bytes_of(pl);
    if (sched_bytes + ws_bytes > kNoAllocScratchBytes) return MLA_ERR_SCRATCH_TOO_SMALL;
    void* base = nullptr;
    rc = noalloc_scratch(&base);
    if (rc != MLA_OK) return rc;
    uint8_t* schedule = static_cast<uint8_t*>(base);
    uint8_t* workspace = schedule + sched_bytes;
    rc = mla_decode_get_schedule(dims, cache_seqlens, schedule, stream);
    if (rc != MLA_OK) return rc;
    return mla_decode_fwd(dims, schedule, workspace, q, kv_cache, block_table, cache_seqlens, softmax_scale,
                          out, lse, stream);
}

int mla_decode_get_status(const void* schedule, int32_t* host_status) {
    if (!aligned16(schedule) || host_status == nullptr) return MLA_ERR_INVALID_ARG;
    const int32_t* src = static_cast<const int32_t*>(schedule) + kHdrStatus;
    if (cudaMemcpy(host_status, src, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

int mla_absorb_q(const mla_absorb_dims* dims, const void* q_in, const void* w_uk, void* q_out, int32_t* status,
                 void* stream) {
    int rc = validate_absorb(dims);
    if (rc != MLA_OK) return rc;
    if (!aligned16(q_in) || !aligned16(w_uk) || !aligned16(q_out)) return MLA_ERR_INVALID_ARG;
    if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return MLA_ERR_INVALID_ARG;
    return launch_absorb<0>(dims, q_in, w_uk, q_out, status, static_cast<cudaStream_t>(stream));
}

int mla_absorb_o(const mla_absorb_dims* dims, const void* o, const void* w_uv, void* out, int32_t* status,
                 void* stream) {
    int rc = validate_absorb(dims);
    if (rc != MLA_OK) return rc;
    if (!aligned16(o) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
    if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return MLA_ERR_INVALID_ARG;
    return launch_absorb<1>(dims, o, w_uv, out, status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

template <typename TIn>
int combine_ranks(int32_t num_ranks, int32_t batch, int32_t s_q, int32_t num_heads, int32_t d_v,
                  const void* o_parts, const float* lse_parts, void* out, float* lse, void* stream) {
    if (num_ranks < 1 || num_ranks > kRankCombineMaxRanks || batch < 1 || s_q < 1 || num_heads < 1)
        return MLA_ERR_INVALID_ARG;
    if (d_v != kDv && d_v != ShapeGqa::kDv) return MLA_ERR_UNSUPPORTED;
    const long long rows = (long long)batch * s_q * num_heads;
    const long long blocks = (rows + kRankCombineWarps - 1) / kRankCombineWarps;
    if (blocks > 0x7fffffffLL || rows * num_ranks * d_v > (1LL << 40)) return MLA_ERR_INVALID_ARG;
    if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(out) || !aligned16(lse))
        return MLA_ERR_INVALID_ARG;
    RankCombineParams p;
    p.o_parts = o_parts;
    p.lse_parts = lse_parts;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.R = num_ranks;
    p.B = batch;
    p.s_q = s_q;
    p.h = num_heads;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_v == kDv)
        mla_rank_combine_kernel<kDv, TIn><<<(unsigned)blocks, 32 * kRankCombineWarps, 0, st>>>(p);
    else
        mla_rank_combine_kernel<ShapeGqa::kDv, TIn><<<(unsigned)blocks, 32 * kRankCombineWarps, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

extern "C" {

int mla_decode_combine_ranks(int32_t num_ranks, int32_t batch, int32_t s_q, int32_t num_heads, int32_t d_v,
                             const void* o_parts, const float* lse_parts, void* out, float* lse, void* stream) {
    return combine_ranks<__nv_bfloat16>(num_ranks, batch, s_q, num_heads, d_v, o_parts, lse_parts, out, lse, stream);
}

int mla_decode_combine_ranks_f32(int32_t num_ranks, int32_t batch, int32_t s_q, int32_t num_heads, int32_t d_v,
                                 const float* o_parts, const float* lse_parts, void* out, float* lse,
                                 void* stream) {
    return combine_ranks<float>(num_ranks, batch, s_q, num_heads, d_v, o_parts, lse_parts, out, lse, stream);
}

}  // extern "C"
