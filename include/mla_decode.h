/*
 * mla_decode.h — C ABI of the B200 (sm_100a) absorbed-MQA MLA decode library.
 *
 * The operation (one decode step of Multi-Head Latent Attention in its
 * absorbed, multi-query form):
 *
 *   For request b, new-token index s < s_q and head h, with L_b the cached
 *   length and L_vis = L_b - s_q + 1 + s when causal (else L_b):
 *     z_t = softmax_scale * <q[b,s,h,0:576], row_t[0:576]>,  t < L_vis
 *     out[b,s,h,:] = sum_t softmax(z)_t * row_t[0:512]
 *     lse[b,h,s]   = log(sum_t exp(z_t))                      (natural log)
 *   where row_t = kv_cache[block_table[b][t/64]][t%64][0][:].
 *
 *   - All heads attend directly to one shared latent cache whose rows are a
 *     512-wide latent plus a 64-wide shared RoPE key: the full row is the key,
 *     the latent is the value.  GQLA technical summary (gist.science, pt,
 *     2605.15250), "Caminho MQA-Absorvido"; FlashMLA-ETAP technical summary
 *     (gist.science, pt, 2506.01969), "Limitações" (16 heads, head dim 576).
 *   - The kernel evaluates it in the transposed order S^T = K Q^T,
 *     P^T = softmax(S^T) over the KV axis, O = (V^T P^T)^T, so that the long
 *     KV axis is the MMA M dimension and heads x s_q is N.  FlashMLA-ETAP
 *     technical summary, "Mecanismo Central" (and the arXiv abstract of
 *     2506.01969 on fugumt.com).  The result equals the definition above up
 *     to floating-point rounding.
 *   - Long KV ranges are split across CTAs (split-KV); the fp32 partials are
 *     merged by LSE weighting, which is exact: the softmax over a union of
 *     disjoint ranges is the LSE-weighted mix of the per-range softmaxes.
 *
 * Conventions for every entry point:
 *   - Data pointers are CUDA device pointers owned by the caller (e.g. from
 *     PyTorch); the library never allocates or frees device memory, never
 *     synchronises the device (except mla_decode_get_status, which copies one
 *     word to the host), and enqueues work only on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream).
 *   - Every device pointer must be 16-byte aligned and every tensor
 *     contiguous in the layout stated.
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* code; arguments are
 *     checked before anything is enqueued, so an error return means nothing
 *     was launched.  mla_decode_strerror() names a code.
 *   - Faults the device detects while running (a block-table entry outside
 *     [0, num_blocks), a cache length outside [0, 64*max_blocks_per_seq), a
 *     pipeline wait that exceeded its time limit) are OR-ed as MLA_STATUS_*
 *     bits into a status word kept in the schedule buffer; the kernels skip or
 *     clamp the offending access instead of trapping.  The word is cleared by
 *     mla_decode_get_schedule and read with mla_decode_get_status.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define MLA_OK 0
#define MLA_ERR_INVALID_ARG (-1)  /* null or misaligned pointer, negative size, bad dims */
#define MLA_ERR_UNSUPPORTED (-2)  /* page_size != 64, d_qk != 576, d_v != 512, s_q not 1 or 2, heads*s_q > 256 */
#define MLA_ERR_CUDA (-3)         /* a CUDA runtime/driver call or launch failed */
#define MLA_ERR_BAD_SCHEDULE (-4) /* schedule buffer was not built for these dims */
#define MLA_ERR_SCRATCH_TOO_SMALL (-5) /* mla_decode_fwd_noalloc: the request needs more than its built-in scratch */

/* device status bits (mla_decode_get_status) */
#define MLA_STATUS_BAD_BLOCK_TABLE 0x1 /* an entry was outside [0, num_blocks); page 0 was read instead */
#define MLA_STATUS_TIMEOUT 0x2         /* a pipeline wait exceeded its limit; that CTA stopped early */
#define MLA_STATUS_BAD_SEQLEN 0x4      /* cache_seqlens[b] outside [0, 64*max_blocks_per_seq]; clamped */
#define MLA_STATUS_BAD_SCHEDULE 0x8    /* schedule header did not match the launch; nothing written */
#define MLA_STATUS_SMEM_ALIGN 0x10     /* dynamic shared memory base not 1 KB aligned (64-column groups,
                                          which have no room to realign); nothing written */

/* dims.flags */
#define MLA_FLAG_NO_COMBINE 0x1 /* mla_decode_fwd does not enqueue the combine; call mla_decode_combine */
/* Test hook for the timeout path, never set in normal use: the producer of
 * every CTA leaves the first page of its first work item unloaded, so the
 * GEMM1 wait on it runs out after its 1 s limit.  The call then reports
 * MLA_STATUS_TIMEOUT through mla_decode_get_status, its outputs are undefined,
 * and the device stays usable. */
#define MLA_FLAG_TEST_STALL 0x2
/* `out` is fp32 [batch][s_q][num_heads][d_v] instead of bf16: the result as
 * accumulated, before any rounding to bf16.  For a caller that feeds the
 * output to an fp32 consumer (for example the output projection, or an
 * exchange of partial results between GPUs), and for accuracy checks of the
 * accumulation itself.  Applies to mla_decode_fwd, mla_decode_combine and
 * the GQA-path calls; pass the same flags to both when combining separately. */
#define MLA_FLAG_FP32_OUT 0x4
/* mla_decode_fwd (and mla_gqa_decode_fwd) build the split-KV plan themselves
 * from cache_seqlens, so a step needs no mla_decode_get_schedule call: for
 * query groups of up to 64 columns (heads * s_q <= 64; every GQA shape) the
 * decode kernel computes its own work range in its prologue, which removes
 * the schedule kernel's launch from the step, and writes the same plan
 * mla_decode_get_schedule would into `schedule`; for wider groups, or more
 * request-groups than its shared memory holds (batch * groups > 18,384 for
 * MLA, > 10,192 for GQA), the call enqueues the schedule kernel before the
 * decode kernel.  The status word is not cleared by these calls: call
 * mla_decode_get_schedule once on a new buffer to clear it, after which it
 * collects the faults of every later call until the next
 * mla_decode_get_schedule.  Pass the same flags to mla_decode_combine.
 * The decode kernel is a programmatic dependent of the kernel before it on
 * the stream and reads cache_seqlens before it waits for that kernel's end:
 * the lengths must be final when that kernel lets its dependents start.
 * Kernels that do not use programmatic launch, and this library's own
 * kernels, always satisfy this. */
#define MLA_FLAG_INLINE_PLAN 0x8

typedef struct mla_decode_dims {
    int32_t batch;              /* B >= 1 */
    int32_t s_q;                /* new tokens per request: 1 or 2 (else MLA_ERR_UNSUPPORTED) */
    int32_t num_heads;          /* h >= 1, h * s_q <= 256 */
    int32_t num_blocks;         /* pages in the pool */
    int32_t max_blocks_per_seq; /* row stride of block_table */
    int32_t page_size;          /* must be 64 */
    int32_t d_qk;               /* must be 576 (512 latent + 64 RoPE) */
    int32_t d_v;                /* must be 512 (the latent columns) */
    int32_t causal;             /* 1: token s sees rows [0, L - s_q + s]; ignored when s_q == 1 */
    int32_t num_sms;            /* persistent CTAs; 0 = the current device's SM count */
    int32_t flags;              /* MLA_FLAG_* */
    int32_t reserved;           /* must be 0 */
} mla_decode_dims;

/* Size in bytes of the schedule buffer for these dims (0 if dims are invalid
 * or num_sms == 0 and no device can be queried). */
size_t mla_decode_schedule_bytes(const mla_decode_dims* dims);

/* Size in bytes of the workspace: fp32 partial outputs and LSEs of split
 * requests (at most 2 per persistent CTA). 0 if dims are invalid. */
size_t mla_decode_workspace_bytes(const mla_decode_dims* dims);

/* Split-KV work partitioning.  Reads cache_seqlens (device, int32 [batch])
 * and writes the persistent-CTA work plan into `schedule` (device,
 * mla_decode_schedule_bytes(dims) bytes).  Each request x head-group costs
 * its page count plus a fixed overhead; the total is cut into equal
 * contiguous ranges, one per CTA, so a long request is spread over several
 * CTAs and short ones share a CTA.  Recompute whenever cache_seqlens
 * changes; the plan can be reused by every layer of one decode step.
 * Clears the device status word. */
int mla_decode_get_schedule(const mla_decode_dims* dims, const int32_t* cache_seqlens,
                            void* schedule, void* stream);

/* The same plan computed on the host from host arrays (for inspection and
 * tests); `schedule_host` is host memory of mla_decode_schedule_bytes(dims)
 * bytes.  dims->num_sms must be > 0.  No CUDA call is made. */
int mla_decode_get_schedule_host(const mla_decode_dims* dims, const int32_t* cache_seqlens_host,
                                 void* schedule_host);

/* Decode attention.
 *   q            bf16 [batch][s_q][num_heads][576]
 *   kv_cache     bf16 [num_blocks][64][1][576]   (page pool; 73,728 B per page)
 *   block_table  int32 [batch][max_blocks_per_seq]: page ids; only the first
 *                ceil(L_b / 64) entries of row b are read
 *   cache_seqlens int32 [batch]: L_b, the cached length including the s_q new tokens
 *   softmax_scale scale applied to q.k (e.g. 192^-0.5)
 *   out          bf16 [batch][s_q][num_heads][512] (fp32 with MLA_FLAG_FP32_OUT)
 *   lse          fp32 [batch][num_heads][s_q]  (natural log; -inf if nothing is visible)
 *   schedule     from mla_decode_get_schedule with the same dims and lengths
 *                (with MLA_FLAG_INLINE_PLAN: any buffer of
 *                mla_decode_schedule_bytes(dims) bytes; the call writes the plan)
 *   workspace    mla_decode_workspace_bytes(dims) bytes, no initialisation needed
 * Enqueues the persistent decode kernel and then (unless MLA_FLAG_NO_COMBINE)
 * the combine kernel on `stream`.  A request whose visible range is empty
 * gets out = 0 and lse = -inf. */
int mla_decode_fwd(const mla_decode_dims* dims, void* schedule, void* workspace,
                   const void* q, const void* kv_cache, const int32_t* block_table,
                   const int32_t* cache_seqlens, float softmax_scale, void* out, float* lse,
                   void* stream);

/* LSE-weighted merge of the split partials left in `workspace` by
 * mla_decode_fwd: L* = log sum_i exp(lse_i), out = sum_i exp(lse_i - L*) O_i.
 * Also writes out = 0, lse = -inf for empty requests.  Requests that were not
 * split were already written by mla_decode_fwd and are not touched. */
int mla_decode_combine(const mla_decode_dims* dims, const void* schedule, const void* workspace,
                       void* out, float* lse, void* stream);

/* Copies the device status word (OR of MLA_STATUS_* bits since the last
 * mla_decode_get_schedule, including those of every MLA_FLAG_INLINE_PLAN call
 * since) to *host_status.  Synchronous: waits for the copy
 * on the legacy default stream, so call it after the work it should cover has
 * finished (e.g. after synchronising the stream that ran it). */
int mla_decode_get_status(const void* schedule, int32_t* host_status);

/* Static text for an MLA_* return code. */
const char* mla_decode_strerror(int code);

/* Allocation-free decode: schedule + decode + combine in one call, for callers
 * that cannot allocate device memory themselves -- for example a runtime or
 * plugin host that plans every device buffer ahead of time and gives a kernel
 * library no allocator, or a decode loop that cannot afford cudaMalloc's
 * implicit device synchronisation.  The pages describe no such entry point;
 * it exists for the library's users only.
 *
 * Arguments and results are those of mla_decode_fwd (dims->flags must not
 * contain MLA_FLAG_NO_COMBINE).  Instead of caller-provided schedule and
 * workspace buffers it uses one scratch array of MLA_NOALLOC_SCRATCH_BYTES
 * that the library declares in device memory; every GPU that loads the
 * library holds that array until the process exits.  Requests whose schedule
 * plus split partials would exceed it return MLA_ERR_SCRATCH_TOO_SMALL before
 * anything is enqueued; use mla_decode_fwd then.
 *   - No call allocates or frees device or host memory.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, cached per device); make that first call before
 *     any stream capture on that device.
 *   - All calls share the one array, and it keeps the previous call's
 *     contents (the schedule kernel rewrites the parts that must start fresh).
 *     Calls whose GPU work overlaps -- different streams without ordering,
 *     or several threads at once -- race on it and give wrong results;
 *     serialise them.
 *   - The device status word lives in the array and is not reported. */
#define MLA_NOALLOC_SCRATCH_BYTES (24u << 20)
int mla_decode_fwd_noalloc(const mla_decode_dims* dims, const void* q, const void* kv_cache,
                           const int32_t* block_table, const int32_t* cache_seqlens,
                           float softmax_scale, void* out, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * GQA-path decode over a group-expanded cache (GQLA technical summary,
 * gist.science, pt, 2605.15250, "Arquitetura", item 2 "Caminho GQA": the
 * latent is expanded into g groups of keys and values; the cache keeps the
 * per-group keys and values, 2 g d_h values per token, plus the shared RoPE
 * key; decode is grouped-query attention).  Same transposed kernel as the
 * MLA path (S^T = K Q^T, P^T = softmax over the KV axis, O^T = V^T P^T), with
 * K = [K_g | RoPE] (192 wide) and V = V_g (128 wide) per group.
 *
 *   q            bf16 [batch][s_q][num_q_heads][192]: per head its 128-wide
 *                group part, then its 64-wide RoPE part
 *   kv_cache     bf16 [num_blocks][64][2 * num_kv_groups * 128 + 64]: per
 *                token K_0 .. K_{g-1}, V_0 .. V_{g-1} (128 each), RoPE key (64)
 *   block_table, cache_seqlens, causal rule: as for mla_decode_fwd
 *   out          bf16 [batch][s_q][num_q_heads][128]
 *   lse          fp32 [batch][num_q_heads][s_q] (natural log)
 * Query head i reads group i / 16: num_q_heads must be 16 * num_kv_groups and
 * s_q 1 or 2; d_head 128, d_rope 64, page_size 64 (else MLA_ERR_UNSUPPORTED).
 * Errors, status word, schedule and workspace ownership, stream ordering and
 * MLA_FLAG_* as for the mla_decode_* calls above; the schedule and workspace
 * sizes come from the two _bytes calls below.  There is no allocation-free
 * variant.  Each (request, KV group) is one work item of the split-KV plan.
 * ---------------------------------------------------------------------- */
typedef struct mla_gqa_dims {
    int32_t batch;              /* B >= 1 */
    int32_t s_q;                /* 1 or 2 */
    int32_t num_q_heads;        /* 16 * num_kv_groups */
    int32_t num_kv_groups;      /* g >= 1 */
    int32_t num_blocks;         /* pages in the pool */
    int32_t max_blocks_per_seq; /* row stride of block_table */
    int32_t page_size;          /* must be 64 */
    int32_t d_head;             /* must be 128 */
    int32_t d_rope;             /* must be 64 */
    int32_t causal;             /* as in mla_decode_dims */
    int32_t num_sms;            /* persistent CTAs; 0 = the current device's SM count */
    int32_t flags;              /* MLA_FLAG_* */
} mla_gqa_dims;

size_t mla_gqa_decode_schedule_bytes(const mla_gqa_dims* dims);
size_t mla_gqa_decode_workspace_bytes(const mla_gqa_dims* dims);
int mla_gqa_decode_get_schedule(const mla_gqa_dims* dims, const int32_t* cache_seqlens, void* schedule,
                                void* stream);
/* The same GQA plan computed on the host from host arrays (for inspection and
 * tests); `schedule_host` is host memory of mla_gqa_decode_schedule_bytes(dims)
 * bytes.  dims->num_sms must be > 0.  No CUDA call is made. */
int mla_gqa_decode_get_schedule_host(const mla_gqa_dims* dims, const int32_t* cache_seqlens_host,
                                     void* schedule_host);
int mla_gqa_decode_fwd(const mla_gqa_dims* dims, void* schedule, void* workspace, const void* q,
                       const void* kv_cache, const int32_t* block_table, const int32_t* cache_seqlens,
                       float softmax_scale, void* out, float* lse, void* stream);
int mla_gqa_decode_combine(const mla_gqa_dims* dims, const void* schedule, const void* workspace, void* out,
                           float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Absorbed projections around the decode (GQLA technical summary,
 * gist.science, pt, 2605.15250, "Caminho MQA-Absorvido": the key and value
 * up-projections are absorbed into the query and output projections, so every
 * head attends to the 512-wide latent cache directly).  Per token t and head h:
 *
 *   mla_absorb_q:  q_out[t][h] = [ q_in[t][h][0:128] . w_uk[h]  |  q_in[t][h][128:192] ]
 *                  (512-wide latent query, then the 64-wide RoPE part unchanged:
 *                  exactly the q layout mla_decode_fwd takes)
 *   mla_absorb_o:  out[t][h]   =   o[t][h][0:512] . w_uv[h]
 *                  (the decode output over latent rows to the head's 128-wide
 *                  value space)
 *
 *   q_in   bf16 [tokens][num_heads][192]      w_uk  bf16 [num_heads][128][512]
 *   q_out  bf16 [tokens][num_heads][576]
 *   o      bf16 [tokens][num_heads][512]      w_uv  bf16 [num_heads][512][128]
 *   out    bf16 [tokens][num_heads][128]
 * All row-major and contiguous; tokens = batch * s_q.  Products accumulate in
 * fp32 and round once to bf16.  Every pointer is device memory owned by the
 * caller, 16-byte aligned; input and output must not overlap.  status is an
 * optional device int32 (NULL or 4-byte aligned) into which a kernel ORs
 * MLA_STATUS_TIMEOUT if one of its waits gave up (after ~1 s; the output is
 * then incomplete).  Work is enqueued on `stream` (NULL = legacy default);
 * nothing is allocated.  Returns MLA_ERR_INVALID_ARG for a NULL or
 * misaligned pointer, tokens outside [1, 4194240] or num_heads outside
 * [1, 65535]; MLA_ERR_UNSUPPORTED unless d_nope 128, d_rope 64, d_latent 512,
 * d_v_head 128; MLA_ERR_CUDA if a launch fails.
 * ---------------------------------------------------------------------- */
typedef struct mla_absorb_dims {
    int32_t tokens;    /* T >= 1 */
    int32_t num_heads; /* h >= 1 */
    int32_t d_nope;    /* must be 128 */
    int32_t d_rope;    /* must be 64 */
    int32_t d_latent;  /* must be 512 */
    int32_t d_v_head;  /* must be 128 */
} mla_absorb_dims;

int mla_absorb_q(const mla_absorb_dims* dims, const void* q_in, const void* w_uk, void* q_out,
                 int32_t* status, void* stream);
int mla_absorb_o(const mla_absorb_dims* dims, const void* o, const void* w_uv, void* out,
                 int32_t* status, void* stream);

/* ------------------------------------------------------------------------
 * Split-KV across GPUs: merge of per-rank decode results.  Each of R ranks
 * decodes the same queries against a disjoint part of every request's KV
 * (for example a contiguous range of its pages, held in that rank's own
 * pool); the ranks exchange their outputs and fp32 LSEs (an all-gather over
 * NVLink) and each merges them with this call (bf16 outputs) or with
 * mla_decode_combine_ranks_f32 (fp32 outputs):
 *
 *   L* = log sum_i exp(lse_i),  out = sum_i exp(lse_i - L*) o_i,  lse = L*
 *
 * (the same LSE-weighted merge mla_decode_combine applies to the split
 * partials inside one GPU).  A rank whose part is empty or fully masked
 * reports lse_i = -inf and weighs nothing; a row with every lse_i = -inf gets
 * out = 0 and lse = -inf.  For causal decode (s_q > 1), the rank that holds a
 * request's last tokens runs with causal = 1 and every other rank with
 * causal = 0: the causal rule only ever masks the request's last s_q - 1
 * positions.
 *
 *   o_parts    bf16 [num_ranks][batch][s_q][num_heads][d_v]  (rank-major
 *              stack of mla_decode_fwd / mla_gqa_decode_fwd outputs)
 *   lse_parts  fp32 [num_ranks][batch][num_heads][s_q]
 *   out        bf16 [batch][s_q][num_heads][d_v]
 *   lse        fp32 [batch][num_heads][s_q]
 * d_v is 512 (MLA path) or 128 (GQA path), else MLA_ERR_UNSUPPORTED.
 * 1 <= num_ranks <= 64; batch, s_q, num_heads >= 1; every pointer device
 * memory, 16-byte aligned, owned by the caller; out and lse must not overlap
 * the inputs (else MLA_ERR_INVALID_ARG / undefined).  Enqueued on `stream`
 * (NULL = legacy default); nothing is allocated.  Accumulates in fp32 and
 * rounds once to bf16.
 * ---------------------------------------------------------------------- */
int mla_decode_combine_ranks(int32_t num_ranks, int32_t batch, int32_t s_q, int32_t num_heads, int32_t d_v,
                             const void* o_parts, const float* lse_parts, void* out, float* lse,
                             void* stream);

/* The same merge of fp32 per-rank results: o_parts fp32 [num_ranks][batch]
 * [s_q][num_heads][d_v], as mla_decode_fwd / mla_gqa_decode_fwd write them
 * with MLA_FLAG_FP32_OUT.  The merged row is rounded to bf16 once, as the
 * combine of split partials inside one GPU does; exchanging bf16 outputs
 * instead rounds each rank's result first.  Other arguments and errors as
 * for mla_decode_combine_ranks. */
int mla_decode_combine_ranks_f32(int32_t num_ranks, int32_t batch, int32_t s_q, int32_t num_heads,
                                 int32_t d_v, const float* o_parts, const float* lse_parts, void* out,
                                 float* lse, void* stream);

/* Library ABI version (increments on any change of these declarations). */
int mla_decode_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
