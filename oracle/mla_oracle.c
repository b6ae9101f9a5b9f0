/*
 * fp64 CPU oracle for absorbed-MQA MLA decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this file or
 * the library built from it: only tests/, __graft_entry__.smoke() and the CPU
 * baseline / reference arm of bench.py may.  It shares no code, header, table
 * or helper with the CUDA library.
 *
 * What it computes is the plain, non-transposed definition of one decode
 * attention step, evaluated in double precision:
 *
 *   for every request b, new-token index s in [0, s_q) and query head h:
 *     L_vis = L_b - s_q + 1 + s   if causal and s_q > 1, else L_b
 *     z_t   = scale * sum_{c < d_qk} q[b,s,h,c] * row_t[c]        t < L_vis
 *     m     = max_t z_t,   l = sum_t exp(z_t - m)
 *     O[c]  = sum_t exp(z_t - m) * row_t[c] / l                    c < d_v
 *     LSE   = m + log(l)          (natural log)
 *   with row_t = kv[block_table[b][t / page_size]][t % page_size][:].
 *
 * Sources (web pages on FlashMLA-ETAP and GQLA):
 *  - FlashMLA-ETAP technical summary (gist.science, pt, 2506.01969),
 *    section "Mecanismo Central": the standard flow S = Q K^T, P = softmax(S),
 *    O = P V, of which the transposed pipeline is an exact re-arrangement.
 *  - GQLA technical summary (gist.science, pt, 2605.15250), section
 *    "Caminho MQA-Absorvido": every query head attends directly to the shared
 *    compact latent cache, which stores the latent plus one shared RoPE key.
 *    The full row (latent + RoPE key) is the key; the latent (the first d_v
 *    columns) is the value.
 *  - FlashMLA-ETAP technical summary, "Estabilidade Numérica": accuracy is
 *    measured against a double-precision reference, which this is.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): the causal rule for s_q > 1 above; an empty visible range gives
 * O = 0 and LSE = -inf; no epsilon is added to l; LSE is the natural log.
 *
 * The file also holds gqa_oracle_fwd (at the end): the GQLA "GQA path" over a
 * group-expanded cache, pinned in tests/test_oracle_gqa.py.
 *
 * Inputs are either fp64 arrays or bf16 bit patterns (uint16), converted to
 * double exactly.  Parallelism: OpenMP over query rows only; the arithmetic
 * inside a row is a plain sequential loop in token order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_BLOCK_TABLE -2
#define ORACLE_ERR_NOMEM -3

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, size_t i, int is_bf16) {
    if (is_bf16) return bf16_bits_to_double(((const uint16_t*)base)[i]);
    return ((const double*)base)[i];
}

int mla_oracle_version(void) { return 1; }

/*
 * q            [batch][s_q][num_heads][d_qk]            (fp64 or bf16 bits)
 * kv           [num_blocks][page_size][d_qk]            (fp64 or bf16 bits)
 * block_table  [batch][max_blocks_per_seq]  int32
 * cache_seqlens[batch]                      int32
 * rows         optional list of flattened query rows r = (b*s_q + s)*num_heads + h;
 *              NULL means every row in that order
 * out          [num_rows][d_v]    lse [num_rows]
 * probs        optional [num_rows][probs_stride]: P_t for t < L_vis (tiny cases)
 */
int mla_oracle_fwd(int batch, int s_q, int num_heads, int d_qk, int d_v, int page_size,
                   int causal, int max_blocks_per_seq, long long num_blocks,
                   const void* q, const void* kv, int inputs_are_bf16,
                   const int32_t* block_table, const int32_t* cache_seqlens,
                   double softmax_scale,
                   const int32_t* rows, int num_rows,
                   double* out, double* lse,
                   double* probs, long long probs_stride,
                   int num_threads) {
    if (batch < 0 || s_q < 1 || num_heads < 1 || d_qk < 1 || d_v < 1 || d_v > d_qk ||
        page_size < 1 || max_blocks_per_seq < 0 || num_blocks < 0 || !q || !kv ||
        !block_table || !cache_seqlens || !out || !lse)
        return ORACLE_ERR_ARG;
    const long long total_rows = (long long)batch * s_q * num_heads;
    long long nr = rows ? (long long)num_rows : total_rows;
    if (rows) {
        for (long long i = 0; i < nr; ++i)
            if (rows[i] < 0 || rows[i] >= total_rows) return ORACLE_ERR_ARG;
    }
    for (int b = 0; b < batch; ++b) {
        int L = cache_seqlens[b];
        if (L < 0) return ORACLE_ERR_ARG;
        long long pages = ((long long)L + page_size - 1) / page_size;
        if (pages > max_blocks_per_seq) return ORACLE_ERR_BLOCK_TABLE;
        for (long long j = 0; j < pages; ++j) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + j];
            if (phys < 0 || phys >= num_blocks) return ORACLE_ERR_BLOCK_TABLE;
        }
    }
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#endif
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = 0; i < nr; ++i) {
        long long r = rows ? rows[i] : i;
        int h = (int)(r % num_heads);
        int s = (int)((r / num_heads) % s_q);
        int b = (int)(r / ((long long)num_heads * s_q));
        int L = cache_seqlens[b];
        long long Lvis = (causal && s_q > 1) ? (long long)L - s_q + 1 + s : (long long)L;
        if (Lvis < 0) Lvis = 0;
        double* o = out + (size_t)i * d_v;
        for (int c = 0; c < d_v; ++c) o[c] = 0.0;
        if (Lvis == 0) {
            lse[i] = -INFINITY;
            continue;
        }
        double* z = (double*)malloc((size_t)Lvis * sizeof(double));
        if (!z) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        const size_t q_off = (size_t)r * d_qk;
        /* scores */
        for (long long t = 0; t < Lvis; ++t) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + t / page_size];
            size_t row_off = ((size_t)phys * page_size + (size_t)(t % page_size)) * d_qk;
            double acc = 0.0;
            for (int c = 0; c < d_qk; ++c)
                acc += load_elem(q, q_off + c, inputs_are_bf16) * load_elem(kv, row_off + c, inputs_are_bf16);
            z[t] = softmax_scale * acc;
        }
        /* softmax statistics */
        double m = z[0];
        for (long long t = 1; t < Lvis; ++t)
            if (z[t] > m) m = z[t];
        double l = 0.0;
        for (long long t = 0; t < Lvis; ++t) l += exp(z[t] - m);
        /* weighted sum of the value columns (the first d_v columns of each row) */
        for (long long t = 0; t < Lvis; ++t) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + t / page_size];
            size_t row_off = ((size_t)phys * page_size + (size_t)(t % page_size)) * d_qk;
            double w = exp(z[t] - m);
            for (int c = 0; c < d_v; ++c) o[c] += w * load_elem(kv, row_off + c, inputs_are_bf16);
        }
        for (int c = 0; c < d_v; ++c) o[c] /= l;
        lse[i] = m + log(l);
        if (probs) {
            double* p = probs + (size_t)i * (size_t)probs_stride;
            for (long long t = 0; t < Lvis && t < probs_stride; ++t) p[t] = exp(z[t] - m) / l;
        }
        free(z);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

int mla_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * GQA-path decode over a group-expanded cache, fp64 (GQLA technical summary,
 * gist.science, pt, 2605.15250, section "Arquitetura", item 2 "Caminho GQA":
 * the latent is expanded into g groups of keys and values, the cache keeps the
 * per-group keys and values (2 g d_h per token) plus the shared RoPE key, and
 * decode is standard grouped-query attention).  TEST INFRASTRUCTURE ONLY, like
 * the rest of this file.
 *
 *   q      [batch][s_q][num_q_heads][d_head + d_rope]   (query head i, its
 *          group part then its RoPE part)
 *   kv     [num_blocks][page_size][2 * groups * d_head + d_rope]: per token
 *          K_0 .. K_{g-1} (d_head each), V_0 .. V_{g-1} (d_head each), then
 *          the shared RoPE key (d_rope)
 *   head i belongs to group k = i / (num_q_heads / groups)
 *   z_t  = scale * (<q_i[0:d_head], K_k[t]> + <q_i[d_head:], rope[t]>)
 *   O_i  = sum_t softmax(z)_t * V_k[t]   (d_head wide),  LSE = m + log l
 * with the same visible range and empty-range rule as mla_oracle_fwd.
 * out [num_rows][d_head], lse [num_rows]; rows as in mla_oracle_fwd.
 */
int gqa_oracle_fwd(int batch, int s_q, int num_q_heads, int groups, int d_head, int d_rope,
                   int page_size, int causal, int max_blocks_per_seq, long long num_blocks,
                   const void* q, const void* kv, int inputs_are_bf16,
                   const int32_t* block_table, const int32_t* cache_seqlens,
                   double softmax_scale, const int32_t* rows, int num_rows,
                   double* out, double* lse, int num_threads) {
    if (batch < 0 || s_q < 1 || num_q_heads < 1 || groups < 1 || num_q_heads % groups != 0 ||
        d_head < 1 || d_rope < 0 || page_size < 1 || max_blocks_per_seq < 0 || num_blocks < 0 || !q ||
        !kv || !block_table || !cache_seqlens || !out || !lse)
        return ORACLE_ERR_ARG;
    const int d_q = d_head + d_rope;
    const long long row_w = 2LL * groups * d_head + d_rope;
    const int heads_per_group = num_q_heads / groups;
    const long long total_rows = (long long)batch * s_q * num_q_heads;
    long long nr = rows ? (long long)num_rows : total_rows;
    if (rows) {
        for (long long i = 0; i < nr; ++i)
            if (rows[i] < 0 || rows[i] >= total_rows) return ORACLE_ERR_ARG;
    }
    for (int b = 0; b < batch; ++b) {
        int L = cache_seqlens[b];
        if (L < 0) return ORACLE_ERR_ARG;
        long long pages = ((long long)L + page_size - 1) / page_size;
        if (pages > max_blocks_per_seq) return ORACLE_ERR_BLOCK_TABLE;
        for (long long j = 0; j < pages; ++j) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + j];
            if (phys < 0 || phys >= num_blocks) return ORACLE_ERR_BLOCK_TABLE;
        }
    }
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#endif
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = 0; i < nr; ++i) {
        long long r = rows ? rows[i] : i;
        int h = (int)(r % num_q_heads);
        int s = (int)((r / num_q_heads) % s_q);
        int b = (int)(r / ((long long)num_q_heads * s_q));
        int k = h / heads_per_group;
        int L = cache_seqlens[b];
        long long Lvis = (causal && s_q > 1) ? (long long)L - s_q + 1 + s : (long long)L;
        if (Lvis < 0) Lvis = 0;
        double* o = out + (size_t)i * d_head;
        for (int c = 0; c < d_head; ++c) o[c] = 0.0;
        if (Lvis == 0) {
            lse[i] = -INFINITY;
            continue;
        }
        double* z = (double*)malloc((size_t)Lvis * sizeof(double));
        if (!z) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        const size_t q_off = (size_t)r * d_q;
        const size_t k_col = (size_t)k * d_head;                            /* K_k */
        const size_t v_col = (size_t)groups * d_head + (size_t)k * d_head;  /* V_k */
        const size_t r_col = (size_t)2 * groups * d_head;                   /* shared RoPE key */
        for (long long t = 0; t < Lvis; ++t) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + t / page_size];
            size_t row_off = ((size_t)phys * page_size + (size_t)(t % page_size)) * (size_t)row_w;
            double acc = 0.0;
            for (int c = 0; c < d_head; ++c)
                acc += load_elem(q, q_off + c, inputs_are_bf16) * load_elem(kv, row_off + k_col + c, inputs_are_bf16);
            for (int c = 0; c < d_rope; ++c)
                acc += load_elem(q, q_off + d_head + c, inputs_are_bf16) *
                       load_elem(kv, row_off + r_col + c, inputs_are_bf16);
            z[t] = softmax_scale * acc;
        }
        double m = z[0];
        for (long long t = 1; t < Lvis; ++t)
            if (z[t] > m) m = z[t];
        double l = 0.0;
        for (long long t = 0; t < Lvis; ++t) l += exp(z[t] - m);
        for (long long t = 0; t < Lvis; ++t) {
            int phys = block_table[(size_t)b * max_blocks_per_seq + t / page_size];
            size_t row_off = ((size_t)phys * page_size + (size_t)(t % page_size)) * (size_t)row_w;
            double w = exp(z[t] - m);
            for (int c = 0; c < d_head; ++c) o[c] += w * load_elem(kv, row_off + v_col + c, inputs_are_bf16);
        }
        for (int c = 0; c < d_head; ++c) o[c] /= l;
        lse[i] = m + log(l);
        free(z);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
