/*
 * Plain, slow, fp64 CPU oracle for paged decode attention and the slot-mapped
 * KV write.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * bench's CPU-baseline leg call it; the product path never does.  It shares
 * no code, header or helper with the CUDA library.
 *
 * Sources (web pages on vLLM / PagedAttention):
 *  [P3] "4. vLLM核心机制：PagedAttention、Continuous Batching、动态批处理",
 *       section 4.2: the KV cache is cut into fixed-size pages of 16 or 32
 *       tokens; a per-request page table maps logical page i to a physical
 *       page anywhere in the pool (worked example: logical 0,1,2 -> physical
 *       7,2,5); attention looks the pages up one by one through the table and
 *       never assumes the K/V rows are contiguous; pages of a shared prefix
 *       may be named by several requests' tables.
 *       Section 4.3: each decode iteration produces the new token together
 *       with the updated KV cache.
 *  [P1] "vLLM：大型语言模型推理优化的革命性突破", section 2.1: the attention
 *       kernel indexes the scattered blocks through the table with no data
 *       movement and no zero padding, i.e. the result is ordinary attention
 *       over the logical sequence.
 *  [P2] pinggu.org forum post, section "PagedAttention：让显存像虚拟内存一样灵活":
 *       a page holds a fixed number of tokens (16 by default) and logical
 *       continuity is separated from physical placement.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - cache layout [num_blocks][num_kv_heads][block_size][head_dim];
 *  - query head hq reads kv head hq / (num_q_heads / num_kv_heads);
 *  - context_lens[s] counts every token the step attends to, including the
 *    one written by this step's KV write;
 *  - a negative slot in the slot mapping means "write nothing";
 *  - a sequence with context length 0 yields an all-zero output row.
 *
 * Storage elements are IEEE binary16 (dtype 1) or bfloat16 (dtype 2) bit
 * patterns; they are widened to double here from their format definitions.
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
#define ORACLE_ERR_BLOCK_ID -2
#define ORACLE_ERR_SLOT -3
#define ORACLE_ERR_CONTEXT -4
#define ORACLE_ERR_NOMEM -5

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        mag = f ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(f + 1024), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return (double)x;
}

static double widen(uint16_t bits, int dtype) {
    return dtype == 2 ? oracle_bf16_to_double(bits) : oracle_half_to_double(bits);
}

/*
 * KV write ([P3] section 4.3): for every new token t and kv head h, the
 * slot s = slot_mapping[t] names physical block s / block_size and row
 * s % block_size; k[t][h][:] and v[t][h][:] are copied there bit for bit.
 * k, v: [num_tokens][num_kv_heads][head_dim]; caches as in the layout above.
 */
int oracle_write_kv(const uint16_t *k, const uint16_t *v, uint16_t *k_cache, uint16_t *v_cache,
                    const int64_t *slot_mapping, int64_t num_tokens, int64_t num_kv_heads,
                    int64_t head_dim, int64_t block_size, int64_t num_blocks) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return ORACLE_ERR_ARG;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) return ORACLE_ERR_SLOT;
        int64_t block = slot / block_size;
        int64_t row = slot % block_size;
        for (int64_t h = 0; h < num_kv_heads; ++h) {
            for (int64_t i = 0; i < head_dim; ++i) {
                int64_t src = (t * num_kv_heads + h) * head_dim + i;
                int64_t dst = ((block * num_kv_heads + h) * block_size + row) * head_dim + i;
                k_cache[dst] = k[src];
                v_cache[dst] = v[src];
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Step 1 of both attention functions ([P3] section 4.2): the L logical tokens
 * of one sequence and kv head h, gathered through its page-table row: token j
 * lives in physical block table_row[j / block_size], row j % block_size.
 * Writes contiguous K[L][d] and V[L][d].
 */
static void gather_rows(const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *table_row, int64_t L,
                        int64_t h, int64_t num_kv_heads, int64_t head_dim, int64_t block_size, int dtype,
                        double *K, double *V) {
    for (int64_t j = 0; j < L; ++j) {
        int64_t p = table_row[j / block_size];
        int64_t row = j % block_size;
        const uint16_t *kr = k_cache + ((p * num_kv_heads + h) * block_size + row) * head_dim;
        const uint16_t *vr = v_cache + ((p * num_kv_heads + h) * block_size + row) * head_dim;
        for (int64_t i = 0; i < head_dim; ++i) {
            K[j * head_dim + i] = widen(kr[i], dtype);
            V[j * head_dim + i] = widen(vr[i], dtype);
        }
    }
}

/*
 * Steps 2-4 for one query row qr over the first `count` gathered tokens
 * ([P1] section 2.1: plain attention over the logical tokens):
 *   z_j = scale * sum_i q[i] * K[j][i];  w_j = exp(z_j - max_j z_j);
 *   o[i] += sum_j (w_j / sum_j w_j) * V[j][i].
 * z is scratch of `count` doubles; o must hold zeros on entry.
 */
static void attend(const uint16_t *qr, const double *K, const double *V, int64_t count, int64_t head_dim,
                   int dtype, double scale, double *z, double *o) {
    for (int64_t j = 0; j < count; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < head_dim; ++i) acc += widen(qr[i], dtype) * K[j * head_dim + i];
        z[j] = scale * acc;
    }
    double m = z[0];
    for (int64_t j = 1; j < count; ++j)
        if (z[j] > m) m = z[j];
    double Z = 0.0;
    for (int64_t j = 0; j < count; ++j) {
        z[j] = exp(z[j] - m);
        Z += z[j];
    }
    for (int64_t j = 0; j < count; ++j) {
        double w = z[j] / Z;
        for (int64_t i = 0; i < head_dim; ++i) o[i] += w * V[j * head_dim + i];
    }
}

/*
 * Decode attention for one new query token per sequence.  For sequence s and
 * query head hq (kv head h = hq / group), gather the L = context_lens[s]
 * tokens (step 1) and attend over all of them (steps 2-4).
 * q: [num_seqs][num_q_heads][head_dim]; block_tables: [num_seqs][table_stride];
 * out: [num_seqs][num_q_heads][head_dim] doubles.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *block_tables, int64_t table_stride, const int32_t *context_lens,
                  int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                  int64_t block_size, int64_t num_blocks, int dtype, double scale, double *out) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_q_heads % num_kv_heads != 0 || (dtype != 1 && dtype != 2))
        return ORACLE_ERR_ARG;
    int64_t group = num_q_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t L = context_lens[s];
        if (L < 0 || L > table_stride * block_size) return ORACLE_ERR_CONTEXT;
        for (int64_t j = 0; j < L; j += block_size) {
            int32_t p = block_tables[s * table_stride + j / block_size];
            if (p < 0 || p >= num_blocks) return ORACLE_ERR_BLOCK_ID;
        }
    }
    double *K = NULL, *V = NULL, *z = NULL;
    int rc = ORACLE_OK;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t L = context_lens[s];
        if (L > 0) {
            K = (double *)malloc((size_t)(L * head_dim) * sizeof(double));
            V = (double *)malloc((size_t)(L * head_dim) * sizeof(double));
            z = (double *)malloc((size_t)L * sizeof(double));
            if (!K || !V || !z) { rc = ORACLE_ERR_NOMEM; goto done; }
        }
        for (int64_t hq = 0; hq < num_q_heads; ++hq) {
            int64_t h = hq / group;
            double *o = out + (s * num_q_heads + hq) * head_dim;
            for (int64_t i = 0; i < head_dim; ++i) o[i] = 0.0;
            if (L == 0) continue;
            gather_rows(k_cache, v_cache, block_tables + s * table_stride, L, h, num_kv_heads, head_dim,
                        block_size, dtype, K, V);
            attend(q + (s * num_q_heads + hq) * head_dim, K, V, L, head_dim, dtype, scale, z, o);
        }
        free(K); free(V); free(z);
        K = V = z = NULL;
    }
done:
    free(K); free(V); free(z);
    return rc;
}

/*
 * The same decode, with the (sequence, query head) pairs shared among the
 * host's cores by OpenMP when this file is compiled with -fopenmp (without
 * it the pragmas are ignored and the loop runs on one thread).  Each pair
 * runs exactly the steps of oracle_decode -- gather through the table, then
 * attend -- on buffers private to its thread, so the results are identical
 * to oracle_decode's, bit for bit, whatever the thread count.  Used only to
 * time the oracle on every core; the checks of the GPU path use
 * oracle_decode.
 */
int oracle_decode_parallel(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *block_tables, int64_t table_stride, const int32_t *context_lens,
                           int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                           int64_t block_size, int64_t num_blocks, int dtype, double scale, double *out) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_q_heads % num_kv_heads != 0 || (dtype != 1 && dtype != 2))
        return ORACLE_ERR_ARG;
    int64_t max_len = 0;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t L = context_lens[s];
        if (L < 0 || L > table_stride * block_size) return ORACLE_ERR_CONTEXT;
        for (int64_t j = 0; j < L; j += block_size) {
            int32_t p = block_tables[s * table_stride + j / block_size];
            if (p < 0 || p >= num_blocks) return ORACLE_ERR_BLOCK_ID;
        }
        if (L > max_len) max_len = L;
    }
    int64_t group = num_q_heads / num_kv_heads;
    int64_t pairs = num_seqs * num_q_heads;
    int rc = ORACLE_OK;
#pragma omp parallel
    {
        size_t cap = (size_t)(max_len > 0 ? max_len : 1);
        double *K = (double *)malloc(cap * (size_t)head_dim * sizeof(double));
        double *V = (double *)malloc(cap * (size_t)head_dim * sizeof(double));
        double *z = (double *)malloc(cap * sizeof(double));
        int ok = K && V && z;
        if (!ok) {
#pragma omp atomic write
            rc = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < pairs; ++u) {
            int64_t s = u / num_q_heads, hq = u % num_q_heads;
            int64_t L = context_lens[s];
            double *o = out + (s * num_q_heads + hq) * head_dim;
            for (int64_t i = 0; i < head_dim; ++i) o[i] = 0.0;
            if (L == 0 || !ok) continue;
            const uint16_t *qrow = q + u * head_dim;  /* u = s * num_q_heads + hq */
            gather_rows(k_cache, v_cache, block_tables + s * table_stride, L, hq / group, num_kv_heads, head_dim,
                        block_size, dtype, K, V);
            attend(qrow, K, V, L, head_dim, dtype, scale, z, o);
        }
        free(K); free(V); free(z);
    }
    return rc;
}

/* Threads oracle_decode_parallel uses (1 when compiled without OpenMP). */
int oracle_parallel_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Block copy ([P3] section 4.2: pages of a shared prefix are named by several
 * tables; a sequence about to append to a shared, partly filled page first
 * gets a private copy of it -- copy-on-write -- and section 4.4: preemption
 * moves a sequence's pages to a CPU-side pool and back).  For every pair i,
 * block mapping[i][0] of the source pool is copied, all kv heads, rows and
 * dims, to block mapping[i][1] of the destination pool (which may be the
 * same pool).  A pair with a negative entry is skipped.  Pools:
 * [num_blocks][num_kv_heads][block_size][head_dim] 2-byte elements.
 */
int oracle_copy_blocks(const uint16_t *src_k, const uint16_t *src_v, uint16_t *dst_k, uint16_t *dst_v,
                       const int64_t *mapping, int64_t num_pairs, int64_t num_kv_heads, int64_t block_size,
                       int64_t head_dim, int64_t src_blocks, int64_t dst_blocks) {
    if (num_pairs < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0) return ORACLE_ERR_ARG;
    const int64_t per_block = num_kv_heads * block_size * head_dim;
    for (int64_t i = 0; i < num_pairs; ++i) {
        const int64_t src = mapping[2 * i], dst = mapping[2 * i + 1];
        if (src < 0 || dst < 0) continue;
        if (src >= src_blocks || dst >= dst_blocks) return ORACLE_ERR_BLOCK_ID;
        for (int64_t e = 0; e < per_block; ++e) {
            dst_k[dst * per_block + e] = src_k[src * per_block + e];
            dst_v[dst * per_block + e] = src_v[src * per_block + e];
        }
    }
    return ORACLE_OK;
}

/*
 * Prefill / chunked prefill through the page table ([P3] section 4.3: the
 * prompt's tokens enter the cache before decoding starts, and a long prompt
 * may be processed in pieces across iterations).  Sequence s brings
 * n = query_start[s+1] - query_start[s] new query tokens; its K/V rows for
 * all L = context_lens[s] tokens, the new ones included, are already in the
 * paged cache.  New token t sits at logical position pos = L - n + t and
 * attends causally to tokens 0..pos: steps 1-4 of decode with the first
 * pos + 1 gathered tokens.  With n = 1 this is exactly decode.
 * q, out: [total_new_tokens][num_q_heads][head_dim], token-major.
 */
int oracle_prefill(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                   const int32_t *block_tables, int64_t table_stride, const int32_t *query_start,
                   const int32_t *context_lens, int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                   int64_t head_dim, int64_t block_size, int64_t num_blocks, int dtype, double scale,
                   double *out) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_q_heads % num_kv_heads != 0 || (dtype != 1 && dtype != 2))
        return ORACLE_ERR_ARG;
    if (num_seqs > 0 && query_start[0] != 0) return ORACLE_ERR_ARG;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t n = (int64_t)query_start[s + 1] - query_start[s];
        int64_t L = context_lens[s];
        if (n < 0) return ORACLE_ERR_ARG;
        if (L < n || L > table_stride * block_size) return ORACLE_ERR_CONTEXT;
        for (int64_t j = 0; j < L; j += block_size) {
            int32_t p = block_tables[s * table_stride + j / block_size];
            if (p < 0 || p >= num_blocks) return ORACLE_ERR_BLOCK_ID;
        }
    }
    int64_t group = num_q_heads / num_kv_heads;
    double *K = NULL, *V = NULL, *z = NULL;
    int rc = ORACLE_OK;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t n = (int64_t)query_start[s + 1] - query_start[s];
        int64_t L = context_lens[s];
        if (n == 0) continue;
        K = (double *)malloc((size_t)(L * head_dim) * sizeof(double));
        V = (double *)malloc((size_t)(L * head_dim) * sizeof(double));
        z = (double *)malloc((size_t)L * sizeof(double));
        if (!K || !V || !z) { rc = ORACLE_ERR_NOMEM; goto done; }
        for (int64_t h = 0; h < num_kv_heads; ++h) {
            gather_rows(k_cache, v_cache, block_tables + s * table_stride, L, h, num_kv_heads, head_dim,
                        block_size, dtype, K, V);
            for (int64_t hq = h * group; hq < (h + 1) * group; ++hq) {
                for (int64_t t = 0; t < n; ++t) {
                    int64_t pos = L - n + t;
                    int64_t tok = query_start[s] + t;
                    double *o = out + (tok * num_q_heads + hq) * head_dim;
                    for (int64_t i = 0; i < head_dim; ++i) o[i] = 0.0;
                    attend(q + (tok * num_q_heads + hq) * head_dim, K, V, pos + 1, head_dim, dtype, scale, z, o);
                }
            }
        }
        free(K); free(V); free(z);
        K = V = z = NULL;
    }
done:
    free(K); free(V); free(z);
    return rc;
}
