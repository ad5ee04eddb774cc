/*
 * pkv_oracle.c -- plain, slow CPU oracle for paged attention over a block-pooled KV cache.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference arm may load this file's library. The product library shares no code, header,
 * table or helper with it, and never calls it.
 *
 * Sources (page title, section):
 *   [P1] blog.mckayzhao.com/?p=56
 *        "PagedAttention：操作系统课本里翻出来的灵感" -- 16-token KV blocks, block table as a
 *        logical->physical map, the kernel reads K and V block by block through the table and the
 *        result equals contiguous storage; a sequence of N tokens needs ceil(N/block_size) blocks and
 *        wastes at most block_size-1 slots.
 *        "还不止是分页：Copy-on-Write 和内存共享" -- shared blocks, reference counts, copy-on-write:
 *        copy the block, modify the copy, leave the original unchanged.
 *        "进阶特性：让推理再快一点" / "V1 架构：推倒重来的勇气" -- chunked prefill; one mixed batch
 *        described by {request_id: num_tokens}.
 *   [P3] 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？
 *        "快速回顾 prefill、decode 和 KV cache" -- every processed token appends one K/V entry.
 *        "PagedAttention：核心思路" (block-pool figure) -- a pool of equal blocks, one table per request.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - pool layout [num_blocks][num_kv_heads][block_size][head_dim], K and V in separate pools;
 *   - query row j of a request with n rows and context ctx sits at position ctx-n+j and attends
 *     keys 0..ctx-n+j (causal inside the chunk, everything before it);
 *   - grouped query heads: query head h reads KV head h / (Hq/Hkv);
 *   - softmax(scale * q.k) with the maximum subtracted, in double precision.
 *
 * Arithmetic is double throughout. Inputs are decoded from their storage type by the small
 * decoders below, written from the IEEE-754 binary16 and bfloat16 definitions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Storage type codes for q, k, v. */
enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

/* Error codes returned by the oracle (0 = ok). */
enum { ORACLE_OK = 0, ORACLE_BAD_ARG = -1, ORACLE_BAD_TABLE = -2, ORACLE_NO_MEM = -3 };

int oracle_elem_bytes(int dtype) { return dtype == ORACLE_F32 ? 4 : 2; }

/* binary16: 1 sign bit, 5 exponent bits with bias 15, 10 fraction bits. */
double oracle_half_to_double(uint16_t h) {
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
#ifdef ORACLE_MUTANT_HALF_BIAS
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(f | 0x400), e - 24);
#else
    if (e == 0) v = ldexp((double)f, -24);                 /* subnormal: f * 2^(1-15-10) */
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(f | 0x400), e - 25);           /* (2^10 + f) * 2^(e-15-10) */
#endif
    return sign ? -v : v;
}

/* bfloat16 is the upper 16 bits of a binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, int64_t i, int dtype) {
    if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
    uint16_t bits = ((const uint16_t*)base)[i];
    return dtype == ORACLE_F16 ? oracle_half_to_double(bits) : oracle_bf16_to_double(bits);
}

/* [P1] "PagedAttention：操作系统课本里翻出来的灵感": N tokens occupy ceil(N / block_size) blocks. */
int64_t oracle_blocks_for_tokens(int64_t n, int block_size) {
    if (n <= 0) return 0;
    return (n + block_size - 1) / block_size;
}

/* Same section: the only waste is the unused tail of the last block (at most block_size - 1). */
int64_t oracle_wasted_slots(int64_t n, int block_size) {
    return oracle_blocks_for_tokens(n, block_size) * (int64_t)block_size - n;
}

/*
 * Slot of each new token ([P3] "快速回顾 prefill、decode 和 KV cache": each token appends one entry;
 * [P1] block table = logical -> physical map). Request r contributes n_r = qsl[r+1]-qsl[r] tokens at
 * positions ctx_r - n_r + j; the slot is physical_block * block_size + offset inside the block.
 */
int oracle_slot_mapping(const int32_t* block_tables, int max_blocks, const int32_t* query_start_loc,
                        const int32_t* context_lens, int num_reqs, int block_size, int64_t* slots) {
    for (int r = 0; r < num_reqs; ++r) {
        int n = query_start_loc[r + 1] - query_start_loc[r];
        int ctx = context_lens[r];
        if (n < 0 || ctx < n) return ORACLE_BAD_ARG;
        for (int j = 0; j < n; ++j) {
#ifdef ORACLE_MUTANT_SLOT_POS
            int64_t pos = (int64_t)ctx - n + j - 1;
            if (pos < 0) pos = 0;
#else
            int64_t pos = (int64_t)ctx - n + j;
#endif
            int64_t logical_block = pos / block_size;
            if (logical_block >= max_blocks) return ORACLE_BAD_TABLE;
            int64_t phys = block_tables[(int64_t)r * max_blocks + logical_block];
            slots[query_start_loc[r] + j] = phys * block_size + pos % block_size;
        }
    }
    return ORACLE_OK;
}

/*
 * Append new K/V rows into their slots, in token order; slot < 0 means "skip".
 * new: [T][Hkv][D]; pool: [NB][Hkv][block_size][D]; elements are copied as raw bytes.
 */
int oracle_kv_cache_write(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                          const int64_t* slots, int num_tokens, int num_blocks, int num_kv_heads,
                          int head_dim, int block_size, int elem_bytes) {
    const int64_t row = (int64_t)head_dim * elem_bytes;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slots[t];
        if (slot < 0) continue;
        int64_t blk = slot / block_size, off = slot % block_size;
        if (blk >= num_blocks) return ORACLE_BAD_TABLE;
        for (int h = 0; h < num_kv_heads; ++h) {
#ifdef ORACLE_MUTANT_WRITE_OFFSET
            int64_t dst = ((blk * num_kv_heads + h) * block_size + (off + 1) % block_size) * row;
#else
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row;
#endif
            int64_t src = ((int64_t)t * num_kv_heads + h) * row;
            memcpy((char*)k_pool + dst, (const char*)k_new + src, (size_t)row);
            memcpy((char*)v_pool + dst, (const char*)v_new + src, (size_t)row);
        }
    }
    return ORACLE_OK;
}

/*
 * Copy-on-write block copy ([P1] "还不止是分页：Copy-on-Write 和内存共享"): for every layer and every
 * (src, dst) pair, in pair order, the whole K block and the whole V block (all KV heads) of src are
 * copied onto dst. pairs: [num_pairs][2] = (src, dst).
 */
int oracle_copy_blocks(void* const* k_pools, void* const* v_pools, int num_layers, const int32_t* pairs,
                       int num_pairs, int num_blocks, int num_kv_heads, int head_dim, int block_size,
                       int elem_bytes) {
    const int64_t blk_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes;
    for (int l = 0; l < num_layers; ++l) {
        for (int p = 0; p < num_pairs; ++p) {
            int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
            if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) return ORACLE_BAD_TABLE;
            if (src == dst) continue;
            memcpy((char*)k_pools[l] + dst * blk_bytes, (const char*)k_pools[l] + src * blk_bytes, (size_t)blk_bytes);
#ifndef ORACLE_MUTANT_COPY_K_ONLY
            memcpy((char*)v_pools[l] + dst * blk_bytes, (const char*)v_pools[l] + src * blk_bytes, (size_t)blk_bytes);
#endif
        }
    }
    return ORACLE_OK;
}

/* Request that owns query row `row` (query_start_loc is non-decreasing). */
static int request_of_row(const int32_t* qsl, int num_reqs, int row) {
    int lo = 0, hi = num_reqs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (qsl[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/*
 * Paged attention for the rows of one mixed batch ([P1] "V1 架构：推倒重来的勇气": one batch holds
 * decode rows and chunked-prefill rows, keyed {request_id: num_tokens}).
 *
 * For query row `row` of request r (n = qsl[r+1]-qsl[r] rows, prior P = ctx_r - n, j = row - qsl[r]):
 *   K_r[t] = k_pool[bt[r][t / bs]][g][t % bs][:], g = h / (Hq/Hkv)     (read through the table, [P1])
 *   s_t    = scale * sum_d q[row][h][d] * K_r[t][d]                   for t <= P + j
 *   out    = sum_t softmax(s)_t * V_r[t]
 *
 * row_list (optional): compute only these query rows; out is then [num_rows][Hq][D], else
 * [total rows][Hq][D]. nthreads <= 0 uses the OpenMP default. Returns 0 or a negative code.
 */
int oracle_paged_attention(double* out, const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                           const int32_t* query_start_loc, int num_reqs, int num_q_heads, int num_kv_heads,
                           int head_dim, int block_size, int num_blocks, double scale, int dtype,
                           const int32_t* row_list, int num_rows, int nthreads) {
    if (num_reqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return ORACLE_BAD_ARG;
    if (num_q_heads % num_kv_heads != 0) return ORACLE_BAD_ARG;
    const int total_rows = num_reqs > 0 ? query_start_loc[num_reqs] : 0;
    const int rows = row_list ? num_rows : total_rows;
    const int group = num_q_heads / num_kv_heads;
    for (int r = 0; r < num_reqs; ++r) {
        int n = query_start_loc[r + 1] - query_start_loc[r];
        if (n < 0 || context_lens[r] < n || (n > 0 && context_lens[r] < 1)) return ORACLE_BAD_ARG;
        int64_t nb = oracle_blocks_for_tokens(context_lens[r], block_size);
        if (n > 0 && nb > max_blocks) return ORACLE_BAD_TABLE;
        for (int64_t i = 0; n > 0 && i < nb; ++i) {
            int32_t b = block_tables[(int64_t)r * max_blocks + i];
            if (b < 0 || b >= num_blocks) return ORACLE_BAD_TABLE;
        }
    }
    int status = ORACLE_OK;
    const int64_t work = (int64_t)rows * num_q_heads;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t w = 0; w < work; ++w) {
        const int i = (int)(w / num_q_heads);
        const int h = (int)(w % num_q_heads);
        const int row = row_list ? row_list[i] : i;
        const int r = request_of_row(query_start_loc, num_reqs, row);
        const int n = query_start_loc[r + 1] - query_start_loc[r];
        const int64_t prior = (int64_t)context_lens[r] - n;
        const int64_t j = row - query_start_loc[r];
#ifdef ORACLE_MUTANT_CAUSAL
        const int64_t limit = prior + j;
#else
        const int64_t limit = prior + j + 1;                    /* keys 0 .. prior + j */
#endif
#ifdef ORACLE_MUTANT_GQA
        const int g = h % num_kv_heads;
#else
        const int g = h / group;
#endif
        double* o = out + ((int64_t)i * num_q_heads + h) * head_dim;
        double* s = (double*)malloc(sizeof(double) * (size_t)(limit > 0 ? limit : 1));
        if (!s) { status = ORACLE_NO_MEM; continue; }
        const int64_t qbase = ((int64_t)row * num_q_heads + h) * head_dim;
        double m = -INFINITY;
        for (int64_t t = 0; t < limit; ++t) {
#ifdef ORACLE_MUTANT_TABLE_INDEX
            const int64_t blk = block_tables[(int64_t)r * max_blocks + t % block_size % max_blocks];
            const int64_t off = t / block_size % block_size;
#else
            const int64_t blk = block_tables[(int64_t)r * max_blocks + t / block_size];
            const int64_t off = t % block_size;
#endif
#ifdef ORACLE_MUTANT_POOL_STRIDE
            const int64_t kbase = (((int64_t)g * num_blocks + blk) * block_size + off) * head_dim;
#else
            const int64_t kbase = ((blk * num_kv_heads + g) * block_size + off) * head_dim;
#endif
            double dot = 0.0;
            for (int d = 0; d < head_dim; ++d) dot += load_elem(q, qbase + d, dtype) * load_elem(k_pool, kbase + d, dtype);
#ifdef ORACLE_MUTANT_NO_SCALE
            s[t] = dot;
#else
            s[t] = scale * dot;
#endif
            if (s[t] > m) m = s[t];
        }
        double denom = 0.0;
        for (int64_t t = 0; t < limit; ++t) { s[t] = exp(s[t] - m); denom += s[t]; }
        for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
        for (int64_t t = 0; t < limit; ++t) {
            const int64_t blk = block_tables[(int64_t)r * max_blocks + t / block_size];
            const int64_t vbase = ((blk * num_kv_heads + g) * block_size + t % block_size) * head_dim;
            for (int d = 0; d < head_dim; ++d) o[d] += s[t] * load_elem(v_pool, vbase + d, dtype);
        }
        for (int d = 0; d < head_dim; ++d) o[d] /= denom;
        free(s);
    }
    return status;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
