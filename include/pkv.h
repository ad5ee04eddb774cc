/*
 * pkv.h -- C ABI of a B200 (sm_100a) PagedAttention library.
 *
 * The KV cache lives in one pool of fixed 16-token blocks; each request owns an ordered table of
 * physical block ids; attention reads K and V block by block through that table and returns what
 * contiguous storage would (blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感";
 * 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention：核心思路").
 *
 * Conventions for every call:
 *   - Device pointers are caller-owned (typically torch tensors). The library makes no device
 *     allocation; the only device memory it owns is module-scope: a 16-byte error word per device
 *     (pkv_device_error) and the fixed scratch array of pkv_paged_attention_static_ws, the one
 *     call that does not take a caller workspace. Host pointers are read during the call only.
 *   - Kernels run asynchronously on the caller's stream `stream` (0 = legacy default stream).
 *   - Argument errors are detected on the host before any launch and returned as a pkv_status;
 *     no call traps on the device. Kernels that find an out-of-range block id or slot at run time
 *     skip that access and record the first such event in a device error word read by
 *     pkv_device_error(). Bounded waits that expire record PKV_ERR_DEVICE_TIMEOUT there.
 *   - The element type (pkv_dtype) is the same for q, k, v, new K/V and the output.
 *
 * Layouts (row-major, element counts):
 *   q, out          [T, Hq, D]                 T = query rows of the batch
 *   k_pool, v_pool  [num_blocks, Hkv, 16, D]   one (block, kv head) is a contiguous 16*D run
 *   k_new, v_new    [T_new, Hkv, D]
 *   block_tables    int32 [R, max_blocks_per_seq]; entries past ceil(context/16) are ignored
 *   context_lens    int32 [R]   tokens in the cache after this step's tokens are appended
 *   query_start_loc int32 [R+1] prefix sum of the step's {request_id: num_tokens} counts
 *   slot_mapping    int64 [T_new] physical slot = block_id * 16 + offset; negative = skip
 * Query head h reads KV head h / (Hq / Hkv). Row j of a request with n rows and context ctx sits
 * at position ctx - n + j and attends keys 0 .. ctx - n + j.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pkv_stream_t; /* same handle as cudaStream_t */

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,          /* a null pointer, a negative size, an inconsistent batch */
    PKV_ERR_UNSUPPORTED = 2,          /* a shape or type this build does not handle */
    PKV_ERR_CUDA = 3,                 /* a CUDA runtime call failed; see pkv_last_error() */
    PKV_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes below what the plan needs */
    PKV_ERR_DEVICE_TIMEOUT = 5,       /* a kernel's bounded wait expired (device error word only) */
    PKV_ERR_DEVICE_RANGE = 6,         /* a kernel met an out-of-range id (device error word only) */
    PKV_ERR_OUT_OF_BLOCKS = 7         /* the block pool has too few free blocks; nothing was changed */
} pkv_status;

typedef enum pkv_dtype { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2 } pkv_dtype;

#define PKV_BLOCK_SIZE 16
#define PKV_PLAN_MAGIC 0x706b7631u /* "pkv1" */

/* Human-readable name of a status (static storage). */
const char* pkv_status_string(pkv_status s);
/* Message of the last failing call on this host thread (static thread-local storage). */
const char* pkv_last_error(void);
/* Library version string. */
const char* pkv_version(void);

/*
 * pkv_slot_mapping -- physical slot of every token this step appends.
 * Source: 一文搞懂vLLM, "快速回顾 prefill、decode 和 KV cache" (every processed token adds one K/V entry)
 * and "PagedAttention：核心思路" (a new block is used once the previous one is full, tracked in the
 * request's block table); blog.mckayzhao.com/?p=56, "PagedAttention" section (table = logical ->
 * physical map). Row j of request r lands at position p = ctx_r - n_r + j and
 *   slot = block_tables[r][p / 16] * 16 + p % 16.
 * Device inputs: block_tables [R, max_blocks_per_seq], query_start_loc [R+1], context_lens [R].
 * Device output: slot_mapping [num_tokens] (num_tokens = query_start_loc[R], given by the caller).
 * A table entry outside [0, num_blocks) yields slot -1 and sets the device error word.
 * Errors: INVALID_ARG for null pointers (with num_tokens > 0) or negative sizes.
 */
pkv_status pkv_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq, const int32_t* query_start_loc,
                            const int32_t* context_lens, int num_reqs, int num_blocks, int64_t* slot_mapping,
                            int num_tokens, pkv_stream_t stream);

/*
 * pkv_kv_cache_write -- append new K/V rows into their slots:
 *   k_pool[slot / 16][h][slot % 16][:] = k_new[t][h][:]   (same for V), for every slot >= 0.
 * Source: 一文搞懂vLLM, "快速回顾 prefill、decode 和 KV cache" (the cache grows by one entry per token).
 * Slots must be distinct within one call (else which row lands is unspecified); slots at or
 * beyond num_blocks * 16 are skipped and set the device error word. Bit-exact copy.
 * Errors: INVALID_ARG (null pointer with num_tokens > 0, negative sizes), UNSUPPORTED
 * (block_size != 16, head_dim * element size not a multiple of 16 bytes or above 1024 bytes).
 */
pkv_status pkv_kv_cache_write(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                              const int64_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                              int head_dim, int block_size, pkv_dtype dtype, pkv_stream_t stream);

/*
 * pkv_copy_blocks -- copy-on-write block copy: for every layer l and every (src, dst) pair,
 * block dst of k_pools[l] and of v_pools[l] (all KV heads) becomes a copy of block src.
 * Source: blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存共享" (copy the shared block,
 * modify the copy, leave the original unchanged); 一文搞懂vLLM, "PagedAttention 是怎么共享内存的".
 * k_pools, v_pools: HOST arrays of num_layers device pointers, each [num_blocks, Hkv, 16, D].
 * block_mapping: DEVICE int32 [num_pairs][2] = (src, dst). Preconditions: no dst repeats and no
 * dst is also a src in the same call; src == dst is a no-op; ids outside [0, num_blocks) are
 * skipped and set the device error word. Bit-exact.
 * Errors: INVALID_ARG (null pointers, negative sizes), UNSUPPORTED (block_size != 16).
 */
pkv_status pkv_copy_blocks(void* const* k_pools, void* const* v_pools, int num_layers,
                           const int32_t* block_mapping, int num_pairs, int num_blocks, int num_kv_heads,
                           int head_dim, int block_size, pkv_dtype dtype, pkv_stream_t stream);

/* Planner knobs (all zero = defaults). */
typedef struct pkv_plan_options {
    int32_t split_blocks;      /* >0: decode/support rows are cut into chunks of this many blocks;
                                  0: chosen from the batch size and the SM count */
    int32_t no_split;          /* 1: every row is one chunk (no log-sum-exp merge) */
    int32_t cuda_core_only;    /* 1: no tcgen05 tiles; multi-row requests also go to the split-K
                                  decode kernel (warp-MMA or FMA) */
    int32_t num_sms;           /* SM count the chunking targets; 0 = query the current device
                                  (pkv_attention_plan) or 148 (pkv_attention_plan_host) */
    int32_t heads_per_item;    /* query heads of one group served by one split-K work item (1..16
                                  for the warp-MMA kernel, 1..8 for the FMA kernel); 0 = the group,
                                  capped at that slot count. Larger groups are split into items
                                  that read the same K/V blocks */
    int32_t rows_per_item;     /* consecutive query rows of one request served by one split-K item,
                                  capped so rows x heads fits the kernel's slots; 0 = as many as
                                  fit. Such an item streams each K/V block once for all its
                                  (row, head) pairs */
    int32_t tc_min_rows;       /* requests with at least this many rows (>= 2) go to the tcgen05
                                  tiles where the shape allows; fewer rows, the split-K kernel.
                                  0 = rows x group > 16 with the MMA kernel (a request whose
                                  (row, head) pairs fit one MMA item stays there), else 2 */
    int32_t decode_kernel;     /* kernel for the rows not on tcgen05 tiles: 0 = chosen by the
                                  planner, 1 = FMA kernel (items of <= 8 (row, head) slots),
                                  2 = warp-MMA kernel (<= 16 slots; f16/bf16, head_dim 128) */
    /* Shared prefixes (optional; read during the planning call only). A run of consecutive decode
     * requests (one row each) whose tables start with the same >= min_shared_blocks physical
     * blocks (each fully inside every member's context) reads those blocks once for all of them;
     * each request's own blocks are read separately and the parts are merged by log-sum-exp. The
     * pages' sharing of a common prefix (parallel samples, beam candidates, cached prompts):
     * 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention 是怎么共享内存的". */
    const int32_t* h_block_tables;   /* host copy of block_tables, or NULL (no sharing) */
    int32_t block_table_stride;      /* its row length (max_blocks_per_seq) */
    int32_t min_shared_blocks;       /* 0 = 4 */
    /* Mixed batches (tcgen05 tiles and warp-MMA split-K items in one plan): the tile kernel's
     * persistent CTAs (one per SM) serve both queues in one launch -- decode_sms of them start on
     * the split-K items and the others on the tiles, and each turns to the other queue once its own
     * is empty -- so the tensor-bound tiles and the HBM-bound items share the GPU. 0 = sized by the
     * planner, which simulates the greedy tile schedule beside the items' streaming for splits
     * near the balanced share and takes the middle of the near-best run; -1 = no overlap (the
     * split-K kernel runs after the tiles). */
    int32_t decode_sms;
} pkv_plan_options;

/*
 * Host description of a planned batch (caller-owned memory, filled by the planner). The work
 * lists themselves live in the caller's device workspace at the byte offsets below.
 */
typedef struct pkv_plan {
    uint32_t magic;              /* PKV_PLAN_MAGIC once filled */
    int32_t num_reqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim, dtype;
    int32_t num_decode_rows;     /* rows served by the split-K decode kernel */
    int32_t num_prefill_rows;    /* rows served by the tcgen05 tile kernel */
    int32_t num_items;           /* split-K work items (rows, kv head, heads, block chunk) */
    int32_t num_tiles;           /* tcgen05 tiles (request, kv head, 128 packed rows) */
    int32_t num_merge_rows;      /* chunked split-K items' (rows, heads) sets merged from partials */
    int32_t num_partials;        /* chunk partial results in the workspace */
    int32_t split_blocks;        /* chunk length in blocks used for this batch */
    int32_t max_blocks;          /* longest context in blocks */
    int32_t heads_per_item;      /* query heads per split-K work item */
    int32_t rows_per_item;       /* most consecutive rows any split-K item serves (0: no items) */
    int32_t decode_kernel;       /* 1 FMA kernel, 2 warp-MMA kernel, 0 no split-K items */
    int32_t part_stride;         /* (row, head) slots per partial-result entry: the largest item's */
    int32_t merge_slots;         /* most (row, head) slots of any merge row (the merge grid's stride) */
    int64_t off_items, off_tiles, off_merge, off_part_o, off_part_ml; /* byte offsets into workspace */
    int64_t meta_bytes;          /* bytes uploaded by pkv_attention_plan (work lists) */
    int64_t ws_bytes;            /* total workspace bytes this plan needs */
    int64_t kv_bytes;            /* algorithmic K+V bytes read: sum over rows' attended keys of
                                    2*D*elem per (kv head, key), counted once per (request, kv head)
                                    for decode rows and once per request for prefill rows */
    int64_t attn_flops;          /* 4*D per (query row, query head, attended key) */
    int64_t core_kv_bytes;       /* K+V bytes the split-K kernel must read: its requests' contexts,
                                    with a prefix shared by a run of requests counted once */
    int64_t tile_kv_bytes;       /* part of kv_bytes read by the tcgen05 tiles */
    int64_t tile_flops;          /* part of attn_flops computed by the tcgen05 tiles */
    int32_t decode_sms;          /* > 0: one launch of the tile kernel also serves the split-K items,
                                    with this many CTAs starting on them; 0: the split-K kernel runs
                                    after the tiles */
    uint32_t flags;              /* PKV_PLAN_* bits below */
} pkv_plan;

/* pkv_plan.flags: every K/V block the split-K items read is read by exactly one item (no shared-
 * prefix group, one item per KV head's query group and per request's rows), so the split-K kernel
 * may mark those reads to leave L2 first. */
#define PKV_PLAN_SINGLE_READ 1u

/*
 * pkv_attention_workspace_size -- bytes of device workspace pkv_attention_plan will need for this
 * batch (same host inputs as the planner). Host-only; does not touch the GPU unless
 * opts->num_sms == 0, in which case it reads the current device's SM count.
 */
pkv_status pkv_attention_workspace_size(const int32_t* h_query_start_loc, const int32_t* h_context_lens,
                                        int num_reqs, int num_q_heads, int num_kv_heads, int head_dim,
                                        pkv_dtype dtype, const pkv_plan_options* opts, size_t* bytes);

/*
 * pkv_attention_plan_host -- split the batch into work lists on the host, without any CUDA call.
 * Source for the batch: blog.mckayzhao.com/?p=56, "V1 架构：推倒重来的勇气" (one step = a dict
 * {request_id: num_tokens}; decode rows and chunked-prefill rows share the batch) and "进阶特性"
 * (chunked prefill). Requests with fewer than tc_min_rows rows (by default: all whose rows x
 * group fit one 16-slot warp-MMA item, so decode and short speculative-verify rows) become split-K
 * work: items of up to 16 (row, head) slots (8 for the FMA kernel) of one request and KV head,
 * consecutive rows packed together, each slot with its own causal limit. The warp-MMA kernel
 * serves them when dtype is f16/bf16 and head_dim is 128, the FMA kernel otherwise. Requests with
 * more rows go to the tcgen05 tile kernel when dtype is f16/bf16, head_dim is 128 and Hq/Hkv
 * divides 128 (otherwise to the split-K kernel). Long contexts are cut into block chunks whose
 * partial results a log-sum-exp merge combines. With opts->h_block_tables, runs of decode
 * requests that start with the same physical blocks become one shared-prefix item set plus
 * per-request suffix items, merged the same way.
 * h_meta (host, meta_capacity bytes) receives the image that pkv_attention_plan uploads to the
 * start of the workspace; pass NULL to only fill *plan.
 * Errors: INVALID_ARG (query_start_loc not starting at 0 or decreasing, context < num_tokens,
 * num_tokens > 0 with context 0, Hq % Hkv != 0, decode_kernel outside 0..2), UNSUPPORTED (head_dim
 * not 64/128, decode_kernel 2 asked for where the warp-MMA kernel does not apply),
 * WORKSPACE_TOO_SMALL (meta_capacity below plan->meta_bytes).
 */
pkv_status pkv_attention_plan_host(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                                   const pkv_plan_options* opts, void* h_meta, size_t meta_capacity,
                                   pkv_plan* plan);

/*
 * pkv_attention_plan -- pkv_attention_plan_host, then one cudaMemcpyAsync of the work lists into
 * d_workspace on `stream`. A plan stays valid for any number of pkv_paged_attention calls on the
 * same batch shape (e.g. every layer of a model step) while the workspace is not reused.
 * Errors: as pkv_attention_plan_host, plus WORKSPACE_TOO_SMALL (ws_bytes < plan->ws_bytes) and CUDA.
 */
pkv_status pkv_attention_plan(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                              int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                              const pkv_plan_options* opts, void* d_workspace, size_t ws_bytes, pkv_plan* plan,
                              pkv_stream_t stream);

/*
 * pkv_attention_plan_async -- the per-step planning call of a serving loop: plans the batch on the
 * host straight into caller-owned page-locked memory and enqueues its uploads on `stream`, so the
 * host never waits for a copy:
 *   h_meta[0, plan->meta_bytes)  -> d_workspace[0, plan->meta_bytes)   (the work lists)
 *   h_desc[0, 2R + 1)            -> d_desc[0, 2R + 1)                  (R = num_reqs, int32)
 * where h_desc receives query_start_loc (R + 1 entries) followed by context_lens (R entries), so
 * d_desc and d_desc + R + 1 are the device query_start_loc and context_lens of the batch (pass
 * h_desc = d_desc = NULL to skip that copy). h_meta and h_desc must be page-locked and stay
 * untouched until the copies have run: record an event on `stream` after the call and wait for
 * it before reusing them. The batch is the one pkv_attention_plan_host describes (same source).
 * Errors: as pkv_attention_plan_host; WORKSPACE_TOO_SMALL when meta_capacity < plan->meta_bytes
 * or ws_bytes < plan->ws_bytes -- nothing is enqueued and *plan holds the sizes needed, with its
 * magic cleared so that it cannot be launched; INVALID_ARG when only one of h_desc / d_desc is
 * NULL; CUDA.
 */
pkv_status pkv_attention_plan_async(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                                    int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                                    const pkv_plan_options* opts, void* h_meta, size_t meta_capacity,
                                    void* d_workspace, size_t ws_bytes, int32_t* h_desc, int32_t* d_desc,
                                    pkv_plan* plan, pkv_stream_t stream);

/*
 * pkv_paged_attention -- attention for every row of a planned mixed batch.
 * Source: blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感" (find each block
 * through the table, read K and V block by block; same result as contiguous storage) and
 * "V1 架构：推倒重来的勇气" (decode and chunked-prefill rows in one batch).
 *   out[row][h][:] = sum_t softmax_t(scale * q[row][h] . K_r[t]) V_r[t],  t = 0 .. ctx_r - n_r + j
 * with K_r[t] = k_pool[block_tables[r][t/16]][h / (Hq/Hkv)][t%16]. Softmax and accumulation in fp32;
 * the output is rounded to the element type. Launches, on `stream`: the tcgen05 prefill tile
 * kernel (if the plan has tiles; persistent CTAs, one per SM, taking tiles longest first), the
 * split-K decode kernel the plan names (warp-MMA or FMA, if it has items) -- or, when
 * plan->decode_sms > 0, one tile-kernel launch that serves the warp-MMA items as well -- and the
 * log-sum-exp merge kernel (if it has merge rows). The kernels take their work from ticket
 * counters in the workspace header, which the plan upload zeroes and each launch leaves at zero.
 * The plan and workspace must come from pkv_attention_plan with the same batch; q/out shapes must
 * match it; launches sharing one workspace must not overlap on the GPU.
 * Errors: INVALID_ARG (null pointers, plan magic/shape mismatch), WORKSPACE_TOO_SMALL, CUDA.
 */
pkv_status pkv_paged_attention(void* out, const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               const int32_t* query_start_loc, int num_blocks, float scale, const pkv_plan* plan,
                               void* d_workspace, size_t ws_bytes, pkv_stream_t stream);

/*
 * Host-side validators (no CUDA calls). They check the preconditions the kernels rely on and
 * return INVALID_ARG with a message in pkv_last_error() on the first violation.
 *   pkv_validate_tables: for every request, entries [0, ceil(ctx/16)) lie in [0, num_blocks) and
 *     ceil(ctx/16) <= max_blocks_per_seq.
 *   pkv_validate_slots: every slot >= 0 is below num_blocks*16 and no slot repeats.
 *   pkv_validate_copy_pairs: ids in range, no dst repeats, no dst is also a src.
 */
pkv_status pkv_validate_tables(const int32_t* h_block_tables, const int32_t* h_context_lens, int num_reqs,
                               int max_blocks_per_seq, int num_blocks);
pkv_status pkv_validate_slots(const int64_t* h_slot_mapping, int num_tokens, int num_blocks);
pkv_status pkv_validate_copy_pairs(const int32_t* h_pairs, int num_pairs, int num_blocks);

/*
 * pkv_device_error -- read and clear the device error word of the current device (synchronises
 * `stream`). *code receives PKV_OK or the first PKV_ERR_DEVICE_* recorded since the last read;
 * *detail receives the offending index (or -1).
 */
pkv_status pkv_device_error(int* code, int64_t* detail, pkv_stream_t stream);

/*
 * pkv_paged_attention_static_ws -- plan and run paged attention with no device allocation at all.
 * The pages have no counterpart to this call; it exists for callers that cannot call cudaMalloc
 * where they run attention (an engine whose memory manager already owns nearly all of HBM, a
 * plugin inside a runtime that owns every allocation, code running where allocation calls are
 * forbidden or would stall). Instead of a caller workspace it uses one library-owned device array
 * of PKV_STATIC_WS_BYTES, held by every GPU that loads the library until the process exits.
 * Arguments: the host batch description and options of pkv_attention_plan, then the device
 * tensors and scale of pkv_paged_attention (same layouts and meaning); out receives the result.
 * The array's device address is looked up on the first call made on each device (and again when
 * that device's current CUDA context is a different one, e.g. after cudaDeviceReset), with
 * cudaGetSymbolAddress. The batch is planned once per call, on the host. Every call reuses the same array, which keeps the
 * last call's contents; calls that may overlap on the GPU (other streams or host threads) race on
 * it and must be serialised by the caller. No part of it has to start zeroed: each call writes
 * what its kernels read.
 * Errors: those of pkv_attention_plan and pkv_paged_attention, and WORKSPACE_TOO_SMALL when the
 * batch needs more scratch than PKV_STATIC_WS_BYTES (checked on the host before any launch).
 */
#define PKV_STATIC_WS_BYTES (32u << 20)
pkv_status pkv_paged_attention_static_ws(const int32_t* h_query_start_loc, const int32_t* h_context_lens,
                                         int num_reqs, int num_q_heads, int num_kv_heads, int head_dim,
                                         pkv_dtype dtype, const pkv_plan_options* opts, void* out, const void* q,
                                         const void* k_pool, const void* v_pool, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens,
                                         const int32_t* query_start_loc, int num_blocks, float scale,
                                         pkv_stream_t stream);

/*
 * pkv_selftest_exp2 -- test aid with no counterpart on the pages: y[i] = 2^x[i] computed by the
 * FMA-pipe exponential the prefill softmax uses for part of its elements (range reduction to
 * [-1/2, 1/2] and a fitted degree-4 polynomial, relative error below 3e-6 for -126 <= x <= 127).
 * x, y: device float arrays of n elements. Errors: INVALID_ARG, CUDA.
 */
pkv_status pkv_selftest_exp2(const float* x, float* y, int n, pkv_stream_t stream);

/*
 * Host block manager (host memory only; no CUDA call). Owns the allocation state of one block pool:
 * which physical blocks are free, each sequence's ordered block list and token count, a reference
 * count per block and, optionally, a cache of full blocks keyed by the token prefix they end.
 *   - 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention：核心思路": a sequence gets blocks
 *     on demand (a new one only once its last block is full; any free block will do) and returns all
 *     of them to the pool when it finishes.
 *   - blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感": N tokens hold
 *     ceil(N / block_size) blocks, so at most block_size - 1 slots of a sequence are unused.
 *   - same page, "还不止是分页：Copy-on-Write 和内存共享": forked sequences share blocks under a
 *     reference count; before a sequence writes into a shared block, the block is copied and the
 *     writer's table points at the copy (copy-on-write); the original is left as it was.
 *   - 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention 是怎么共享内存的": requests that
 *     begin with the same prefix store its blocks once and each table points at them;
 *     blog.mckayzhao.com/?p=56, "进阶特性：让推理再快一点" (Prefix Caching), and vLLM 简介
 *     (docs.freetools.me), "自动前缀缓存": prefix caching is hash based: when the beginning of a new
 *     request matches blocks computed before, those KV blocks are reused instead of recomputed.
 * Policy (not fixed by the pages, stated so results are reproducible): free blocks form a queue. A
 * new pool hands out ids 0, 1, 2, ... in order; a block whose count drops to 0 joins the back, and
 * allocation takes the front, so the least recently released block is reused first. A sequence's
 * blocks are released last to first (its later blocks leave the cache before its prefix). Only the
 * last block of a sequence can be partially filled, so only it can need a copy.
 * Prefix cache (managers created with PKV_BM_PREFIX_CACHE): every block of a token-tracked sequence
 * that becomes full is registered under a chain hash of all tokens up to its end (SplitMix64 mixing
 * of the previous block's key and the block's token ids). A released registered block stays
 * reusable, with its contents, until allocation takes it from the front of the queue (eviction).
 * A lookup accepts a block only if its recorded token ids and the identity of the block before it
 * match, so a hit is exact, not merely hash-equal.
 * Every call either succeeds completely or changes nothing. A manager is not thread-safe: callers
 * serialise calls on one manager. Sequence ids are arbitrary int64 keys.
 */
typedef struct pkv_block_manager pkv_block_manager; /* opaque */

#define PKV_BM_PREFIX_CACHE 1 /* pkv_bm_create_ex flag: keep a prefix cache of full blocks */

typedef struct pkv_pool_stats {
    int64_t num_blocks;     /* pool size */
    int64_t free_blocks;    /* blocks with reference count 0 (cached ones included) */
    int64_t used_blocks;    /* num_blocks - free_blocks */
    int64_t shared_blocks;  /* blocks with reference count > 1 */
    int64_t num_sequences;  /* live sequences */
    int64_t logical_tokens; /* sum of sequence lengths (a shared token counts once per sharer) */
    int64_t stored_tokens;  /* filled slots of used blocks (a shared slot counts once) */
    int64_t wasted_slots;   /* used_blocks * block_size - stored_tokens: reserved but unfilled */
    int64_t cow_copies;     /* copy-on-write copies requested since creation */
    int64_t cached_blocks;  /* blocks a prefix lookup can currently return (held or free) */
    int64_t cache_queries;  /* full prompt blocks looked up since creation */
    int64_t cache_hits;     /* of those, blocks reused from the cache */
} pkv_pool_stats;

/* Creates a manager for a pool of num_blocks blocks of block_size tokens (all free), without a
 * prefix cache. Errors: INVALID_ARG (null out, num_blocks < 0, block_size < 1). */
pkv_status pkv_bm_create(int num_blocks, int block_size, pkv_block_manager** out);
/* Same, with flags (0 or PKV_BM_PREFIX_CACHE). Errors: as above, or unknown flag bits. */
pkv_status pkv_bm_create_ex(int num_blocks, int block_size, int flags, pkv_block_manager** out);
/* Frees the manager (null is ignored). */
void pkv_bm_destroy(pkv_block_manager* bm);
/* Starts sequence seq_id holding num_tokens tokens: ceil(num_tokens / block_size) fresh blocks.
 * Its token ids are unknown, so none of its blocks enters the prefix cache.
 * Errors: INVALID_ARG (null, negative count, id already live), OUT_OF_BLOCKS. */
pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, int64_t num_tokens);
/* Starts token-tracked sequence seq_id from the longest cached prefix of its prompt tokens[0, n)
 * (host int32 token ids): the sequence holds the hit blocks (each block's count + 1) and
 * *num_cached_tokens = hits * block_size of them. At most (n - 1) / block_size blocks are taken
 * from the cache, so at least one prompt token is always left to compute. The caller appends the
 * remaining tokens[*num_cached_tokens, n) with pkv_bm_append_tokens or pkv_bm_step; their K/V must
 * be computed and written, the cached ones must not. Without a prefix cache nothing hits.
 * Errors: INVALID_ARG (null, n < 0, id already live). Takes no free block for itself. */
pkv_status pkv_bm_add_cached_prefix(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t n,
                                    int64_t* num_cached_tokens);
/* Starts sequence child sharing every block of parent (each block's count + 1), same length and
 * token ids. Errors: INVALID_ARG (null, unknown parent, child already live). */
pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child);
/* Appends num_new_tokens tokens to seq_id, allocating the blocks they need. If the first new token
 * goes into a partially filled last block that is shared, that block is copied first: cow_pair
 * (2 int32, required) receives {source, destination} for pkv_copy_blocks, the sequence's last
 * entry becomes the destination and the source's count drops by 1; otherwise {-1, -1}.
 * The token ids are not given: a token-tracked sequence stops being tracked (its later blocks
 * are not cached). Errors: INVALID_ARG (null, negative count, unknown id), OUT_OF_BLOCKS. */
pkv_status pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int64_t num_new_tokens, int32_t* cow_pair);
/* Same, with the new tokens' ids (host int32 [num_new_tokens]); on a prefix-caching manager each
 * block of a token-tracked sequence that becomes full is registered in the cache. */
pkv_status pkv_bm_append_tokens(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                                int64_t num_new_tokens, int32_t* cow_pair);
/* Ends seq_id: each of its blocks' counts drops by 1, last block first; blocks reaching 0 join the
 * back of the free queue (a registered block keeps its cache entry until it is taken again).
 * Errors: INVALID_ARG (null, unknown id). */
pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);
/* Reads one sequence: *num_tokens, *num_blocks, and (when blocks is not null) its block ids into
 * blocks[0 .. *num_blocks). Errors: INVALID_ARG (null outputs, unknown id, capacity too small). */
pkv_status pkv_bm_sequence(const pkv_block_manager* bm, int64_t seq_id, int64_t* num_tokens, int32_t* blocks,
                           int capacity, int* num_blocks);
/* Writes the block tables of num_seqs sequences as int32 rows of max_blocks_per_seq entries
 * (host memory, caller-owned), unused entries -1. Errors: INVALID_ARG (unknown id, row too short). */
pkv_status pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int32_t* tables,
                               int max_blocks_per_seq);
/* Reads one block's reference count. Errors: INVALID_ARG (null, id outside the pool). */
pkv_status pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* count);
/* Fills *stats. Errors: INVALID_ARG (null). */
pkv_status pkv_bm_stats(const pkv_block_manager* bm, pkv_pool_stats* stats);
/*
 * One scheduling step of a {request_id: num_tokens} batch, all on the host: appends
 * num_new_tokens[r] tokens to live sequence seq_ids[r] for every r (ids distinct), then writes the
 * step's attention inputs into caller-owned host arrays: block_tables [num_seqs, max_blocks_per_seq]
 * (-1 padded), context_lens [num_seqs] (lengths after the append), query_start_loc [num_seqs + 1]
 * (prefix sum of num_new_tokens), and the copy-on-write pairs the appends need into
 * cow_pairs [num_seqs, 2] with their count in *num_cow_pairs (at most one per sequence, in batch
 * order). The pairs must be copied (pkv_copy_blocks) before this step's K/V is written.
 * new_tokens (nullable) holds the new tokens' ids, concatenated in batch order
 * (query_start_loc[num_seqs] entries) as pkv_bm_append_tokens takes them; when null, every
 * token-tracked member stops being tracked, as with pkv_bm_append.
 * Errors: INVALID_ARG (null, unknown or repeated id, negative count, row too short, a length over
 * INT32_MAX), OUT_OF_BLOCKS (checked for the whole batch first; nothing changes).
 */
pkv_status pkv_bm_step(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* num_new_tokens, int num_seqs,
                       const int32_t* new_tokens, int32_t* block_tables, int max_blocks_per_seq,
                       int32_t* context_lens, int32_t* query_start_loc, int32_t* cow_pairs, int* num_cow_pairs);

/*
 * Kernel timing (no counterpart on the pages; a measurement aid). Between pkv_profile_start and
 * pkv_profile_stop, every kernel the library launches on the calling host thread is bracketed by
 * a pair of CUDA events recorded on the launch stream. pkv_profile_stop synchronises those events,
 * writes per-kind totals (milliseconds) and launch counts into arrays of PKV_KERNEL_KINDS entries,
 * and stops recording. At most `capacity` launches are timed; later ones are counted but not
 * timed (*dropped receives how many). Events are created on the current device at start.
 * Errors: INVALID_ARG (capacity < 1, null outputs, stop without start), CUDA.
 */
typedef enum pkv_kernel_kind {
    PKV_KERNEL_SLOT_MAPPING = 0,
    PKV_KERNEL_KV_WRITE = 1,
    PKV_KERNEL_COPY_BLOCKS = 2,
    PKV_KERNEL_DECODE = 3,
    PKV_KERNEL_MERGE = 4,
    PKV_KERNEL_PREFILL_TC = 5,
    PKV_KERNEL_KINDS = 6
} pkv_kernel_kind;

pkv_status pkv_profile_start(int capacity);
pkv_status pkv_profile_stop(double* total_ms, int* launches, int* dropped);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
