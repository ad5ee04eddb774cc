// Internal declarations shared by the library's translation units (host and device).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

constexpr int kBlockSize = 16;      // tokens per KV block
constexpr int kMaxGroupPerItem = 8; // (row, head) slots one FMA-kernel work item serves
constexpr int kMmaSlots = 16;       // (row, head) slots one MMA-kernel work item serves

// First device-side error and its detail (an index); zero when none happened.
struct DeviceError {
    int code;
    int pad;
    long long detail;
};

// One unit of CUDA-core work: num_rows consecutive query rows of one request, a KV head, up to 8
// query heads of its group and a contiguous range of the request's KV blocks. The item's
// (row, head) pairs -- num_rows x heads, at most 8 -- share every K/V block it streams; row
// row + j sees keys at positions < limit + j.
struct DecodeItem {
    int32_t row;        // first query row (index into q/out)
    int32_t req;        // request (row of the block table)
    int16_t kv_head;
    int16_t num_rows;   // consecutive query rows served (>= 1)
    int32_t head0;      // first query head of the group served here (offset inside the group)
    int32_t blk_begin;  // KV block range [blk_begin, blk_end) of the request
    int32_t blk_end;
    int32_t limit;      // the first row sees keys at positions < limit
    int32_t partial;    // partial-result slot, or -1 when the item covers whole rows
};
static_assert(sizeof(DecodeItem) == 32, "DecodeItem layout");

// One tcgen05 tile: 128 packed (query row, query head) rows of one request and KV head.
struct PrefillTile {
    int32_t req;
    int32_t kv_head;
    int32_t tok0;       // first query row of the tile, relative to the request's first row
    int32_t key_tiles;  // 128-key tiles this tile iterates (planner's estimate, for ordering)
};
static_assert(sizeof(PrefillTile) == 16, "PrefillTile layout");

// The (row, head) slots of one item whose partials the log-sum-exp merge combines: slot s is
// query row row + s / heads_per_row, query head q_head0 + s % heads_per_row. Its partials are the
// entries first_partial .. first_partial + count - 1 (slot s of each) and, for a request whose
// leading blocks are shared with others, the shared items' entries extra_first ..
// extra_first + extra_count - 1 (slot extra_slot + s of each).
struct MergeRow {
    int32_t row;
    int32_t q_head0;       // first query head
    int32_t num_slots;     // (row, head) slots in this entry (<= 16)
    int32_t first_partial;
    int32_t count;
    int32_t heads_per_row;
    int32_t extra_first;   // -1 when there are no shared partials
    int32_t extra_count;
    int32_t extra_slot;
    int32_t pad[3];
};
static_assert(sizeof(MergeRow) == 48, "MergeRow layout");

struct DecodeArgs {
    const void* q;
    void* out;
    const void* k_pool;
    const void* v_pool;
    const int32_t* block_tables;
    const DecodeItem* items;
    float* part_o;       // [num_partials][part_stride][D]
    float* part_ml;      // [num_partials][part_stride][2] (max in log2 units, sum)
    DeviceError* err;
    int* work;           // warp-MMA items: [0] item ticket counter, [1] finished warps (zero at launch)
    int num_items;
    int max_blocks_per_seq;
    int num_blocks;
    int num_q_heads;
    int num_kv_heads;
    int group;           // Hq / Hkv
    int heads_per_item;  // query heads one item serves (<= 8)
    int slots_per_item;  // largest num_rows x heads of any item: selects the kernel variant
    int part_stride;     // slots per partial-result entry (8 for the FMA kernel, 16 for the MMA kernel)
    float scale_log2;    // scale * log2(e)
    bool pdl;            // launch with programmatic dependent launch (false after an event wait)
    bool evict_first;    // the warp-MMA kernel's K/V copies carry an L2 evict-first hint (every
                         // block is read by one item: nothing is lost by letting it leave L2 first)
};

struct MergeArgs {
    void* out;
    const MergeRow* rows;
    const float* part_o;
    const float* part_ml;
    int num_rows;
    int num_q_heads;
    int slots_per_entry;  // largest num_slots of any merge row: warps launched per row
    int part_stride;      // slots per partial-result entry
    bool pdl;             // launch with programmatic dependent launch (false after an event wait)
};

struct PrefillArgs {
    const void* q;
    void* out;
    const void* k_pool;
    const void* v_pool;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start_loc;
    const PrefillTile* tiles;
    DeviceError* err;
    int* work;           // [2] tile ticket counter, [3] finished CTAs (zero at launch)
    int decode_ctas;     // CTAs that start on the split-K items passed beside the tiles
    int num_tiles;
    int max_blocks_per_seq;
    int num_blocks;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int num_q_tokens;
    float scale_log2;
    bool pdl;            // launch with programmatic dependent launch (false after an event wait)
};

// Launchers (return the launch error, if any).
cudaError_t launch_decode(int dtype, int head_dim, const DecodeArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_merge(int dtype, int head_dim, const MergeArgs& a, cudaStream_t s);
cudaError_t launch_decode_mma(int dtype, const DecodeArgs& a, int num_sms, cudaStream_t s);
bool decode_mma_supported(int dtype, int head_dim);
// The tcgen05 tile kernel: persistent CTAs over the tiles and, when d.num_items > 0, the split-K
// items of d (warp-MMA kind) as well.
cudaError_t launch_prefill_tc(int dtype, const PrefillArgs& a, const DecodeArgs& d, int num_sms, cudaStream_t s);
bool prefill_tc_supported(int dtype, int head_dim, int group);
cudaError_t launch_slot_mapping(const int32_t* bt, int max_blocks, const int32_t* qsl, const int32_t* ctx,
                                int num_reqs, int num_blocks, int64_t* slots, int num_tokens, DeviceError* err,
                                cudaStream_t s);
cudaError_t launch_kv_write(const void* k_new, const void* v_new, void* k_pool, void* v_pool, const int64_t* slots,
                            int num_tokens, int num_blocks, int num_kv_heads, int row_bytes, DeviceError* err,
                            cudaStream_t s);
cudaError_t launch_copy_blocks(void* const* k_pools, void* const* v_pools, int num_layers, const int32_t* pairs,
                               int num_pairs, int num_blocks, long long block_bytes, DeviceError* err,
                               cudaStream_t s);

// Device error word of the current device.
DeviceError* device_error_word();

// Replaces the calling thread's pkv_last_error() message.
void set_last_error(const char* msg);

// Unique id of the calling thread's current CUDA context (0 when none is current or the driver
// cannot say).
unsigned long long current_context_id();

}  // namespace pkv
