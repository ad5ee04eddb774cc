// Slot mapping, KV append and copy-on-write block copy kernels.
//
//  * slot_mapping_kernel: 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "快速回顾 prefill、decode 和
//    KV cache" (each processed token appends one K/V entry) and "PagedAttention：核心思路" (a request
//    fills its blocks in table order; a new block is used once the previous one is full).
//  * kv_write_kernel: the append itself, a bit-exact scatter of 16-byte vectors.
//  * copy_blocks_kernel: blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存共享" -- the
//    block copy made before a shared block is modified.
// All three are pure integer/byte work bound by memory latency and launch cost; they move data with
// 128-bit loads and stores, coalesced across the head dimension.
#include "common.cuh"

namespace pkv {
namespace {

// One CTA per request; its threads walk the request's new rows.
__global__ void __launch_bounds__(128) slot_mapping_kernel(const int32_t* __restrict__ bt, int max_blocks,
                                                           const int32_t* __restrict__ qsl,
                                                           const int32_t* __restrict__ ctx, int num_blocks,
                                                           int64_t* __restrict__ slots, int num_tokens,
                                                           DeviceError* err) {
    griddep_wait();
    const int r = blockIdx.x;
    const int begin = qsl[r], end = qsl[r + 1];
    const int n = end - begin;
    const long long first_pos = (long long)ctx[r] - n;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int row = begin + j;
        if (row < 0 || row >= num_tokens) {
            record_error(err, 6, row);
            continue;
        }
        const long long pos = first_pos + j;
        const long long lb = pos / kBlockSize;
        long long slot = -1;
        if (pos >= 0 && lb < max_blocks) {
            const int id = bt[(size_t)r * max_blocks + lb];
            if (id >= 0 && id < num_blocks) slot = (long long)id * kBlockSize + pos % kBlockSize;
        }
        if (slot < 0) record_error(err, 6, row);
        slots[row] = slot;
    }
}

// 16 bytes from src (read under L2 policy `rd`) to dst (written under `wr`).
__device__ __forceinline__ void copy16(uint4* dst, const uint4* src, uint64_t rd, uint64_t wr) {
    uint4 x;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                 : "l"(src), "l"(rd));
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst), "r"(x.x), "r"(x.y), "r"(x.z),
                 "r"(x.w), "l"(wr)
                 : "memory");
}

// One thread per 16-byte chunk of one (token, KV head) row, for K and for V. The new K/V is read
// once (an L2 evict-first policy lets it go first); the pool rows written stay in L2 longer (evict
// last), where the attention kernels that follow read them (measured: the 32 k-token append of
// the parallel-sampling batch 45.9 -> 43.9 us and its decode 53.6 -> 51.2 us; the 64-row decode
// step unchanged; evict-first loads alone were slower).
__global__ void __launch_bounds__(256) kv_write_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                                       uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                                       const int64_t* __restrict__ slots, long long num_chunks,
                                                       int num_kv_heads, int cpr, long long num_slots,
                                                       DeviceError* err) {
    griddep_wait();
    uint64_t read_once, keep;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(read_once));
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
    const long long per_token = (long long)num_kv_heads * cpr;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < num_chunks;
         i += (long long)gridDim.x * blockDim.x) {
        const long long t = i / per_token;
        const int rest = (int)(i - t * per_token);
        const int h = rest / cpr;
        const int c = rest - h * cpr;
        const long long slot = __ldg(slots + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            record_error(err, 6, t);
            continue;
        }
        const long long blk = slot / kBlockSize, off = slot % kBlockSize;
        const long long dst = ((blk * num_kv_heads + h) * kBlockSize + off) * cpr + c;
        copy16(k_pool + dst, k_new + i, read_once, keep);
        copy16(v_pool + dst, v_new + i, read_once, keep);
    }
}

constexpr int kMaxLayersPerLaunch = 64;
struct LayerPtrs {
    uint4* k[kMaxLayersPerLaunch];
    uint4* v[kMaxLayersPerLaunch];
};

// grid.x = pair, grid.y = layer (within this launch), grid.z = 0 for K, 1 for V.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const LayerPtrs ptrs, const int32_t* __restrict__ pairs,
                                                          int num_blocks, long long chunks_per_block,
                                                          DeviceError* err) {
    griddep_wait();
    const int p = blockIdx.x;
    const int src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
        if (threadIdx.x == 0) record_error(err, 6, p);
        return;
    }
    if (src == dst) return;
    uint4* base = blockIdx.z == 0 ? ptrs.k[blockIdx.y] : ptrs.v[blockIdx.y];
    const uint4* s = base + (long long)src * chunks_per_block;
    uint4* d = base + (long long)dst * chunks_per_block;
    // Eight 16-byte loads in flight per thread before their stores (a copy that stored each chunk
    // before loading the next paid one memory latency per chunk). Source and destination are
    // distinct blocks, so they never overlap.
    constexpr int U = 8;
    const long long n = chunks_per_block;
    for (long long i0 = threadIdx.x; i0 < n; i0 += (long long)blockDim.x * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + (long long)u * blockDim.x;
            if (i < n) v[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + (long long)u * blockDim.x;
            if (i < n) d[i] = v[u];
        }
    }
}

}  // namespace

cudaError_t launch_slot_mapping(const int32_t* bt, int max_blocks, const int32_t* qsl, const int32_t* ctx,
                                int num_reqs, int num_blocks, int64_t* slots, int num_tokens, DeviceError* err,
                                cudaStream_t s) {
    if (num_reqs <= 0 || num_tokens <= 0) return cudaSuccess;
    return launch_pdl(slot_mapping_kernel, dim3(num_reqs), dim3(128), 0, s, bt, max_blocks, qsl, ctx, num_blocks, slots,
                      num_tokens, err);
}

cudaError_t launch_kv_write(const void* k_new, const void* v_new, void* k_pool, void* v_pool, const int64_t* slots,
                            int num_tokens, int num_blocks, int num_kv_heads, int row_bytes, DeviceError* err,
                            cudaStream_t s) {
    const int cpr = row_bytes / 16;
    const long long chunks = (long long)num_tokens * num_kv_heads * cpr;
    if (chunks <= 0) return cudaSuccess;
    long long grid = (chunks + 255) / 256;
    if (grid > 148LL * 16) grid = 148LL * 16;
    return launch_pdl(kv_write_kernel, dim3((unsigned)grid), dim3(256), 0, s, static_cast<const uint4*>(k_new),
                      static_cast<const uint4*>(v_new), static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), slots,
                      chunks, num_kv_heads, cpr, (long long)num_blocks * kBlockSize, err);
}

cudaError_t launch_copy_blocks(void* const* k_pools, void* const* v_pools, int num_layers, const int32_t* pairs,
                               int num_pairs, int num_blocks, long long block_bytes, DeviceError* err,
                               cudaStream_t s) {
    if (num_pairs <= 0 || num_layers <= 0) return cudaSuccess;
    for (int l0 = 0; l0 < num_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = num_layers - l0 < kMaxLayersPerLaunch ? num_layers - l0 : kMaxLayersPerLaunch;
        LayerPtrs ptrs{};
        for (int i = 0; i < nl; ++i) {
            ptrs.k[i] = static_cast<uint4*>(k_pools[l0 + i]);
            ptrs.v[i] = static_cast<uint4*>(v_pools[l0 + i]);
        }
        cudaError_t e = launch_pdl(copy_blocks_kernel, dim3(num_pairs, nl, 2), dim3(256), 0, s, ptrs, pairs, num_blocks,
                                   block_bytes / 16, err);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pkv
