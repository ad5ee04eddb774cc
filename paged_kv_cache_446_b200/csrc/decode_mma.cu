// Paged attention on warp-level tensor-core MMAs for work items of up to 16 (row, head) slots.
//
// What it computes is what decode.cu computes (blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里
// 翻出来的灵感": every KV block of a request is found through its block table and read block by
// block; the result equals attention over contiguous storage), for items that pack up to 16
// (query row, query head) slots sharing one KV head: a query group of 8 or 16 heads, or several
// rows of one request (a speculative verify step: 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？,
// "V1 架构：推倒重来的勇气", a request submits k+1 tokens in one {request_id: num_tokens} step).
//
// Why tensor cores here: per 16-token block an item contracts a 16-slot x 128 Q tile with K and
// the 16-slot softmax weights with V -- two small dense products. On CUDA cores that costs about
// a thousand warp instructions per block for 8 slots, so the kernel is bound by instruction issue,
// not by HBM; as m16n8k16 MMAs (fp32 accumulation) it is 32 MMAs and 16 ldmatrix per block and the
// kernel streams K/V at memory speed. The MMAs run per warp: each warp stays an independent
// persistent worker with its own copy ring, as in decode.cu, and needs no tensor memory or
// CTA-wide synchronisation.
//
// Per warp and block: K and V of one (block, KV head) -- 16 rows of 128 elements -- arrive by one
// tensor-map TMA copy each (both 64-column halves, 128-byte swizzle, so ldmatrix reads are free of
// bank conflicts) into a ring of shared-memory stages tracked by mbarriers; the item's q rows come
// once by plain bulk copies. S = Q K^T as 16 MMAs (two 8-token n-tiles x 8 k-steps); the online
// softmax runs on the accumulator fragments in the log2 domain (a slot's scores sit in one lane
// quad); P, rounded to the input type, is reused in registers as the A operand of P V (16 MMAs
// over 8-column n-tiles, V fragments by transposing ldmatrix). Masking follows each slot's own
// causal limit; V rows past the item's last visible key are zeroed first (stale slots may hold
// anything). Items that cover part of a row write (unnormalised O, max, sum) partials for the
// log-sum-exp merge in decode.cu. Every wait is bounded, as in decode.cu.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "decode_mma.cuh"
#include "tma_host.h"

namespace pkv {
namespace {

using namespace mma;

constexpr int kMmaWarps = 2;                   // independent warps per CTA

// Shared memory: stages [kMmaWarps][NSTAGE], then mbarriers [kMmaWarps][NSTAGE], then each warp's ring
// of item indices [kMmaWarps][kFifo].
template <int NSTAGE>
constexpr int smem_bytes() { return 1024 + kMmaWarps * NSTAGE * (kStage + 8) + kMmaWarps * kFifo * 4; }

// Warp gw of the W launched starts with item gw; further items come from tickets (item W + ticket).
// The last warp to finish (a.work[1] counts them) resets both counters for the next launch.
template <typename T, int NSTAGE, bool T8>
__global__ void __launch_bounds__(kMmaWarps * 32)
    decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    unsigned char* wbase = smem + warp * NSTAGE * kStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kMmaWarps * NSTAGE * kStage) + warp * NSTAGE;
    volatile int* fifo = reinterpret_cast<int*>(smem + kMmaWarps * NSTAGE * (kStage + 8)) + warp * kFifo;
    griddep_wait();
    const int W = gridDim.x * kMmaWarps;
    (void)decode_warp<T, NSTAGE, T8>(a, &tm_k, &tm_v, wbase, bars, fifo, blockIdx.x * kMmaWarps + warp, W);
    // Every warp passes here exactly once on its way out.
    if (lane == 0 && atomicAdd(&a.work[1], 1) == W - 1) {
        atomicExch(&a.work[0], 0);
        atomicExch(&a.work[1], 0);
    }
}

template <typename T, int NSTAGE, bool T8>
cudaError_t launch_mma_t(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    const CUtensorMapDataType dt =
        std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const long long rows = (long long)a.num_blocks * a.num_kv_heads * kBlockSize;
    CUtensorMap mk, mv;
    if (!encode_block_halves(&mk, dt, a.k_pool, rows) || !encode_block_halves(&mv, dt, a.v_pool, rows))
        return cudaErrorInvalidValue;
    constexpr int smem = smem_bytes<NSTAGE>();
    static int per_sm_cache[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < 64) ? per_sm_cache[dev] : 0;
    if (per_sm == 0) {
        e = cudaFuncSetAttribute(decode_mma_kernel<T, NSTAGE, T8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_mma_kernel<T, NSTAGE, T8>, kMmaWarps * 32, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        if (dev >= 0 && dev < 64) per_sm_cache[dev] = per_sm;
    }
    const int need = (a.num_items + kMmaWarps - 1) / kMmaWarps;
    int grid = num_sms * per_sm;
    if (grid > need) grid = need;
    if (grid < 1) return cudaSuccess;
    return launch_k(a.pdl, decode_mma_kernel<T, NSTAGE, T8>, dim3(grid), dim3(kMmaWarps * 32), smem, s, a, mk, mv);
}

// Ring depth: 2 stages (24 KiB per warp, so 4 CTAs = 8 warps fit an SM; measured best on every
// configuration against 3 and 4), or PKV_DECODE_MMA_STAGES (2..4) as a tuning override.
inline int mma_stages() {
    static const int v = [] {
        const char* e = getenv("PKV_DECODE_MMA_STAGES");
        const int x = e ? atoi(e) : 0;
        return (x >= 2 && x <= 4) ? x : 2;
    }();
    return v;
}

template <typename T, bool T8>
cudaError_t launch_mma_s(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    switch (mma_stages()) {
        case 3: return launch_mma_t<T, 3, T8>(a, num_sms, s);
        case 4: return launch_mma_t<T, 4, T8>(a, num_sms, s);
        default: return launch_mma_t<T, 2, T8>(a, num_sms, s);
    }
}

// Items of at most 8 (row, head) slots run the transposed form (half the MMAs per block).
template <typename T>
cudaError_t launch_mma_k(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    return a.slots_per_item <= 8 ? launch_mma_s<T, true>(a, num_sms, s) : launch_mma_s<T, false>(a, num_sms, s);
}

}  // namespace

bool decode_mma_supported(int dtype, int head_dim) { return (dtype == 1 || dtype == 2) && head_dim == 128; }

cudaError_t launch_decode_mma(int dtype, const DecodeArgs& a, int num_sms, cudaStream_t s) {
    if (a.num_items <= 0) return cudaSuccess;
    if (!a.work) return cudaErrorInvalidValue;
    if ((long long)a.num_blocks * a.num_kv_heads * kBlockSize >= (1LL << 31) - 1) return cudaErrorInvalidValue;
    if (((uintptr_t)a.q | (uintptr_t)a.k_pool | (uintptr_t)a.v_pool) & 15) return cudaErrorInvalidValue;
    return dtype == 1 ? launch_mma_k<__half>(a, num_sms, s) : launch_mma_k<__nv_bfloat16>(a, num_sms, s);
}

}  // namespace pkv
