// Paged attention without any device allocation: the scratch lives in a fixed, file-scope device
// array instead of a caller-provided workspace.
//
// Who needs this: callers that may not call cudaMalloc at the point where they run attention --
// for example an engine whose memory manager has already reserved nearly all of HBM for its KV
// pool and treats any further allocation as a failure, a plugin hosted by a runtime that owns
// every device allocation, or code that runs where the CUDA runtime forbids or stalls on
// allocation calls. They still own q, the pools, the tables and the output; only the planner's
// work lists and the split-K partials move into the library's own array.
//
// The array (PKV_STATIC_WS_BYTES) is part of this file's device module: every GPU that loads it
// holds the memory until the process exits. Its device address is looked up with
// cudaGetSymbolAddress on the first call made with a device current; the address is kept per CUDA
// context and looked up again when the device's current context is a different one (for example
// after cudaDeviceReset). All calls share
// the one array and it keeps the contents of the last call: calls that can overlap on the GPU
// (different streams, or different host threads) race on it and must be serialised by the caller.
// Nothing in it has to start at zero -- each call writes every byte its kernels read (the uploaded
// work lists, then the partials) before reading it.
#include <cuda.h>

#include <cstdio>
#include <mutex>

#include "internal.h"
#include "pkv.h"

namespace pkv {
namespace {

static __device__ __align__(256) unsigned char g_static_ws[PKV_STATIC_WS_BYTES];

// Device address of g_static_ws for the current device and context (host code may not use the
// symbol itself: in host code its name is a host-side stand-in, not a device address).
void* static_ws_address(pkv_status* st) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    static unsigned long long ctx_of[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        set_last_error("static workspace: no usable current device");
        *st = PKV_ERR_CUDA;
        return nullptr;
    }
    const unsigned long long ctx = current_context_id();  // 0 while no context is current yet
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess || !p) {
            set_last_error("static workspace: cudaGetSymbolAddress failed");
            *st = PKV_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
        ctx_of[dev] = current_context_id();  // the lookup made the device's context current
    }
    *st = PKV_OK;
    return addr[dev];
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attention_static_ws(
    const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs, int num_q_heads, int num_kv_heads,
    int head_dim, pkv_dtype dtype, const pkv_plan_options* opts, void* out, const void* q, const void* k_pool,
    const void* v_pool, const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    const int32_t* query_start_loc, int num_blocks, float scale, pkv_stream_t stream) {
    pkv_status st = PKV_OK;
    void* ws = pkv::static_ws_address(&st);
    if (!ws) return st;
    // One planning pass: the planner refuses a batch whose scratch exceeds the array before it
    // uploads anything.
    pkv_plan plan;
    st = pkv_attention_plan(h_query_start_loc, h_context_lens, num_reqs, num_q_heads, num_kv_heads, head_dim, dtype,
                            opts, ws, PKV_STATIC_WS_BYTES, &plan, stream);
    if (st == PKV_ERR_WORKSPACE_TOO_SMALL) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "batch needs %lld bytes of scratch, above the static workspace limit of %zu bytes "
                 "(use pkv_attention_plan with a caller workspace, or larger split_blocks)",
                 (long long)plan.ws_bytes, (size_t)PKV_STATIC_WS_BYTES);
        pkv::set_last_error(msg);
        return st;
    }
    if (st != PKV_OK) return st;
    return pkv_paged_attention(out, q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens,
                               query_start_loc, num_blocks, scale, &plan, ws, PKV_STATIC_WS_BYTES, stream);
}
