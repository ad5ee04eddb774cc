// Device helpers shared by the library's kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "internal.h"

namespace pkv {

constexpr unsigned FULL_MASK = 0xffffffffu;
// Bounded waits give up after this many SM clock cycles (about a second at B200 clocks) and
// record PKV_ERR_DEVICE_TIMEOUT instead of spinning forever.
constexpr long long WAIT_BUDGET_CYCLES = 2000000000LL;

__device__ __forceinline__ void record_error(DeviceError* e, int code, long long detail) {
    if (atomicCAS(&e->code, 0, code) == 0) atomicExch(reinterpret_cast<unsigned long long*>(&e->detail),
                                                      static_cast<unsigned long long>(detail));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase with the given parity to complete; false if the budget ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > WAIT_BUDGET_CYCLES) return false;
    }
    return true;
}

// ---- bulk asynchronous copies (TMA engine, no tensor map, no multicast) ----------------------
// Copies `bytes` (multiple of 16, both addresses 16-byte aligned) from global to this CTA's
// shared memory; completion is signalled as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Same, with an L2 eviction-priority hint (policy from createpolicy).
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Tiled 2-D tensor copy (TMA, tensor map in kernel-parameter or global memory, no multicast) of the
// box at element coordinates (x, y) into this CTA's shared memory, signalled on `bar`. x times the
// element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Orders this thread's generic-proxy shared-memory accesses before later async-proxy accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- math ----------------------------------------------------------------------------------
// 2^x via the PTX ex2.approx instruction (ex2(-inf) = +0).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for two values at once (offloads the MUFU unit, which the prefill softmax
// saturates). Range reduction: x = n + f with n = round(x) and f in [-1/2, 1/2], n obtained by
// adding 1.5 * 2^23 (the sum's low mantissa bits then hold n). 2^f comes from a degree-4 polynomial
// fitted here to 2^f on [-1/2, 1/2] for minimum relative error (weighted least squares on
// Chebyshev nodes with iterative reweighting); evaluated in fp32 its relative error is below
// 3e-6. 2^n is added into the exponent field. Inputs are clamped to -126 (results below 2^-126
// flush towards 0); inputs must be at most 127.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float kC0 = 0.99999928474426270f, kC1 = 0.69312179088592530f, kC2 = 0.24024748802185059f,
                    kC3 = 0.055917855352163315f, kC4 = 0.009569923393428326f;
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
    const float2 r = __fadd2_rn(t, make_float2(-kRound, -kRound));
    const float2 f = __fadd2_rn(x, make_float2(-r.x, -r.y));
    float2 p = __ffma2_rn(make_float2(kC4, kC4), f, make_float2(kC3, kC3));
    p = __ffma2_rn(p, f, make_float2(kC2, kC2));
    p = __ffma2_rn(p, f, make_float2(kC1, kC1));
    p = __ffma2_rn(p, f, make_float2(kC0, kC0));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// ---- element types ------------------------------------------------------------------------
// Unpack one 16-byte chunk into fp32 values.
template <typename T>
struct Chunk;

template <>
struct Chunk<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <>
struct Chunk<__half> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    // bfloat16 -> fp32 is exact: the 16 bits become the high half of the fp32 word.
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// Two fp32 values rounded (to nearest even) to a 16-bit type T and packed, `lo` in the low half.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (std::is_same<T, __half>::value) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
}
// The two 16-bit values of a packed word as fp32 (low half first).
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if constexpr (std::is_same<T, __half>::value) {
        return __half22float2(*reinterpret_cast<const __half2*>(&w));
    } else {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
}

// A CUDA-core work item, read with two 16-byte loads.
__device__ __forceinline__ DecodeItem load_item(const DecodeItem* items, int i) {
    const int4* p = reinterpret_cast<const int4*>(items + i);
    const int4 a = __ldg(p), b = __ldg(p + 1);
    DecodeItem it;
    it.row = a.x;
    it.req = a.y;
    it.kv_head = (int16_t)(a.z & 0xffff);         // low half of the third word
    it.num_rows = (int16_t)((unsigned)a.z >> 16); // high half
    it.head0 = a.w;
    it.blk_begin = b.x;
    it.blk_end = b.y;
    it.limit = b.z;
    it.partial = b.w;
    return it;
}

// ---- programmatic dependent launch -------------------------------------------------------------
// Kernels are launched so that they may start while the previous kernel on the stream finishes;
// each calls griddep_wait() before its first global read or write, which returns once that
// predecessor has completed and its memory is visible (immediately when launched normally).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kernel` on `s`, with the programmatic-stream-serialisation attribute when `pdl` is set
// (the kernel may then start while its predecessor on `s` finishes; it waits in griddep_wait()).
// Launches that follow an event wait on a side stream go without it.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
    return launch_k(true, kernel, grid, block, smem, s, std::forward<Args>(args)...);
}

}  // namespace pkv
