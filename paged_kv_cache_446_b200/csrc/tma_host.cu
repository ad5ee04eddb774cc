// Tensor-map encoding through the driver entry point (host code).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tma_host.h"

namespace pkv {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

bool encode_tiled(CUtensorMap* m, CUtensorMapDataType t, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, t, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_block_halves(CUtensorMap* m, CUtensorMapDataType t, const void* base, long long rows) {
    const cuuint64_t dims[3] = {64, (cuuint64_t)rows, 2};
    const cuuint64_t strides[2] = {128 * 2, 64 * 2};
    const cuuint32_t box[3] = {64, 16, 2};
    return encode_tiled(m, t, 3, base, dims, strides, box);
}

}  // namespace pkv
