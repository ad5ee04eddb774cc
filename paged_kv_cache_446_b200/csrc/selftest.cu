// Device self-test entry point: evaluates the library's FMA-pipe exponential on given inputs so it
// can be compared with the hardware exp2 (no counterpart on the pages; a test aid).
#include "common.cuh"
#include "pkv.h"

namespace pkv {
namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    } else if (i < n) {
        y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
    }
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_selftest_exp2(const float* x, float* y, int n, pkv_stream_t stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return PKV_ERR_INVALID_ARG;
    if (n == 0) return PKV_OK;
    const int threads = 256, pairs = (n + 1) / 2;
    pkv::exp2_poly_kernel<<<(pairs + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
