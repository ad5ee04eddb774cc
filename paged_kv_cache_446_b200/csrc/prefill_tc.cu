// tcgen05 chunked-prefill tiles (not yet enabled: every row goes to the CUDA-core kernel).
#include "common.cuh"

namespace pkv {

bool prefill_tc_supported(int, int, int) { return false; }

cudaError_t launch_prefill_tc(int, const PrefillArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace pkv
