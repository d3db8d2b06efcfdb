// Watchdog self-test (failure detection): one thread waits on an mbarrier that nothing
// completes, through the same bounded wait the tensor-core kernel uses for every ring and
// accumulator handoff. When the limit expires the wait records a watchdog bit in the
// library's device error word and returns; the kernel then exits normally, so the context
// stays usable and the host learns of the failure from bitnet_check_device_errors.
#include <cuda_runtime.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

__global__ void selftest_wait_kernel(int32_t* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Phase 0 of `bar` never completes: nothing arrives on it.
        mbar_wait_bounded(&bar, 0, err, kErrSelfTest, &abort_flag, limit_ns);
    }
}

}  // namespace
}  // namespace bitnet

extern "C" bitnet_status bitnet_selftest_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns < 1000000 || limit_ns > 2000000000) return BITNET_ERR_UNSUPPORTED;
    int32_t* err = bitnet::device_error_word();
    if (!err) return BITNET_ERR_CUDA;
    bitnet::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        err, static_cast<uint64_t>(limit_ns));
    return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
