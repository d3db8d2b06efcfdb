// bitnet_linear_noalloc: bitnet_linear for callers that cannot allocate device memory.
//
// Some callers must not allocate device memory while they run: a serving loop where
// cudaMalloc can synchronise the device and stall every other stream, or a plug-in hosted by
// a runtime that owns all device memory and forbids allocations of its own. For them this
// entry point takes no workspace argument: the tensor-core path's scratch (quantised
// activations, per-token scales and the split-K area) lives in the file-scope device array
// below, which every GPU that loads the library holds until the process exits. Nothing here
// calls cudaMalloc, cudaFree or an allocating library routine.
//
// The array's name is only a host-side stand-in in host code; its device address is looked
// up once per device with cudaGetSymbolAddress, with that device current, on the first call
// made on that device, and cached for the life of the process (so the library must not be
// used on a device again after cudaDeviceReset of that device).
#include <cuda_runtime.h>

#include <mutex>

#include "bitnet.h"
#include "bitnet_internal.h"

static __device__ __align__(256) uint8_t g_noalloc_scratch[BITNET_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (nullptr on failure).
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" bitnet_status bitnet_linear_noalloc(const uint16_t* x, int64_t M, int64_t K,
                                               const uint8_t* packed, const float* s_w,
                                               bitnet_scale_mode mode, int64_t N, void* y,
                                               bitnet_out_dtype out_dtype, void* stream) {
    if (M < 1 || K < 1) return BITNET_ERR_SHAPE;
    void* scratch = scratch_on_current_device();
    if (!scratch) return BITNET_ERR_CUDA;
    // The path bitnet_linear takes with this array as its workspace: the decode GEMV needs no
    // scratch; every other call runs the tensor-core path, whose whole workspace (including
    // the split-K area) must fit the fixed array.
    const bool gemv = bitnet::use_gemv(M, K, BITNET_PATH_AUTO, scratch,
                                       size_t(BITNET_NOALLOC_SCRATCH_BYTES));
    if (!gemv && bitnet_linear_workspace_size(M, K) > size_t(BITNET_NOALLOC_SCRATCH_BYTES))
        return BITNET_ERR_WORKSPACE;
    // No part of the scratch has to start at zero: the quantiser writes every byte the
    // GEMM reads in the same call, and clears the split-K counters and tiles it uses.
    return bitnet_linear_ex(x, M, K, packed, s_w, mode, N, y, out_dtype, scratch,
                            size_t(BITNET_NOALLOC_SCRATCH_BYTES), BITNET_PATH_AUTO, stream);
}
