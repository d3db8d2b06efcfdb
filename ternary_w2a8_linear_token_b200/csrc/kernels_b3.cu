// Base-3 weight format, five ternary weights per byte (page "将 BitNet 三元查找表集成到自定义
// Triton 内核中", step 1 of its recipe: ternary values packed into uint8 bitmaps, 4-5 per byte;
// 3^5 = 243 <= 256, so 1.6 bits per weight against the 2-bit format's 2): the packing kernel.
// The one-token GEMV that reads it is the grid-stride kernel of kernels_gemv_gs.cu.
//
// Layout: a row is cut into chunks of 80 weights (16 bytes); byte p of chunk c holds weights
// k = 80c + 16d + p (d = 0..4) as sum_d (t + 1) 3^d; weights past K count as 0; a row takes
// 16 ceil(K / 80) bytes. Byte p of a chunk thus carries position p of the chunk's five
// 16-weight groups, so a chunk decodes into five 32-bit words of the 2-bit format.
#include <cuda_runtime.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

// One output byte per thread: the five weights of byte p of chunk c of row n.
__global__ void __launch_bounds__(256) pack_b3_kernel(const int8_t* __restrict__ t, int64_t N,
                                                      int64_t K, uint8_t* __restrict__ packed) {
    const int64_t rb = b3_row_bytes(K);
    const int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x;
    if (i >= N * rb) return;
    const int64_t n = i / rb, j = i - n * rb;
    const int64_t c = j >> 4, p = j & 15;
    unsigned byte = 0, place = 1;
#pragma unroll
    for (int d = 0; d < 5; ++d) {
        const int64_t k = 80 * c + 16 * d + p;
        const int w = k < K ? int(t[n * K + k]) : 0;
        byte += unsigned(w + 1) * place;
        place *= 3u;
    }
    packed[i] = uint8_t(byte);
}

}  // namespace

cudaError_t launch_pack_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                           cudaStream_t stream) {
    const int64_t total = N * b3_row_bytes(K);
    pack_b3_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(t, N, K, packed);
    return cudaGetLastError();
}

}  // namespace bitnet
