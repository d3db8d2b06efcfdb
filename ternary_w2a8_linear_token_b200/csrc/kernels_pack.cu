// Offline weight step: absmean scale, ternarisation and 2-bit packing
// (page "BitNet 深度实战", section 2.4 "量化函数的细节" for the quantiser, section 4.3
// "位打包（Bit Packing）存储" for the bit order; code = t + 1).
//
// The scale is a binary64 sum of |W| in index order (row by row, k ascending), so the
// row sums run one thread per row; the per-tensor total is a single-thread sequential
// sum over the rows. Packing is off the per-token path, so this order (chosen for
// bit-reproducible scales) costs nothing that matters.
#include <cuda_runtime.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr float kEps = 1e-5f;

// r_n = sum_k |W[n,k]| in binary64, k ascending. Per-row mode writes the clamped mean.
__global__ void __launch_bounds__(128) absmean_rows_kernel(const float* __restrict__ W, int64_t N,
                                                           int64_t K, int per_row,
                                                           float* __restrict__ s_w,
                                                           double* __restrict__ row_sums) {
    const int64_t n = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (n >= N) return;
    const float4* row = reinterpret_cast<const float4*>(W + n * K);
    double r = 0.0;
    for (int64_t c = 0; c < K / 4; ++c) {
        const float4 v = row[c];
        r += static_cast<double>(fabsf(v.x));
        r += static_cast<double>(fabsf(v.y));
        r += static_cast<double>(fabsf(v.z));
        r += static_cast<double>(fabsf(v.w));
    }
    if (per_row) {
        const float mean = __double2float_rn(__ddiv_rn(r, static_cast<double>(K)));
        s_w[n] = fmaxf(mean, kEps);
    } else {
        row_sums[n] = r;
    }
}

// Per-tensor scale: R = r_0 + ... + r_{N-1} (n ascending), s = max((float)(R / (N K)), eps).
__global__ void absmean_total_kernel(const double* __restrict__ row_sums, int64_t N, int64_t K,
                                     float* __restrict__ s_w) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) total += row_sums[n];
    const double count = static_cast<double>(N) * static_cast<double>(K);
    s_w[0] = fmaxf(__double2float_rn(__ddiv_rn(total, count)), kEps);
}

// One thread packs 16 weights into one 32-bit word: weight e of the word (k = 16w + e)
// goes to bits 2e..2e+1, which is byte e/4, bits 2(e%4) of the row's byte stream.
__global__ void __launch_bounds__(256) ternarize_pack_kernel(const float* __restrict__ W,
                                                             int64_t N, int64_t K, int per_row,
                                                             const float* __restrict__ s_w,
                                                             uint8_t* __restrict__ packed) {
    const int64_t words_per_row = K / 16;
    const int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (idx >= N * words_per_row) return;
    const int64_t n = idx / words_per_row;
    const int64_t wi = idx - n * words_per_row;
    const float s = per_row ? s_w[n] : s_w[0];
    const float4* src = reinterpret_cast<const float4*>(W + n * K + wi * 16);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 v = src[j];
        const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float r = rintf(__fdiv_rn(vals[c], s));
            r = fminf(fmaxf(r, -1.0f), 1.0f);
            const uint32_t code = static_cast<uint32_t>(static_cast<int>(r) + 1);
            word |= code << (2 * (4 * j + c));
        }
    }
    reinterpret_cast<uint32_t*>(packed + n * (K / 4))[wi] = word;
}

// Packs int8 ternary weights: 16 values (one 16-byte load) into one 32-bit word.
__global__ void __launch_bounds__(256) pack_ternary_kernel(const int8_t* __restrict__ t, int64_t N,
                                                           int64_t K, uint8_t* __restrict__ packed) {
    const int64_t words_per_row = K / 16;
    const int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (idx >= N * words_per_row) return;
    const int64_t n = idx / words_per_row;
    const int64_t wi = idx - n * words_per_row;
    const uint4 v = *reinterpret_cast<const uint4*>(t + n * K + wi * 16);
    const uint32_t parts[4] = {v.x, v.y, v.z, v.w};
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int w = static_cast<int8_t>((parts[j] >> (8 * c)) & 0xFFu);
            word |= (static_cast<uint32_t>(w + 1) & 3u) << (2 * (4 * j + c));
        }
    }
    reinterpret_cast<uint32_t*>(packed + n * (K / 4))[wi] = word;
}

}  // namespace

cudaError_t launch_pack_weights(const float* W, int64_t N, int64_t K, int per_row,
                                uint8_t* packed, float* s_w, cudaStream_t stream) {
    // Per-tensor mode parks the N binary64 row sums in `packed` (8N <= N*K/4 for K >= 32)
    // until the total is formed; the pack kernel then overwrites them.
    double* row_sums = reinterpret_cast<double*>(packed);
    const unsigned rows_blocks = static_cast<unsigned>((N + 127) / 128);
    absmean_rows_kernel<<<rows_blocks, 128, 0, stream>>>(W, N, K, per_row, s_w, row_sums);
    if (!per_row) absmean_total_kernel<<<1, 32, 0, stream>>>(row_sums, N, K, s_w);
    const int64_t words = N * (K / 16);
    ternarize_pack_kernel<<<static_cast<unsigned>((words + 255) / 256), 256, 0, stream>>>(
        W, N, K, per_row, s_w, packed);
    return cudaGetLastError();
}

cudaError_t launch_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                cudaStream_t stream) {
    const int64_t words = N * (K / 16);
    pack_ternary_kernel<<<static_cast<unsigned>((words + 255) / 256), 256, 0, stream>>>(t, N, K,
                                                                                       packed);
    return cudaGetLastError();
}

}  // namespace bitnet
