// Integer arithmetic rate probes for the roofline of the one-token GEMV (not part of the
// BitLinear forward). The decode GEMV's products run on dp4a (four int8 products and a sum per
// lane instruction) or on legacy warp-level int8 MMA; how many of those an SM retires per clock
// sets the arithmetic ceiling that the weight bytes are weighed against (the ridge in tokens
// per call). Each probe kernel issues nothing but that instruction in independent chains, so a
// launch's duration measures its issue rate.
#include <cuda_runtime.h>

#include <cstdint>

#include "bitnet.h"

namespace {

constexpr int kProbeThreads = 256;
constexpr int kDp4aChains = 8;  // independent accumulators per thread
constexpr int kMmaChains = 4;   // independent accumulator tiles per warp

// Each chain feeds its own result back as the next first operand, so no product can be
// hoisted out of the loop; eight chains per thread cover the instruction latency.
__global__ void __launch_bounds__(kProbeThreads) dp4a_rate_kernel(int64_t iters, int seed,
                                                                  int32_t* __restrict__ out) {
    int acc[kDp4aChains];
    const int b = seed ^ int(threadIdx.x * 0x01010101u);
#pragma unroll
    for (int c = 0; c < kDp4aChains; ++c) acc[c] = seed + c;
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
        for (int c = 0; c < kDp4aChains; ++c) acc[c] = __dp4a(acc[c], b, acc[c]);
    }
    int r = 0;
#pragma unroll
    for (int c = 0; c < kDp4aChains; ++c) r ^= acc[c];
    if (threadIdx.x == 0 || r == 0x7FFFFFFF) out[blockIdx.x] = r;  // keeps every chain live
}

// m16n8k32 s8 x s8 -> s32: 4096 multiply-adds per warp instruction; four accumulator tiles in
// flight per warp.
__global__ void __launch_bounds__(kProbeThreads) mma_s8_rate_kernel(int64_t iters, int seed,
                                                                    int32_t* __restrict__ out) {
    const uint32_t a0 = uint32_t(seed) ^ threadIdx.x, a1 = a0 * 3u, a2 = a0 * 5u, a3 = a0 * 7u;
    const uint32_t b0 = a0 ^ 0x5A5A5A5Au, b1 = a0 ^ 0x3C3C3C3Cu;
    int32_t d[kMmaChains][4];
#pragma unroll
    for (int c = 0; c < kMmaChains; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) d[c][j] = c + j;
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
        for (int c = 0; c < kMmaChains; ++c)
            asm volatile(
                "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
                "{%8,%9}, {%0,%1,%2,%3};\n"
                : "+r"(d[c][0]), "+r"(d[c][1]), "+r"(d[c][2]), "+r"(d[c][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    int32_t r = 0;
#pragma unroll
    for (int c = 0; c < kMmaChains; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) r ^= d[c][j];
    if (threadIdx.x == 0 || r == 0x7FFFFFFF) out[blockIdx.x] = r;
}

}  // namespace

extern "C" int64_t bitnet_probe_int_ops(int32_t kind, int32_t blocks, int64_t iters) {
    if (blocks < 1 || iters < 1) return 0;
    const int64_t per_iter =
        kind == BITNET_PROBE_DP4A ? int64_t(kProbeThreads) * kDp4aChains * 8  // 4 MACs each
        : kind == BITNET_PROBE_MMA_S8
            ? int64_t(kProbeThreads / 32) * kMmaChains * 16 * 8 * 32 * 2  // per warp instruction
            : 0;
    return per_iter * blocks * iters;
}

extern "C" bitnet_status bitnet_probe_int_rate(int32_t kind, int32_t blocks, int64_t iters,
                                               int32_t* out, void* stream) {
    if (kind != BITNET_PROBE_DP4A && kind != BITNET_PROBE_MMA_S8) return BITNET_ERR_UNSUPPORTED;
    if (blocks < 1 || blocks > 65535 || iters < 1 || iters > (int64_t(1) << 24))
        return BITNET_ERR_SHAPE;
    if (!out) return BITNET_ERR_NULL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kind == BITNET_PROBE_DP4A)
        dp4a_rate_kernel<<<blocks, kProbeThreads, 0, s>>>(iters, 0x1234567, out);
    else
        mma_s8_rate_kernel<<<blocks, kProbeThreads, 0, s>>>(iters, 0x1234567, out);
    return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
