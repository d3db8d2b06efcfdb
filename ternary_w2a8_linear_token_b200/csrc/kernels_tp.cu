// The pieces of the BitLinear forward that tensor-parallel sharding runs separately (page
// "BitNet：1-bit LLM推理框架技术实战指南", section on the distributed engine: a model split by
// layer or by tensor across devices). With a projection's K range split across ranks, each
// rank holds a slice of x and of every packed row. The per-token scale needs the amax of the
// whole row, so each rank reduces its slice (bitnet_act_amax), the ranks all-reduce the maxima,
// each rank quantises its slice with the global amax (bitnet_quant_act_amax) and contracts it
// with its slice of the weights (bitnet_linear_i32), the ranks sum the int32 partial
// accumulators (exact in any order), and the epilogue runs once on the sum (bitnet_dequant).
// Every step is the arithmetic of the fused forward, so the result equals bitnet_linear's bit
// for bit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr int kTpThreads = 256;

// amax[m] = max_k |x[m, k]| (exact: bf16 magnitudes order as unsigned integers). One warp per
// token, eight 8-value pieces in flight per lane.
__global__ void __launch_bounds__(kTpThreads) act_amax_kernel(const uint16_t* __restrict__ x,
                                                              int64_t M, int64_t K,
                                                              float* __restrict__ amax) {
    const int lane = threadIdx.x & 31;
    const int64_t m = int64_t(blockIdx.x) * (kTpThreads / 32) + (threadIdx.x >> 5);
    if (m >= M) return;
    const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
    const int64_t pieces = K >> 3;
    uint32_t mx = 0;
    for (int64_t c0 = 0; c0 < pieces; c0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t c = c0 + lane + 32 * u;
            v[u] = c < pieces ? row[c] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) mx = max(mx, absmax8_bits(v[u]));
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) amax[m] = bf16_lo(mx);
}

// q = clamp(rint(x * s_x), -128, 127) with s_x = 127 / max(amax[m], 1e-5) (binary32 divide):
// the per-token quantiser of bitnet_quant_act with the token's amax supplied. One thread per
// 8-value piece; the clamp never acts (|x| <= amax, see act_quant_device.cuh).
__global__ void __launch_bounds__(kTpThreads) quant_amax_kernel(const uint16_t* __restrict__ x,
                                                                const float* __restrict__ amax,
                                                                int64_t M, int64_t K,
                                                                int8_t* __restrict__ q,
                                                                float* __restrict__ s_x) {
    const int64_t pieces = K >> 3;
    const int64_t i = int64_t(blockIdx.x) * kTpThreads + threadIdx.x;
    if (i >= M * pieces) return;
    const int64_t m = i / pieces, c = i - m * pieces;
    const float s = __fdiv_rn(127.0f, fmaxf(amax[m], kActEps));
    const uint4 v = reinterpret_cast<const uint4*>(x + m * K)[c];
    reinterpret_cast<uint2*>(q + m * K)[c] = quant8(v, s);
    if (c == 0) s_x[m] = s;
}

// The dequant epilogue on its own: y = RN(RN(acc) * RN(s_w * RN(1 / s_x))) in binary32, then
// RNE to bf16 — the same rounding steps as the fused kernels' epilogues.
__global__ void __launch_bounds__(kTpThreads) dequant_kernel(const int32_t* __restrict__ acc,
                                                             int64_t M, int64_t N,
                                                             const float* __restrict__ s_x,
                                                             const float* __restrict__ s_w,
                                                             int per_row, void* __restrict__ y,
                                                             int out_kind) {
    const int64_t i = int64_t(blockIdx.x) * kTpThreads + threadIdx.x;
    if (i >= M * N) return;
    const int64_t m = i / N, n = i - m * N;
    const float f = __fmul_rn(per_row ? s_w[n] : s_w[0], __frcp_rn(s_x[m]));
    const float v = __fmul_rn(__int2float_rn(acc[i]), f);
    if (out_kind == 0)
        static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
    else
        static_cast<float*>(y)[i] = v;
}

unsigned blocks_for(int64_t n) { return static_cast<unsigned>((n + kTpThreads - 1) / kTpThreads); }

}  // namespace

cudaError_t launch_act_amax(const uint16_t* x, int64_t M, int64_t K, float* amax,
                            cudaStream_t stream) {
    act_amax_kernel<<<blocks_for(M * 32), kTpThreads, 0, stream>>>(x, M, K, amax);
    return cudaGetLastError();
}

cudaError_t launch_quant_amax(const uint16_t* x, const float* amax, int64_t M, int64_t K,
                              int8_t* q, float* s_x, cudaStream_t stream) {
    quant_amax_kernel<<<blocks_for(M * (K >> 3)), kTpThreads, 0, stream>>>(x, amax, M, K, q, s_x);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const int32_t* acc, int64_t M, int64_t N, const float* s_x,
                           const float* s_w, int per_row, void* y, int out_kind,
                           cudaStream_t stream) {
    dequant_kernel<<<blocks_for(M * N), kTpThreads, 0, stream>>>(acc, M, N, s_x, s_w, per_row, y,
                                                                   out_kind);
    return cudaGetLastError();
}

}  // namespace bitnet
