// Per-token absmax int8 activation quantiser (page "BitNet-Triton", section
// "技术架构：融合内核的三重优化", item 3 "融合激活量化": one launch instead of a chain of
// framework ops; page "BitNet 1-bit LLM推理优化", section 3.2 "激活量化策略").
//   amax = max_k |x[m,k]|, s_x = 127 / max(amax, 1e-5), q = clamp(rint(x * s_x), -128, 127).
//
// amax is reduced over the bf16 bit patterns (|x| ordered as an unsigned integer, so it is
// exact). Rows of K <= 4096 take one warp each and stay in registers (x read once); rows of
// 4096 < K <= 14336 take four warps each, also in registers; longer rows take one warp and
// two passes (the second an L1/L2 hit). With a per-tensor scale ("BitNet 1-bit LLM推理优化"
// section 2.2, I2_S), amax_parts_kernel first writes partial maxima of the whole input and
// every warp reduces those instead of its row; with block maxima from x's producer (the
// SwiGLU epilogue's maxima of |h| over 16 outputs), every warp reduces its token's I/16
// maxima instead. Two output layouts:
//  - natural (M, K) int8, the public bitnet_quant_act result;
//  - permuted, the operand layout of the tensor-core path: inside every group of 16
//    values along K, byte 4i + b holds k = 4b + i. That is the order in which a packed
//    32-bit weight word unpacks with shifts and masks alone ((w >> 2i) & 0x03030303
//    yields k = i, 4+i, 8+i, 12+i), so the weights need no byte shuffles. Adjacent lanes
//    own the two 8-value halves of a group and swap 16-bit pieces with one shuffle.
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr float kEps = kActEps;
constexpr int kThreads = 256;

// Per-tensor activation scale ("BitNet 1-bit LLM推理优化" §2.2, I2_S; §3.2): the amax of the
// whole input is the maximum of the partial maxima amax_parts_kernel wrote (whole warp).
__device__ __forceinline__ uint32_t parts_max(const uint32_t* __restrict__ parts, int n, int lane) {
    uint32_t m = 0;
    for (int i = lane; i < n; i += 32) m = max(m, parts[i]);
    return __reduce_max_sync(0xFFFFFFFFu, m);
}

// A token's amax from the maxima of its K / 16 blocks of 16 values (bf16 magnitude bits), as
// the SwiGLU epilogue writes them for its output h (whole warp). K % 64 == 0, so a token's
// K / 16 values start on an 8-byte boundary and are read four at a time.
__device__ __forceinline__ uint32_t tok_parts_max(const uint16_t* __restrict__ parts, int64_t K,
                                                  int lane) {
    const uint2* p = reinterpret_cast<const uint2*>(parts);
    const int64_t n = K / 64;
    uint32_t m = 0;  // two 16-bit maxima
#pragma unroll 4
    for (int64_t i = lane; i < n; i += 32) {
        const uint2 w = p[i];
        m = __vmaxu2(m, __vmaxu2(w.x, w.y));
    }
    return __reduce_max_sync(0xFFFFFFFFu, max(m & 0xFFFFu, m >> 16));
}

// One warp per token row; each lane keeps 8 loads in flight. Pass 1 finds amax, pass 2
// re-reads the row (an L1/L2 hit) and writes q.
constexpr int kRowsPerCta = kThreads / 32;
constexpr int kUnroll = 8;
constexpr int kRegPieces = 16;  // rows of up to 32 * 16 pieces (K <= 4096) stay in registers

__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const uint16_t* __restrict__ x,
                                                              const int8_t* __restrict__ q_in,
                                                              int64_t M, int64_t K,
                                                              int8_t* __restrict__ q,
                                                              float* __restrict__ s_x,
                                                              float* __restrict__ r_x,
                                                              int permuted,
                                                              uint4* __restrict__ zero,
                                                              int64_t zero_words,
                                                              int32_t* __restrict__ qsum,
                                                              const uint32_t* __restrict__ amax_parts,
                                                              int n_parts,
                                                              const uint16_t* __restrict__ tok_parts) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t m = int64_t(blockIdx.x) * kRowsPerCta + warp;
    const int64_t pieces = K / 8;  // 8 values per piece; K % 64 == 0 so pieces % 8 == 0

    pdl_wait();
    pdl_trigger();
    // Clear the consumer GEMM's split-K area (counters and accumulation tiles) for this call.
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < zero_words;
         i += int64_t(gridDim.x) * kThreads)
        zero[i] = make_uint4(0u, 0u, 0u, 0u);
    if (m >= M) return;  // whole warp leaves together

    float s = 0.0f;
    const uint4* xr = reinterpret_cast<const uint4*>(x + m * K);
    int8_t* qr = q + m * K;
    if (q_in == nullptr && pieces <= 32 * kRegPieces) {
        // Short rows (K <= 4096): the whole row stays in registers; one read of x.
        uint4 v[kRegPieces];
#pragma unroll
        for (int u = 0; u < kRegPieces; ++u) {
            const int64_t c = u * 32 + lane;
            v[u] = c < pieces ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t mx = 0;
#pragma unroll
        for (int u = 0; u < kRegPieces; ++u) mx = max(mx, absmax8_bits(v[u]));
        // The token's amax: its row's, the whole input's (per-tensor parts) or the maximum of
        // the block maxima that x's producer wrote.
        if (tok_parts)
            mx = tok_parts_max(tok_parts + m * (K / 16), K, lane);
        else if (amax_parts)
            mx = parts_max(amax_parts, n_parts, lane);
        else
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        s = __fdiv_rn(127.0f, fmaxf(bf16_lo(mx), kEps));
        if (lane == 0) {
            if (s_x) s_x[m] = s;
            if (r_x) r_x[m] = __frcp_rn(s);
        }
        int qs = 0;  // this lane's share of sum_k q (padding pieces quantise to 0)
#pragma unroll
        for (int u = 0; u < kRegPieces; ++u) {
            if (u * 32 >= pieces) break;  // warp-uniform
            const int64_t c = u * 32 + lane;
            const uint2 nat = quant8(v[u], s);
            qs = __dp4a(int(nat.x), 0x01010101, __dp4a(int(nat.y), 0x01010101, qs));
            const uint2 out = permuted ? permute_group_half(nat, lane & 1) : nat;
            if (c < pieces) reinterpret_cast<uint2*>(qr)[c] = out;
        }
        if (qsum) {
            qs = __reduce_add_sync(0xFFFFFFFFu, qs);
            if (lane == 0) qsum[m] = qs;
        }
        return;
    }
    if (q_in == nullptr) {
        uint32_t mx = 0;
        for (int64_t c0 = 0; c0 < pieces; c0 += 32 * kUnroll) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                v[u] = c < pieces ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) mx = max(mx, absmax8_bits(v[u]));
        }
        if (tok_parts)
            mx = tok_parts_max(tok_parts + m * (K / 16), K, lane);
        else if (amax_parts)
            mx = parts_max(amax_parts, n_parts, lane);
        else
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        s = __fdiv_rn(127.0f, fmaxf(bf16_lo(mx), kEps));
        if (lane == 0) {
            if (s_x) s_x[m] = s;
            if (r_x) r_x[m] = __frcp_rn(s);
        }
    }

    int qs = 0;
    for (int64_t c0 = 0; c0 < pieces; c0 += 32 * kUnroll) {
        uint2 nat[kUnroll];
        if (q_in == nullptr) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                v[u] = c < pieces ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) nat[u] = quant8(v[u], s);
        } else {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                nat[u] = c < pieces ? reinterpret_cast<const uint2*>(q_in + m * K)[c]
                                    : make_uint2(0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t c = c0 + u * 32 + lane;  // c0 + u*32 is even: lane pairs share a group
            qs = __dp4a(int(nat[u].x), 0x01010101, __dp4a(int(nat[u].y), 0x01010101, qs));
            const uint2 out = permuted ? permute_group_half(nat[u], lane & 1) : nat[u];
            if (c < pieces) reinterpret_cast<uint2*>(qr)[c] = out;
        }
    }
    if (qsum) {
        qs = __reduce_add_sync(0xFFFFFFFFu, qs);
        if (lane == 0) qsum[m] = qs;
    }
}

// Rows of 4096 < K <= 14336: four warps per row, each thread holding up to 14 pieces of 8
// values in registers, so x is read once (the one-warp kernel above takes two passes there).
constexpr int kLongThreads = 256;
constexpr int kLongRowThreads = 128;
constexpr int kLongRows = kLongThreads / kLongRowThreads;
constexpr int kLongPieces = 14;
constexpr int64_t kLongMaxK = int64_t(kLongRowThreads) * kLongPieces * 8;

__global__ void __launch_bounds__(kLongThreads) quant_long_rows_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int8_t* __restrict__ q,
    float* __restrict__ s_x, float* __restrict__ r_x, int permuted, uint4* __restrict__ zero,
    int64_t zero_words, int32_t* __restrict__ qsum, const uint32_t* __restrict__ amax_parts,
    int n_parts, const uint16_t* __restrict__ tok_parts) {
    __shared__ uint32_t s_mx[kLongRows][kLongRowThreads / 32];
    __shared__ int32_t s_qs[kLongRows][kLongRowThreads / 32];
    const int row = threadIdx.x / kLongRowThreads;
    const int t = threadIdx.x % kLongRowThreads;
    const int lane = threadIdx.x & 31;
    const int64_t m = int64_t(blockIdx.x) * kLongRows + row;
    const bool active = m < M;
    const int64_t pieces = K / 8;

    pdl_wait();
    pdl_trigger();
    for (int64_t i = int64_t(blockIdx.x) * kLongThreads + threadIdx.x; i < zero_words;
         i += int64_t(gridDim.x) * kLongThreads)
        zero[i] = make_uint4(0u, 0u, 0u, 0u);
    if (int64_t(blockIdx.x) * kLongRows >= M) return;  // a CTA added for the clearing only

    const uint4* xr = reinterpret_cast<const uint4*>(x + (active ? m : 0) * K);
    uint4 v[kLongPieces];
#pragma unroll
    for (int u = 0; u < kLongPieces; ++u) {
        const int64_t c = int64_t(u) * kLongRowThreads + t;
        v[u] = (active && c < pieces) ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t all = 0;
    if (tok_parts) {
        // the block maxima written by x's producer: no reduction across the row's warps
        all = tok_parts_max(tok_parts + (active ? m : 0) * (K / 16), K, lane);
    } else {
        uint32_t mx = 0;
#pragma unroll
        for (int u = 0; u < kLongPieces; ++u) mx = max(mx, absmax8_bits(v[u]));
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) s_mx[row][t >> 5] = mx;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kLongRowThreads / 32; ++w) all = max(all, s_mx[row][w]);
        if (amax_parts) all = parts_max(amax_parts, n_parts, lane);  // one scale per tensor
    }
    const float s = __fdiv_rn(127.0f, fmaxf(bf16_lo(all), kEps));
    if (active && t == 0) {
        if (s_x) s_x[m] = s;
        if (r_x) r_x[m] = __frcp_rn(s);
    }
    int8_t* qr = q + (active ? m : 0) * K;
    int qs = 0;  // padding pieces quantise to 0
#pragma unroll
    for (int u = 0; u < kLongPieces; ++u) {
        if (int64_t(u) * kLongRowThreads >= pieces) break;  // uniform over the row's warps
        const int64_t c = int64_t(u) * kLongRowThreads + t;  // lane pairs share a 16-group
        const uint2 nat = quant8(v[u], s);
        qs = __dp4a(int(nat.x), 0x01010101, __dp4a(int(nat.y), 0x01010101, qs));
        const uint2 out = permuted ? permute_group_half(nat, lane & 1) : nat;
        if (active && c < pieces) reinterpret_cast<uint2*>(qr)[c] = out;
    }
    if (qsum) {  // uniform over the CTA
        qs = __reduce_add_sync(0xFFFFFFFFu, qs);
        if (lane == 0) s_qs[row][t >> 5] = qs;
        __syncthreads();
        if (active && t == 0) {
            int32_t tot = 0;
#pragma unroll
            for (int w = 0; w < kLongRowThreads / 32; ++w) tot += s_qs[row][w];
            qsum[m] = tot;
        }
    }
}

// Partial maxima of |x| over the whole input (bf16 bit patterns, |x| ordered as unsigned
// integers): CTA b writes the maximum of its grid-stride share to parts[b]. The per-tensor
// quantiser then reduces the parts; no zeroing or atomics are needed.
constexpr int kAmaxThreads = 256;
constexpr int64_t kZeroBytesPerCta = 16 * 1024;  // split-K area cleared per quantiser CTA
constexpr int kAmaxUnroll = 4;

__global__ void __launch_bounds__(kAmaxThreads) amax_parts_kernel(const uint4* __restrict__ x,
                                                                  int64_t pieces,
                                                                  uint32_t* __restrict__ parts) {
    __shared__ uint32_t s_w[kAmaxThreads / 32];
    pdl_wait();
    pdl_trigger();
    uint32_t mx = 0;
    const int64_t stride = int64_t(gridDim.x) * kAmaxThreads;
    for (int64_t c0 = int64_t(blockIdx.x) * kAmaxThreads + threadIdx.x; c0 < pieces;
         c0 += stride * kAmaxUnroll) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {  // independent loads in flight
            const int64_t c = c0 + u * stride;
            v[u] = c < pieces ? x[c] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) mx = max(mx, absmax8_bits(v[u]));
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0;
#pragma unroll
        for (int w = 0; w < kAmaxThreads / 32; ++w) a = max(a, s_w[w]);
        parts[blockIdx.x] = a;
    }
}

}  // namespace

int amax_parts_count(int64_t M, int64_t K) {
    const int64_t pieces = M * K / 8;
    const int64_t per_cta = int64_t(kAmaxThreads) * kAmaxUnroll * 2;
    int64_t n = (pieces + per_cta - 1) / per_cta;
    if (n > kMaxAmaxParts) n = kMaxAmaxParts;
    return static_cast<int>(n < 1 ? 1 : n);
}

cudaError_t launch_amax_parts(const uint16_t* x, int64_t M, int64_t K, uint32_t* parts,
                              cudaStream_t stream, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(amax_parts_count(M, K)));
    cfg.blockDim = dim3(kAmaxThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, amax_parts_kernel, reinterpret_cast<const uint4*>(x),
                              M * K / 8, parts);
}

cudaError_t launch_quant(const uint16_t* x, const int8_t* q_in, int64_t M, int64_t K, int8_t* q,
                         float* s_x, float* r_x, int permuted, cudaStream_t stream, bool pdl,
                         void* zero, int64_t zero_bytes, int32_t* qsum,
                         const uint32_t* amax_parts, int n_parts, const uint16_t* tok_parts) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((M + kRowsPerCta - 1) / kRowsPerCta));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    // Few tokens may come with a large split-K area to clear: add CTAs so that no CTA clears
    // more than kZeroBytesPerCta (the clearing is a grid-stride loop; the added CTAs quantise
    // nothing).
    const int64_t zero_ctas = (zero_bytes + kZeroBytesPerCta - 1) / kZeroBytesPerCta;
    if (zero_ctas > int64_t(cfg.gridDim.x)) cfg.gridDim.x = static_cast<unsigned>(zero_ctas);
    if (q_in == nullptr && K > int64_t(32) * kRegPieces * 8 && K <= kLongMaxK) {
        const int64_t rows_ctas = (M + kLongRows - 1) / kLongRows;
        cfg.gridDim = dim3(static_cast<unsigned>(rows_ctas > zero_ctas ? rows_ctas : zero_ctas));
        cfg.blockDim = dim3(kLongThreads);
        return cudaLaunchKernelEx(&cfg, quant_long_rows_kernel, x, M, K, q, s_x, r_x, permuted,
                                  static_cast<uint4*>(zero), zero_bytes / 16, qsum, amax_parts,
                                  n_parts, tok_parts);
    }
    return cudaLaunchKernelEx(&cfg, quant_rows_kernel, x, q_in, M, K, q, s_x, r_x, permuted,
                              static_cast<uint4*>(zero), zero_bytes / 16, qsum, amax_parts,
                              n_parts, tok_parts);
}

}  // namespace bitnet
