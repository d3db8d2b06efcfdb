// Decode GEMV for M <= 8 tokens: y = dequant(q x t^T) with the activation quantiser fused
// in (page "BitNet-Triton", section "技术架构：融合内核的三重优化", items 1 and 3: the 2-bit
// weights are unpacked inside the kernel and x is quantised in the same launch; page
// "BitNet 1-bit LLM推理优化", section 4.2 "GPU加速：CUDA W2A8路径": packed decode to 8-bit
// and dp4a dot products).
//
// At M <= 8 the product is bound by reading the packed weights from HBM, so the kernel is
// laid out around that stream:
//  - one warp per weight row, each lane holding 16-byte packed
//    chunks in registers; every chunk load is issued before the kernel waits on the
//    previous grid (programmatic dependent launch), since weights never depend on it;
//  - each CTA quantises the M tokens into shared memory in the permuted in-group order
//    (see kernels_quant.cu), so a packed word unpacks with one shift and one mask per
//    four weights: codes c = t + 1 in {0, 1, 2} feed dp4a directly and the
//    code offset is removed once per token: sum q t = sum q c - sum q;
//  - a warp-wide integer reduction and one fp32 epilogue per output.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr float kEps = 1e-5f;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ int q8(float xv, float s) {
    return min(max(__float2int_rn(__fmul_rn(xv, s)), -128), 127);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8) | ((uint32_t(c) & 0xFFu) << 16) |
           (uint32_t(d) << 24);
}

__device__ __forceinline__ int bytesum(uint32_t w) {
    return int(int8_t(w & 0xFF)) + int(int8_t((w >> 8) & 0xFF)) + int(int8_t((w >> 16) & 0xFF)) +
           int(int8_t(w >> 24));
}

// See kernels_quant.cu: lane pair (h = 0, 1) of one 16-group -> this lane's 8 permuted bytes.
__device__ __forceinline__ uint2 permute_group_half(uint2 nat, int h) {
    const uint32_t p01 = __byte_perm(nat.x, nat.y, 0x5140);
    const uint32_t p23 = __byte_perm(nat.x, nat.y, 0x7362);
    const uint32_t own = h ? p23 : p01;
    const uint32_t send = h ? p01 : p23;
    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
    const uint32_t lo = h ? recv : own;
    const uint32_t hi = h ? own : recv;
    return make_uint2(__byte_perm(lo, hi, 0x5410), __byte_perm(lo, hi, 0x7632));
}

// MT: token capacity (compile time); p.M <= MT tokens are real, the rest are zero.
// CPL: 16-byte chunks per lane (K <= CPL * 32 * 64). One weight row per warp.
template <int MT, int CPL>
__global__ void __launch_bounds__(kThreads) gemv_w2a8_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ uint4 s_q[];  // [MT][4][C] permuted q: word i of group 4c + j
    __shared__ uint32_t s_red[kWarps][MT];  // per-warp amax bits
    __shared__ int32_t s_qsum[kWarps][MT];  // per-warp partial sums of q

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int C = static_cast<int>(K >> 6);  // 16-byte chunks per packed row
    const int Mreal = p.M;

    // ---- 1. this warp's weight row -> registers (no dependency on earlier grids)
    const int64_t gr = int64_t(blockIdx.x) * kWarps + warp;
    const bool rvalid = gr < p.total_rows;
    int pj = 0;
#pragma unroll
    for (int jj = 1; jj < kMaxProj; ++jj)
        if (jj < p.nproj && gr >= p.proj[jj].row_begin) pj = jj;
    const int64_t nrow = gr - p.proj[pj].row_begin;
    uint4 w[CPL];
    {
        const uint8_t* rowp = p.proj[pj].packed + nrow * (K >> 2);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int chunk = lane + 32 * c;
            w[c] = (rvalid && chunk < C) ? ldg_stream_v4(rowp + int64_t(chunk) * 16)
                                         : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    float sw = 0.0f;
    if (rvalid && p.out_kind != 2) sw = p.proj[pj].per_row ? p.proj[pj].s_w[nrow] : p.proj[pj].s_w[0];

    pdl_trigger();
    pdl_wait();

    // ---- 2. quantise the tokens into shared memory (pieces of 8 values; pieces % 8 == 0)
    const int64_t pieces = K >> 3;
    float s_tok[MT];
    if (p.q_in == nullptr) {
        uint32_t mx[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) mx[m] = 0;
        for (int64_t c = threadIdx.x; c < pieces; c += kThreads) {
            uint4 v[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m)  // all tokens' loads in flight together
                v[m] = m < Mreal ? reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c]
                                 : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint32_t a = max(max(v[m].x & 0x7FFFu, v[m].x >> 16 & 0x7FFFu),
                                       max(v[m].y & 0x7FFFu, v[m].y >> 16 & 0x7FFFu));
                const uint32_t b = max(max(v[m].z & 0x7FFFu, v[m].z >> 16 & 0x7FFFu),
                                       max(v[m].w & 0x7FFFu, v[m].w >> 16 & 0x7FFFu));
                mx[m] = max(mx[m], max(a, b));
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint32_t r = __reduce_max_sync(0xFFFFFFFFu, mx[m]);
            if (lane == 0) s_red[warp][m] = r;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            uint32_t all = s_red[0][m];
#pragma unroll
            for (int ww = 1; ww < kWarps; ++ww) all = max(all, s_red[ww][m]);
            s_tok[m] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(all << 16), kEps));
        }
    } else {
#pragma unroll
        for (int m = 0; m < MT; ++m) s_tok[m] = 0.0f;
    }

    uint8_t* sq_bytes = reinterpret_cast<uint8_t*>(s_q);
    int qsum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) qsum[m] = 0;
    // warp-uniform trip count: the pair shuffle needs both lanes of a group present
    for (int64_t base = int64_t(warp) * 32; base < pieces; base += kThreads) {
        const int64_t c = base + lane;
        const bool valid = c < pieces;
        uint2 nat[MT];
        if (p.q_in == nullptr) {
            uint4 v[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m)
                v[m] = (valid && m < Mreal) ? reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c]
                                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float s = s_tok[m];
                nat[m].x = pack4(q8(bf16_lo(v[m].x), s), q8(bf16_hi(v[m].x), s),
                                 q8(bf16_lo(v[m].y), s), q8(bf16_hi(v[m].y), s));
                nat[m].y = pack4(q8(bf16_lo(v[m].z), s), q8(bf16_hi(v[m].z), s),
                                 q8(bf16_lo(v[m].w), s), q8(bf16_hi(v[m].w), s));
            }
        } else {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                nat[m] = (valid && m < Mreal)
                             ? reinterpret_cast<const uint2*>(p.q_in + int64_t(m) * K)[c]
                             : make_uint2(0u, 0u);
        }
        const int64_t g = c >> 1;  // group g = c / 2 lives in chunk g / 4, slot j = g % 4
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            qsum[m] += bytesum(nat[m].x) + bytesum(nat[m].y);
            const uint2 out = permute_group_half(nat[m], lane & 1);
            if (valid) {
                const int64_t idx16 = (int64_t(m) * 4 + (g & 3)) * C + (g >> 2);
                *reinterpret_cast<uint2*>(sq_bytes + idx16 * 16 + (c & 1) * 8) = out;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const int r = __reduce_add_sync(0xFFFFFFFFu, qsum[m]);
        if (lane == 0) s_qsum[warp][m] = r;
    }
    __syncthreads();

    // ---- 3. dp4a over the register-resident chunks: sum_k q * code
    int32_t acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int chunk = lane + 32 * c;
        if (chunk < C) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t word = j == 0 ? w[c].x : j == 1 ? w[c].y : j == 2 ? w[c].z : w[c].w;
                const int e0 = int(word & 0x03030303u);
                const int e1 = int((word >> 2) & 0x03030303u);
                const int e2 = int((word >> 4) & 0x03030303u);
                const int e3 = int((word >> 6) & 0x03030303u);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 qv = s_q[(m * 4 + j) * C + chunk];
                    int a = acc[m];
                    a = __dp4a(e0, int(qv.x), a);
                    a = __dp4a(e1, int(qv.y), a);
                    a = __dp4a(e2, int(qv.z), a);
                    a = __dp4a(e3, int(qv.w), a);
                    acc[m] = a;
                }
            }
        }
    }

    // ---- 4. reduce across the warp, remove the code offset (sum q), dequantise, write
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const int32_t total = __reduce_add_sync(0xFFFFFFFFu, acc[m]);
        if (lane == m && rvalid && m < Mreal) {
            int32_t qs = 0;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) qs += s_qsum[ww][m];
            const GemvProj& pr = p.proj[pj];
            const int32_t v = total - qs;
            const int64_t o = int64_t(m) * pr.N + nrow;
            if (p.out_kind == 2) {
                reinterpret_cast<int32_t*>(pr.y)[o] = v;
            } else {
                const float rx = __frcp_rn(s_tok[m]);
                const float yv = __fmul_rn(__int2float_rn(v), __fmul_rn(sw, rx));
                if (p.out_kind == 0)
                    reinterpret_cast<__nv_bfloat16*>(pr.y)[o] = __float2bfloat16_rn(yv);
                else
                    reinterpret_cast<float*>(pr.y)[o] = yv;
            }
        }
    }
}

template <int MT, int CPL>
cudaError_t launch_one(const GemvParams& p, cudaStream_t stream, bool pdl) {
    const size_t smem = size_t(MT) * size_t(p.K);
    auto kern = gemv_w2a8_kernel<MT, CPL>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t rows_per_cta = kWarps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((p.total_rows + rows_per_cta - 1) / rows_per_cta));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int MT>
cudaError_t launch_mt(const GemvParams& p, cudaStream_t stream, bool pdl) {
    const int64_t C = p.K >> 6;
    const int cpl = static_cast<int>((C + 31) / 32);
    if (cpl <= 1) return launch_one<MT, 1>(p, stream, pdl);
    if (cpl <= 2) return launch_one<MT, 2>(p, stream, pdl);
    if (cpl <= 4) return launch_one<MT, 4>(p, stream, pdl);
    if (cpl <= 8) return launch_one<MT, 8>(p, stream, pdl);
    return launch_one<MT, 16>(p, stream, pdl);
}

}  // namespace

bool gemv_supported(int64_t M, int64_t K) {
    const int64_t mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    return M >= 1 && M <= 8 && (K >> 6) <= 16 * 32 && mt * K <= 200 * 1024;
}

cudaError_t launch_gemv(const GemvParams& p, cudaStream_t stream, bool pdl) {
    if (p.M <= 1) return launch_mt<1>(p, stream, pdl);
    if (p.M <= 2) return launch_mt<2>(p, stream, pdl);
    if (p.M <= 4) return launch_mt<4>(p, stream, pdl);
    return launch_mt<8>(p, stream, pdl);
}

}  // namespace bitnet
