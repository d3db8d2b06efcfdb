// Decode GEMV for M <= 8 tokens: y = dequant(q x t^T) with the activation quantiser fused
// in (page "BitNet-Triton", section "技术架构：融合内核的三重优化", items 1 and 3: the 2-bit
// weights are unpacked inside the kernel and x is quantised in the same launch; page
// "BitNet 1-bit LLM推理优化", section 4.2 "GPU加速：CUDA W2A8路径": packed decode to 8-bit
// and dp4a dot products).
//
// At M <= 8 the product is bound by reading the packed weights from HBM, so the kernel is
// laid out around that stream:
//  - one warp per weight row (two rows for short rows), each lane holding 16-byte packed
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
constexpr int kWarps = 8;
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
// CPL: 16-byte chunks per lane per row (K <= CPL * 32 * 64). RW: rows per warp.
template <int MT, int CPL, int RW>
__global__ void __launch_bounds__(kThreads) gemv_w2a8_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ uint4 s_q[];  // [MT][4][C] permuted q: word i of group 4c + j
    __shared__ uint32_t s_red[kWarps][MT];
    __shared__ int32_t s_sumq[MT];
    __shared__ float s_rx[MT];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int C = static_cast<int>(K >> 6);  // 16-byte chunks per packed row
    const int Mreal = p.M;

    // ---- 1. this warp's weight rows -> registers (no dependency on earlier grids)
    uint4 w[RW][CPL];
    int pj[RW];
    int64_t nrow[RW];
    bool rvalid[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int64_t gr = (int64_t(blockIdx.x) * kWarps + warp) * RW + r;
        rvalid[r] = gr < p.total_rows;
        int j = 0;
#pragma unroll
        for (int jj = 1; jj < kMaxProj; ++jj)
            if (jj < p.nproj && gr >= p.proj[jj].row_begin) j = jj;
        pj[r] = j;
        nrow[r] = gr - p.proj[j].row_begin;
        const uint8_t* rowp = p.proj[j].packed + nrow[r] * (K >> 2);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int chunk = lane + 32 * c;
            w[r][c] = (rvalid[r] && chunk < C) ? ldg_stream_v4(rowp + int64_t(chunk) * 16)
                                               : make_uint4(0u, 0u, 0u, 0u);
        }
    }

    pdl_trigger();
    pdl_wait();

    // ---- 2. quantise the tokens into shared memory
    const int64_t pieces = K >> 3;  // 8 values per piece
    if (threadIdx.x < MT) s_sumq[threadIdx.x] = 0;
    float s_tok[MT];
    if (p.q_in == nullptr) {
        uint32_t mx[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            mx[m] = 0;
            if (m < Mreal) {
                const uint4* xr = reinterpret_cast<const uint4*>(p.x + int64_t(m) * K);
                for (int64_t c = threadIdx.x; c < pieces; c += kThreads) {
                    const uint4 v = xr[c];
                    const uint32_t a = max(max(v.x & 0x7FFFu, v.x >> 16 & 0x7FFFu),
                                           max(v.y & 0x7FFFu, v.y >> 16 & 0x7FFFu));
                    const uint32_t b = max(max(v.z & 0x7FFFu, v.z >> 16 & 0x7FFFu),
                                           max(v.w & 0x7FFFu, v.w >> 16 & 0x7FFFu));
                    mx[m] = max(mx[m], max(a, b));
                }
            }
            mx[m] = __reduce_max_sync(0xFFFFFFFFu, mx[m]);
        }
        if (lane == 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m) s_red[warp][m] = mx[m];
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            uint32_t all = s_red[0][m];
#pragma unroll
            for (int ww = 1; ww < kWarps; ++ww) all = max(all, s_red[ww][m]);
            s_tok[m] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(all << 16), kEps));
        }
        if (threadIdx.x < MT) s_rx[threadIdx.x] = __frcp_rn(s_tok[threadIdx.x]);
    } else {
#pragma unroll
        for (int m = 0; m < MT; ++m) s_tok[m] = 0.0f;
    }
    __syncthreads();  // s_sumq zeroed before the atomics below

    uint8_t* sq_bytes = reinterpret_cast<uint8_t*>(s_q);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int qsum = 0;
        for (int64_t base = int64_t(warp) * 32; base < pieces; base += kThreads) {
            const int64_t c = base + lane;  // piece index; pieces is a multiple of 8
            const bool valid = c < pieces;
            uint2 nat = make_uint2(0u, 0u);
            if (valid && m < Mreal) {
                if (p.q_in == nullptr) {
                    const uint4 v = reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c];
                    const float s = s_tok[m];
                    nat.x = pack4(q8(bf16_lo(v.x), s), q8(bf16_hi(v.x), s), q8(bf16_lo(v.y), s),
                                  q8(bf16_hi(v.y), s));
                    nat.y = pack4(q8(bf16_lo(v.z), s), q8(bf16_hi(v.z), s), q8(bf16_lo(v.w), s),
                                  q8(bf16_hi(v.w), s));
                } else {
                    nat = reinterpret_cast<const uint2*>(p.q_in + int64_t(m) * K)[c];
                }
                qsum += bytesum(nat.x) + bytesum(nat.y);
            }
            const uint2 out = permute_group_half(nat, lane & 1);
            if (valid) {
                // group g = c / 2 lives in chunk g / 4, slot j = g % 4
                const int64_t g = c >> 1;
                const int64_t idx16 = (int64_t(m) * 4 + (g & 3)) * C + (g >> 2);
                *reinterpret_cast<uint2*>(sq_bytes + idx16 * 16 + (c & 1) * 8) = out;
            }
        }
        qsum = __reduce_add_sync(0xFFFFFFFFu, qsum);
        if (lane == 0 && qsum != 0) atomicAdd(&s_sumq[m], qsum);
    }
    __syncthreads();

    // ---- 3. dp4a over the register-resident chunks
    int32_t acc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;

#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int chunk = lane + 32 * c;
        if (chunk < C) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 qv = s_q[(m * 4 + j) * C + chunk];
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const uint32_t word = j == 0 ? w[r][c].x : j == 1 ? w[r][c].y
                                            : j == 2 ? w[r][c].z : w[r][c].w;
                        int a = acc[r][m];
                        a = __dp4a(int(word & 0x03030303u), int(qv.x), a);
                        a = __dp4a(int((word >> 2) & 0x03030303u), int(qv.y), a);
                        a = __dp4a(int((word >> 4) & 0x03030303u), int(qv.z), a);
                        a = __dp4a(int((word >> 6) & 0x03030303u), int(qv.w), a);
                        acc[r][m] = a;
                    }
                }
            }
        }
    }

    // ---- 4. reduce across the warp and write
#pragma unroll
    for (int r = 0; r < RW; ++r) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int32_t total = __reduce_add_sync(0xFFFFFFFFu, acc[r][m]);
            if (lane == r * MT + m && rvalid[r] && m < Mreal) {
                const GemvProj& pr = p.proj[pj[r]];
                const int32_t v = total - s_sumq[m];
                const int64_t o = int64_t(m) * pr.N + nrow[r];
                if (p.out_kind == 2) {
                    reinterpret_cast<int32_t*>(pr.y)[o] = v;
                } else {
                    const float sw = pr.per_row ? pr.s_w[nrow[r]] : pr.s_w[0];
                    const float yv = __fmul_rn(__int2float_rn(v), __fmul_rn(sw, s_rx[m]));
                    if (p.out_kind == 0)
                        reinterpret_cast<__nv_bfloat16*>(pr.y)[o] = __float2bfloat16_rn(yv);
                    else
                        reinterpret_cast<float*>(pr.y)[o] = yv;
                }
            }
        }
    }
}

template <int MT, int CPL, int RW>
cudaError_t launch_one(const GemvParams& p, cudaStream_t stream, bool pdl) {
    const size_t smem = size_t(MT) * size_t(p.K);
    auto kern = gemv_w2a8_kernel<MT, CPL, RW>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t rows_per_cta = int64_t(kWarps) * RW;
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
    if (cpl <= 1) return launch_one<MT, 1, (MT <= 2 ? 2 : 1)>(p, stream, pdl);
    if (cpl <= 2) return launch_one<MT, 2, (MT <= 2 ? 2 : 1)>(p, stream, pdl);
    if (cpl <= 4) return launch_one<MT, 4, 1>(p, stream, pdl);
    if (cpl <= 8) return launch_one<MT, 8, 1>(p, stream, pdl);
    return launch_one<MT, 16, 1>(p, stream, pdl);
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
