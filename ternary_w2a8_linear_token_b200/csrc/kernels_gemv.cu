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

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"
#include "swiglu_device.cuh"

namespace bitnet {
namespace {

constexpr float kEps = kActEps;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;

// MT: token capacity (compile time); p.M <= MT tokens are real, the rest are zero.
// CPL: 16-byte chunks per lane (K <= CPL * 32 * 64). RW: weight rows per warp.
// SW: SwiGLU of an interleaved gate/up matrix; each warp takes RW / 2 output pairs, the gate
// row and the up row of each output j (rows 2p and 2p + 1 of the warp), and writes
// h = SwiGLU(g, u).
template <int MT, int CPL, int RW, bool SW>
__global__ void __launch_bounds__(kThreads, MT <= 2 ? 2 : 1) gemv_w2a8_kernel(const __grid_constant__ GemvParams p) {
    static_assert(!SW || RW == 2 || RW == 4, "a SwiGLU warp holds one or two gate/up pairs");
    extern __shared__ uint4 s_q[];  // [MT][4][C] permuted q: word i of group 4c + j
    __shared__ uint32_t s_red[kWarps][MT];  // per-warp amax bits
    __shared__ int32_t s_qsum[kWarps][MT];  // per-warp partial sums of q

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int C = static_cast<int>(K >> 6);  // 16-byte chunks per packed row
    const int Mreal = p.M;

    // ---- 1. this warp's weight rows -> registers (no dependency on earlier grids)
    int64_t gr[RW];
    bool rvalid[RW];
    int pj[RW];
    int64_t nrow[RW];
    uint4 w[RW][CPL];
    float sw[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        pj[r] = 0;
        if constexpr (SW) {
            // output pair j: gate row 32 (j / 16) + j % 16, up row 16 further
            const int64_t j = (int64_t(blockIdx.x) * kWarps + warp) * (RW / 2) + r / 2;
            gr[r] = (j / kSwigluBlock) * (2 * kSwigluBlock) + j % kSwigluBlock +
                    (r & 1) * kSwigluBlock;
            rvalid[r] = j < p.total_rows;
        } else {
            gr[r] = (int64_t(blockIdx.x) * kWarps + warp) * RW + r;
            rvalid[r] = gr[r] < p.total_rows;
#pragma unroll
            for (int jj = 1; jj < kMaxProj; ++jj)
                if (jj < p.nproj && gr[r] >= p.proj[jj].row_begin) pj[r] = jj;
        }
        nrow[r] = gr[r] - p.proj[pj[r]].row_begin;
        const uint8_t* rowp = p.proj[pj[r]].packed + nrow[r] * (K >> 2);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int chunk = lane + 32 * c;
            w[r][c] = (rvalid[r] && chunk < C) ? ldg_stream_v4(rowp + int64_t(chunk) * 16)
                                               : make_uint4(0u, 0u, 0u, 0u);
        }
        sw[r] = 0.0f;
        if (rvalid[r] && p.out_kind != 2)  // per-tensor SwiGLU scales are {s_gate, s_up}
            sw[r] = p.proj[pj[r]].per_row ? p.proj[pj[r]].s_w[nrow[r]]
                                          : p.proj[pj[r]].s_w[SW ? (r & 1) : 0];
    }

    pdl_trigger();
    pdl_wait();

    // ---- 2. quantise the tokens into shared memory (pieces of 8 values; pieces % 8 == 0)
    const int64_t pieces = K >> 3;
    float s_tok[MT];
    // x is staged in shared memory (after q) during the amax pass when it fits, so the
    // quantising pass never goes back to global memory.
    uint4* s_x = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(s_q) + int64_t(MT) * K);
    const bool stage_x = p.stage_x != 0;
    if (p.q_in == nullptr) {
        uint32_t mx[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) mx[m] = 0;
#pragma unroll 2
        for (int64_t c = threadIdx.x; c < pieces; c += kThreads) {
            uint4 v[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m)  // all tokens' loads in flight together
                v[m] = m < Mreal ? reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c]
                                 : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (stage_x) s_x[int64_t(m) * pieces + c] = v[m];
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
        uint32_t all[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            all[m] = s_red[0][m];
#pragma unroll
            for (int ww = 1; ww < kWarps; ++ww) all[m] = max(all[m], s_red[ww][m]);
        }
        if (p.act_per_tensor) {  // one scale for all real tokens ("推理优化" §2.2, I2_S)
            uint32_t t = 0;
#pragma unroll
            for (int m = 0; m < MT; ++m) t = m < Mreal ? max(t, all[m]) : t;
#pragma unroll
            for (int m = 0; m < MT; ++m) all[m] = t;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m)
            s_tok[m] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(all[m] << 16), kEps));
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
                v[m] = (valid && m < Mreal)
                           ? (stage_x ? s_x[int64_t(m) * pieces + c]
                                      : reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c])
                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float s = s_tok[m];
                nat[m].x = pack4(qbits(bf16_lo(v[m].x), s), qbits(bf16_hi(v[m].x), s),
                                 qbits(bf16_lo(v[m].y), s), qbits(bf16_hi(v[m].y), s));
                nat[m].y = pack4(qbits(bf16_lo(v[m].z), s), qbits(bf16_hi(v[m].z), s),
                                 qbits(bf16_lo(v[m].w), s), qbits(bf16_hi(v[m].w), s));
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

    // ---- 3. dp4a over the register-resident chunks: sum_k q * code, independent
    //         accumulator chains per output (four at one token, two otherwise)
    // One token: the codes are masked in place (code_dot_acc, one AND per four weights and
    // four accumulators); more tokens share one shifted unpack of each word instead (and
    // would need more registers for the accumulators than two CTAs per SM leave).
    constexpr bool kMasked = MT == 1;
    int4 acc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = make_int4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int chunk = lane + 32 * c;
        if (chunk < C) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t word[RW];
                int e[RW][4];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    word[r] = j == 0 ? w[r][c].x : j == 1 ? w[r][c].y
                            : j == 2 ? w[r][c].z : w[r][c].w;
                    if constexpr (!kMasked) {
                        e[r][0] = int(word[r] & 0x03030303u);
                        e[r][1] = int((word[r] >> 2) & 0x03030303u);
                        e[r][2] = int((word[r] >> 4) & 0x03030303u);
                        e[r][3] = int((word[r] >> 6) & 0x03030303u);
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 qv = s_q[(m * 4 + j) * C + chunk];
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        if constexpr (kMasked) {
                            code_dot_acc(word[r], qv, acc[r][m]);
                        } else {
                            acc[r][m].x = __dp4a(e[r][0], int(qv.x), acc[r][m].x);
                            acc[r][m].y = __dp4a(e[r][1], int(qv.y), acc[r][m].y);
                            acc[r][m].x = __dp4a(e[r][2], int(qv.z), acc[r][m].x);
                            acc[r][m].y = __dp4a(e[r][3], int(qv.w), acc[r][m].y);
                        }
                    }
                }
            }
        }
    }
    auto dot_total = [](const int4 a) { return kMasked ? code_dot_total(a) : a.x + a.y; };

    // ---- 4. reduce across the warp, remove the code offset (sum q), dequantise, write
    int32_t qs_tot[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int32_t t = 0;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) t += s_qsum[ww][m];
        qs_tot[m] = t;
    }
    if constexpr (SW) {
        // g and u of this warp's output pairs for every token; lane pp * MT + m writes
        // token m's h of pair pp.
#pragma unroll
        for (int pp = 0; pp < RW / 2; ++pp) {
            const int64_t j = (int64_t(blockIdx.x) * kWarps + warp) * (RW / 2) + pp;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int32_t tg =
                    __reduce_add_sync(0xFFFFFFFFu, dot_total(acc[2 * pp][m]));
                const int32_t tu =
                    __reduce_add_sync(0xFFFFFFFFu, dot_total(acc[2 * pp + 1][m]));
                if (lane == pp * MT + m && rvalid[2 * pp] && m < Mreal) {
                    const float rx = __frcp_rn(s_tok[m]);
                    const float g =
                        __fmul_rn(__int2float_rn(tg - qs_tot[m]), __fmul_rn(sw[2 * pp], rx));
                    const float u =
                        __fmul_rn(__int2float_rn(tu - qs_tot[m]), __fmul_rn(sw[2 * pp + 1], rx));
                    static_cast<uint16_t*>(p.proj[0].y)[int64_t(m) * p.proj[0].N + j] =
                        swiglu_bf16_bits(g, u);
                }
            }
        }
    } else {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int32_t total = __reduce_add_sync(0xFFFFFFFFu, dot_total(acc[r][m]));
                if (lane == r * MT + m && rvalid[r] && m < Mreal) {
                    const GemvProj& pr = p.proj[pj[r]];
                    const int32_t v = total - qs_tot[m];
                    const int64_t o = int64_t(m) * pr.N + nrow[r];
                    if (p.out_kind == 2) {
                        reinterpret_cast<int32_t*>(pr.y)[o] = v;
                    } else {
                        const float rx = __frcp_rn(s_tok[m]);
                        const float yv = __fmul_rn(__int2float_rn(v), __fmul_rn(sw[r], rx));
                        if (p.out_kind == 0)
                            reinterpret_cast<__nv_bfloat16*>(pr.y)[o] = __float2bfloat16_rn(yv);
                        else
                            reinterpret_cast<float*>(pr.y)[o] = yv;
                    }
                }
            }
        }
    }
}

int num_sms() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

template <int MT, int CPL, int RW, bool SW = false>
cudaError_t launch_one(const GemvParams& p, cudaStream_t stream, bool pdl) {
    // q (MT*K bytes) plus, when it fits, the staged bf16 activations (2*MT*K bytes)
    GemvParams q = p;
    q.stage_x = (p.q_in == nullptr && 3 * int64_t(MT) * p.K <= 96 * 1024) ? 1 : 0;
    const size_t smem = size_t(MT) * size_t(p.K) * (q.stage_x ? 3 : 1);
    auto kern = gemv_w2a8_kernel<MT, CPL, RW, SW>;
    // Above 48 KB in total (dynamic plus the kernel's static reduction arrays) a launch needs
    // the opt-in attribute.
    const size_t static_smem = sizeof(uint32_t) * kWarps * MT + sizeof(int32_t) * kWarps * MT;
    if (smem + static_smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    // rows of the grid per CTA (SwiGLU: output pairs)
    const int64_t rows_per_cta = SW ? int64_t(kWarps) * (RW / 2) : int64_t(kWarps) * RW;
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
    return cudaLaunchKernelEx(&cfg, kern, q);
}

template <int MT, int CPL>
cudaError_t launch_cpl(const GemvParams& p, cudaStream_t stream, bool pdl) {
    const int rw = gemv_rows_per_warp(p, num_sms());
    if (p.swiglu) {
        if constexpr (MT <= 2 && CPL <= 2) {
            if (rw == 4) return launch_one<MT, CPL, 4, true>(p, stream, pdl);
        }
        return launch_one<MT, CPL, 2, true>(p, stream, pdl);
    }
    if constexpr (MT <= 2) {
        if constexpr (CPL <= 2) {
            if (rw == 4) return launch_one<MT, CPL, 4>(p, stream, pdl);
            if (rw == 2) return launch_one<MT, CPL, 2>(p, stream, pdl);
        }
    } else {
        if constexpr (CPL <= 2 && MT <= 4) {
            if (rw == 3) return launch_one<MT, CPL, 3>(p, stream, pdl);
        }
        if constexpr (CPL <= 2 || (MT <= 4 && CPL <= 4)) {
            if (rw == 2) return launch_one<MT, CPL, 2>(p, stream, pdl);
        }
    }
    return launch_one<MT, CPL, 1>(p, stream, pdl);
}

template <int MT>
cudaError_t launch_mt(const GemvParams& p, cudaStream_t stream, bool pdl) {
    const int64_t C = p.K >> 6;
    const int cpl = static_cast<int>((C + 31) / 32);
    if (cpl <= 1) return launch_cpl<MT, 1>(p, stream, pdl);
    if (cpl <= 2) return launch_cpl<MT, 2>(p, stream, pdl);
    if (cpl <= 4) return launch_cpl<MT, 4>(p, stream, pdl);
    if (cpl <= 8) return launch_cpl<MT, 8>(p, stream, pdl);
    return launch_cpl<MT, 16>(p, stream, pdl);
}

}  // namespace

// Rows per warp of the dp4a GEMV (SwiGLU: 2 per gate/up pair). One or two tokens run two CTAs
// per SM (so the next grid, started early by programmatic dependent launch, loads its weights
// while this one finishes) and take two rows per warp once the grid would exceed two CTAs per
// SM, or one CTA per SM for rows of at least 1 KB (measured on B200 at one token: 2560 x 2560
// runs faster with one row per warp on 160 CTAs, 3.08 -> 3.02 µs per call and the decode sweep
// 3.36 -> 3.22; 4096 x 4096 slower, 3.38 -> 3.58). More rows per warp lengthen the work left
// after the wait for the previous grid, which costs more than it saves (measured on B200),
// except where two rows per warp would need more than two CTAs per SM: four rows keep such a
// matrix in one wave (the 2B-4T layer's batched q/k/v/gate/up, 17664 x 2560 at one token:
// 8.2 -> 6.7 µs per call; 6912 x 2560, which two rows per warp already fit in one wave,
// 4.1 -> 4.8 µs with four); the SwiGLU variant likewise takes two pairs per warp once one pair
// would need more than two CTAs per SM. Four or eight tokens run one CTA per SM and take as
// many rows per warp (up to 3) as let one wave cover every row: a second wave would repeat
// each CTA's quantisation of the tokens and its whole dependent chain. Register-resident
// weights cap the rows per warp (the chunk counts below).
int gemv_rows_per_warp(const GemvParams& p, int sms) {
    const int64_t C = p.K >> 6;
    const int64_t c32 = (C + 31) / 32;  // chunks per lane, rounded up as the kernels are
    const int cpl = c32 <= 1 ? 1 : c32 <= 2 ? 2 : c32 <= 4 ? 4 : c32 <= 8 ? 8 : 16;
    const int mt = p.M <= 1 ? 1 : p.M <= 2 ? 2 : p.M <= 4 ? 4 : 8;
    const int64_t slots = int64_t(sms) * kWarps;  // warps of one CTA per SM
    if (p.swiglu) return (mt <= 2 && cpl <= 2 && p.total_rows > 2 * slots) ? 4 : 2;
    if (mt <= 2) {
        if (cpl <= 2) {
            if (p.total_rows > 4 * slots) return 4;
            if (p.total_rows > 2 * slots || (p.total_rows > slots && p.K >= 4096)) return 2;
        }
        return 1;
    }
    const int64_t need = (p.total_rows + slots - 1) / slots;
    if (cpl <= 2 && mt <= 4 && need >= 3) return 3;
    if ((cpl <= 2 || (mt <= 4 && cpl <= 4)) && need >= 2) return 2;
    return 1;
}

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
