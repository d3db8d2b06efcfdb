// Decode GEMV for M <= 8 tokens on warp-level int8 tensor-core MMA, with the activation
// quantiser fused in (page "BitNet-Triton", section "技术架构：融合内核的三重优化", items 1-3:
// 2-bit weights unpacked inside the kernel, int8 tensor-core arithmetic, x quantised in the same
// launch; page "BitNet 1-bit LLM推理优化", section 4.2: packed decode to 8-bit in the kernel).
//
// At decode sizes a layer is a chain of small dependent products, so a call costs the latency
// of the work left after the kernel may read its input, plus the hand-off between grids. The
// kernel is built around that:
//  - the next calls of a chain are launched early (programmatic dependent launch) and sit
//    resident beside the running one until they may read their input. While they wait they
//    must cost the running call nothing: one warp of each waiting CTA issues bulk async copies
//    (no multicast) of the CTA's weight rows into shared memory and prefetches x into L2 (L2 is
//    coherent with the previous grid's writes; nothing of x enters L1 before the wait), and
//    every other thread goes straight to the wait. (Waiting CTAs that loaded their weights
//    into registers with per-thread loads slowed the running call measurably on B200.)
//  - the contraction is mma.sync.m16n8k32 with the weight rows as the MMA's 16 rows and the
//    tokens as its 8 columns: one warp-wide instruction multiplies 16 rows x 32 K values
//    against every token, the K sum across the warp's lanes happens inside the MMA, and the
//    token operand is read from shared memory once per 16 rows (a dot product per lane would
//    read it once per row);
//  - a CTA owns `rt` tiles of 16 weight rows; its 8 warps split them into rt x (8 / rt)
//    (row tile, K slice) pairs, and one shared-memory reduction joins the K slices.
//
// Operand layout. The activations are quantised into shared memory in the permuted in-group
// order: inside each group of 16 values along K, byte 4i + b holds k = 4b + i, so permuted
// word i of group u holds k = 16u + i, 16u + 4 + i, 16u + 8 + i, 16u + 12 + i. Packed weight
// word u of a row holds the codes of group u, code of k = 16u + 4b + i in bits 2i .. 2i + 1 of
// byte b, so (word >> 2i) & 0x03030303 lines up byte for byte with permuted word i. In the MMA,
// lane (g, t) (g = lane / 4, t = lane % 4) supplies A rows g and g + 8 for K slots 4t .. 4t + 3
// and 16 + 4t .. 16 + 4t + 3, and B column g (token g) for the same K slots: every lane of
// quad position t takes the same packed chunk index, so one K slot means one k for all rows
// and tokens. One packed word pair (rows g, g + 8) feeds two MMAs: shifts 0 and 2 against
// permuted words 0 and 1, shifts 4 and 6 against words 2 and 3. The A operand is the unsigned
// code c = t + 1 in {0, 1, 2}; sum q t = sum q c - sum q, with sum q per token from the
// quantiser.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"
#include "swiglu_device.cuh"

namespace bitnet {
namespace {

constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMaxPieceIters = 8;  // 8-value pieces per thread and token: K <= 8 * 256 * 8

// D (16 x 8, s32) += A (16 x 32, u8, row-major) . B (32 x 8, s8, column-major).
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                                uint32_t a2, uint32_t a3, uint32_t b0,
                                                uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bytes of one token's permuted q in shared memory: 4 groups x C chunks x 16 bytes, plus 16 so
// that the 8 tokens' 16-byte pieces of one chunk fall in different bank groups.
__host__ __device__ inline int64_t mma_tok_stride(int64_t C) { return 64 * C + 16; }

// Bytes of one weight row in shared memory: the packed row plus 16 when that makes the row
// stride an odd multiple of 16 modulo 128, so the 8 rows an MMA's lanes read at one chunk
// offset fall in different 16-byte bank groups (row bytes = K / 4 are a multiple of 16).
__host__ __device__ inline int64_t mma_row_stride(int64_t row_bytes) {
    return (row_bytes / 16) % 2 == 1 ? row_bytes : row_bytes + 16;
}

__host__ inline size_t mma_smem_bytes(int mt, int rt, int64_t K) {
    return size_t(16 * rt) * size_t(mma_row_stride(K >> 2)) + size_t(mt) * size_t(mma_tok_stride(K >> 6)) +
           kMmaWarps * 128 * 4 + 16;
}

// MT: token capacity (p.M <= MT real tokens). CPT: packed chunks per lane and row (a warp's K
// slice spans up to 4 * CPT chunks). SW: SwiGLU of an interleaved gate/up matrix (rt even, so a
// CTA holds both 16-row blocks of every output it writes). rt: 16-row tiles per CTA (1, 2, 4, 8).
template <int MT, int CPT, bool SW>
__global__ void __launch_bounds__(kMmaThreads) gemv_mma_kernel(const __grid_constant__ GemvParams p,
                                                                int rt, int32_t* err) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint32_t s_amax[kMmaWarps][MT];
    __shared__ int32_t s_qs[kMmaWarps][MT];

    pdl_trigger();  // the next call of a chain may start loading its weights at once

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t K = p.K;
    const int C = static_cast<int>(K >> 6);  // 16-byte packed chunks per row
    const int64_t row_bytes = K >> 2;
    const int64_t tok_stride = mma_tok_stride(C);
    const int64_t wstride = mma_row_stride(row_bytes);
    uint8_t* s_w = smem;                                  // [16 rt rows][wstride]
    uint8_t* s_q = smem + 16 * rt * wstride;              // [MT][tok_stride]
    int32_t* s_red = reinterpret_cast<int32_t*>(s_q + MT * tok_stride);  // [8][16][8]
    uint64_t* wbar = reinterpret_cast<uint64_t*>(s_red + kMmaWarps * 128);
    const int ks = kMmaWarps / rt;         // K slices per row tile
    const int wrt = warp / ks;             // this warp's row tile within the CTA
    const int wks = warp - wrt * ks;       // and its K slice
    const int c0 = (wks * C) / ks, c1 = ((wks + 1) * C) / ks;
    const int64_t rows = SW ? 2 * p.total_rows : p.total_rows;  // packed rows in all

    // Base address of packed row r (null past the end); the batch's projections are laid
    // end to end (an interleaved SwiGLU matrix is one projection).
    auto row_base = [&](int64_t r) -> const uint8_t* {
        if (r >= rows) return nullptr;
        int pj = 0;
        if constexpr (!SW) {
#pragma unroll
            for (int j = 1; j < kMaxProj; ++j)
                if (j < p.nproj && r >= p.proj[j].row_begin) pj = j;
        }
        return p.proj[pj].packed + (r - p.proj[pj].row_begin) * row_bytes;
    };

    // ---- 1. before the wait: warp 0 copies the CTA's weight rows into shared memory (one
    //         bulk copy per row, rows padded to wstride so that the 8 rows an MMA reads sit in
    //         different banks), completing on wbar.
    const int64_t row0 = 16 * int64_t(blockIdx.x) * rt;
    if (warp == 0) {
        if (lane == 0) {
            mbar_init(wbar, 1);
            fence_mbar_init();
            const int64_t valid = rows - row0 < 16 * rt ? rows - row0 : 16 * rt;
            mbar_arrive_expect_tx(wbar, uint32_t(valid * row_bytes));
        }
        __syncwarp();
        for (int r = lane; r < 16 * rt; r += 32) {
            const uint8_t* src = row_base(row0 + r);
            if (src) bulk_load_1d(s_w + r * wstride, src, uint32_t(row_bytes), wbar);
        }
    }
    // The input into L2 (it may be cold there; a write by the previous grid lands in L2 too).
    {
        const uint8_t* src = p.q_in ? reinterpret_cast<const uint8_t*>(p.q_in)
                                    : reinterpret_cast<const uint8_t*>(p.x);
        const int64_t bytes = int64_t(p.M) * K * (p.q_in ? 1 : 2);
        for (int64_t off = int64_t(threadIdx.x) * 128; off < bytes; off += kMmaThreads * 128)
            prefetch_l2(src + off);
    }
    // Thread o < outs writes output o (a weight row, or a SwiGLU pair) of the CTA for every
    // token: its destination and scale(s) are fetched here, off the path after the wait.
    const int outs = SW ? 8 * rt : 16 * rt;
    const int o = threadIdx.x;
    const int o_lt = SW ? 2 * (o >> 4) : (o >> 4);  // local row tile (SwiGLU: the gate tile)
    const int o_r16 = o & 15;
    bool o_valid = false;
    void* o_y = nullptr;   // output element of token 0
    int64_t o_ld = 0;      // elements between tokens
    float o_sa = 0.0f, o_sb = 0.0f;
    if (o < outs) {
        if constexpr (SW) {
            const int64_t pair = int64_t(blockIdx.x) * (8 * rt) + o;
            const int64_t gate_row = 16 * (int64_t(blockIdx.x) * rt + o_lt) + o_r16;
            const GemvProj& pr = p.proj[0];
            o_valid = pair < p.total_rows;
            if (o_valid) {
                o_sa = pr.per_row ? pr.s_w[gate_row] : pr.s_w[0];
                o_sb = pr.per_row ? pr.s_w[gate_row + kSwigluBlock] : pr.s_w[1];
                o_y = static_cast<uint16_t*>(pr.y) + pair;
                o_ld = pr.N;
            }
        } else {
            const int64_t r = 16 * (int64_t(blockIdx.x) * rt + o_lt) + o_r16;
            o_valid = r < rows;
            if (o_valid) {
                int pj = 0;
#pragma unroll
                for (int j = 1; j < kMaxProj; ++j)
                    if (j < p.nproj && r >= p.proj[j].row_begin) pj = j;
                const GemvProj& pr = p.proj[pj];
                const int64_t n = r - pr.row_begin;
                const int esz = p.out_kind == 0 ? 2 : 4;
                o_y = static_cast<uint8_t*>(pr.y) + n * esz;
                o_ld = pr.N;
                if (p.out_kind != 2) o_sa = pr.per_row ? pr.s_w[n] : pr.s_w[0];
            }
        }
    }

    pdl_wait();

    // ---- 2. quantise the M tokens into shared memory (8-value pieces; K % 64 == 0). Thread
    //         pieces c = threadIdx.x + 256 it; while there are at most kHold = 8 / MT of them
    //         per token they stay in registers (slot m * kHold + it) between the amax pass and
    //         the quantising pass, else they are re-read.
    constexpr int kHold = 8 / MT;
    const int Mreal = p.M;
    const int pieces = static_cast<int>(K >> 3);
    const int ppt = (pieces + kMmaThreads - 1) / kMmaThreads;
    const bool hold = ppt <= kHold;
    uint4 xv[MT * kHold];
    float s_tok[MT];
    if (p.q_in == nullptr) {
        uint32_t mx[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) mx[m] = 0;
        if (hold) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int it = 0; it < kHold; ++it) {
                    const int c = threadIdx.x + it * kMmaThreads;
                    xv[m * kHold + it] = (m < Mreal && it < ppt && c < pieces)
                                             ? reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c]
                                             : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int it = 0; it < kHold; ++it) mx[m] = max(mx[m], absmax8_bits(xv[m * kHold + it]));
        } else {
            for (int c = threadIdx.x; c < pieces; c += kMmaThreads) {
                uint4 v[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    v[m] = m < Mreal ? reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c]
                                     : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int m = 0; m < MT; ++m) mx[m] = max(mx[m], absmax8_bits(v[m]));
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint32_t r = __reduce_max_sync(0xFFFFFFFFu, mx[m]);
            if (lane == 0) s_amax[warp][m] = r;
        }
        __syncthreads();
        uint32_t all[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            all[m] = s_amax[0][m];
#pragma unroll
            for (int w = 1; w < kMmaWarps; ++w) all[m] = max(all[m], s_amax[w][m]);
        }
        if (p.act_per_tensor) {  // one scale for all real tokens ("推理优化" §2.2, I2_S)
            uint32_t tt = 0;
#pragma unroll
            for (int m = 0; m < MT; ++m) tt = m < Mreal ? max(tt, all[m]) : tt;
#pragma unroll
            for (int m = 0; m < MT; ++m) all[m] = tt;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) s_tok[m] = __fdiv_rn(127.0f, fmaxf(bf16_lo(all[m]), kActEps));
    } else {
#pragma unroll
        for (int m = 0; m < MT; ++m) s_tok[m] = 0.0f;
    }
    int qs[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) qs[m] = 0;
    // Every thread runs the same ppt iterations (the lane-pair shuffle needs both lanes).
#pragma unroll
    for (int it = 0; it < kMaxPieceIters; ++it) {
        if (it >= ppt) break;
        const int c = threadIdx.x + it * kMmaThreads;
        const bool valid = c < pieces;
        const int grp = c >> 1;  // group grp lives in chunk grp / 4 as its group grp % 4
        const int64_t off = (int64_t(grp & 3) * C + (grp >> 2)) * 16 + (c & 1) * 8;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            uint2 nat = make_uint2(0u, 0u);
            if (valid && m < Mreal) {
                if (p.q_in != nullptr) {
                    nat = reinterpret_cast<const uint2*>(p.q_in + int64_t(m) * K)[c];
                } else {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (hold) {
#pragma unroll
                        for (int h = 0; h < kHold; ++h)
                            if (h == it) v = xv[m * kHold + h];
                    } else {
                        v = reinterpret_cast<const uint4*>(p.x + int64_t(m) * K)[c];
                    }
                    nat = quant8(v, s_tok[m]);
                }
            }
            qs[m] += bytesum(nat.x) + bytesum(nat.y);
            const uint2 out = permute_group_half(nat, lane & 1);
            if (valid) *reinterpret_cast<uint2*>(s_q + m * tok_stride + off) = out;
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const int r = __reduce_add_sync(0xFFFFFFFFu, qs[m]);
        if (lane == 0) s_qs[warp][m] = r;
    }
    __syncthreads();

    // ---- 3. the warp's (row tile, K slice): 2 MMAs per packed word pair, into four
    //         accumulators (by word parity and shift pair) so consecutive MMAs do not wait on
    //         each other; the int32 sums are exact in any order. The weight rows must have
    //         landed first (a bounded wait: on expiry the watchdog word records it, the
    //         results are garbage, and the copies still get a bounded wait before exit).
    const bool w_ok = mbar_wait_bounded(wbar, 0, err, kErrWaitTmaFull, nullptr);
    if (!w_ok) mbar_wait_bounded(wbar, 0, err, kErrWaitDrain, nullptr);
    int d[4][4] = {};
    const uint8_t* qtok = s_q + g * tok_stride;  // this lane's token (column g)
    const bool b_lane = g < Mreal;
    const uint8_t* wrow_a = s_w + (16 * wrt + g) * wstride;
    const uint8_t* wrow_b = wrow_a + 8 * wstride;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = c0 + t + 4 * i;
        const bool ok = c < c1;
        if (4 * i < c1 - c0) {  // warp-uniform: some lane of the quad still has chunk i
            uint4 wai = make_uint4(0u, 0u, 0u, 0u), wbi = make_uint4(0u, 0u, 0u, 0u);
            if (ok) {
                wai = *reinterpret_cast<const uint4*>(wrow_a + c * 16);
                wbi = *reinterpret_cast<const uint4*>(wrow_b + c * 16);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (ok && b_lane)
                    q = *reinterpret_cast<const uint4*>(qtok + (int64_t(j) * C + c) * 16);
                const uint32_t ua = j == 0 ? wai.x : j == 1 ? wai.y : j == 2 ? wai.z : wai.w;
                const uint32_t ub = j == 0 ? wbi.x : j == 1 ? wbi.y : j == 2 ? wbi.z : wbi.w;
                mma_u8s8_16832(d[2 * (j & 1)], ua & 0x03030303u, ub & 0x03030303u,
                               (ua >> 2) & 0x03030303u, (ub >> 2) & 0x03030303u, q.x, q.y);
                mma_u8s8_16832(d[2 * (j & 1) + 1], (ua >> 4) & 0x03030303u,
                               (ub >> 4) & 0x03030303u, (ua >> 6) & 0x03030303u,
                               (ub >> 6) & 0x03030303u, q.z, q.w);
            }
        }
    }
    // D fragment: d0 (row g, token 2t), d1 (row g, token 2t + 1), d2 / d3 the same for row g + 8.
    {
        int32_t* r = s_red + warp * 128;
        r[g * 8 + 2 * t] = d[0][0] + d[1][0] + d[2][0] + d[3][0];
        r[g * 8 + 2 * t + 1] = d[0][1] + d[1][1] + d[2][1] + d[3][1];
        r[(g + 8) * 8 + 2 * t] = d[0][2] + d[1][2] + d[2][2] + d[3][2];
        r[(g + 8) * 8 + 2 * t + 1] = d[0][3] + d[1][3] + d[2][3] + d[3][3];
    }
    __syncthreads();

    // ---- 4. epilogue: thread o, every token: sum the K slices, remove sum q,
    //         y = acc * (s_w * (1 / s_x)) with each product rounded
    if (o_valid) {
        auto acc_of = [&](int lt, int m) {
            int32_t a = 0;
            for (int w = lt * ks; w < (lt + 1) * ks; ++w) a += s_red[w * 128 + o_r16 * 8 + m];
            return a;
        };
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= Mreal) break;
            int32_t qtot = 0;
#pragma unroll
            for (int w = 0; w < kMmaWarps; ++w) qtot += s_qs[w][m];
            if constexpr (SW) {
                const float rx = __frcp_rn(s_tok[m]);
                const float gv = __fmul_rn(__int2float_rn(acc_of(o_lt, m) - qtot), __fmul_rn(o_sa, rx));
                const float uv = __fmul_rn(__int2float_rn(acc_of(o_lt + 1, m) - qtot), __fmul_rn(o_sb, rx));
                static_cast<uint16_t*>(o_y)[int64_t(m) * o_ld] = swiglu_bf16_bits(gv, uv);
            } else {
                const int32_t acc = acc_of(o_lt, m) - qtot;
                if (p.out_kind == 2) {
                    static_cast<int32_t*>(o_y)[int64_t(m) * o_ld] = acc;
                } else {
                    const float yv =
                        __fmul_rn(__int2float_rn(acc), __fmul_rn(o_sa, __frcp_rn(s_tok[m])));
                    if (p.out_kind == 0)
                        static_cast<__nv_bfloat16*>(o_y)[int64_t(m) * o_ld] = __float2bfloat16_rn(yv);
                    else
                        static_cast<float*>(o_y)[int64_t(m) * o_ld] = yv;
                }
            }
        }
    }
}

template <int MT, int CPT, bool SW>
cudaError_t launch_mma3(const GemvParams& p, int rt, int grid, int32_t* err, cudaStream_t stream,
                        bool pdl) {
    auto kern = gemv_mma_kernel<MT, CPT, SW>;
    const size_t smem = mma_smem_bytes(MT, rt, p.K);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p, rt, err);
}

constexpr int kMmaCpt[] = {1, 2, 3, 4, 6, 8};
constexpr int kMmaMaxCpt = 8;

template <int MT, bool SW>
cudaError_t launch_mma2(const GemvParams& p, int rt, int grid, int cpt, int32_t* err,
                        cudaStream_t stream, bool pdl) {
    switch (cpt) {
        case 1: return launch_mma3<MT, 1, SW>(p, rt, grid, err, stream, pdl);
        case 2: return launch_mma3<MT, 2, SW>(p, rt, grid, err, stream, pdl);
        case 3: return launch_mma3<MT, 3, SW>(p, rt, grid, err, stream, pdl);
        case 4: return launch_mma3<MT, 4, SW>(p, rt, grid, err, stream, pdl);
        case 6: return launch_mma3<MT, 6, SW>(p, rt, grid, err, stream, pdl);
        default: return launch_mma3<MT, 8, SW>(p, rt, grid, err, stream, pdl);
    }
}

template <int MT>
cudaError_t launch_mma1(const GemvParams& p, int rt, int grid, int cpt, int32_t* err,
                        cudaStream_t stream, bool pdl) {
    return p.swiglu ? launch_mma2<MT, true>(p, rt, grid, cpt, err, stream, pdl)
                    : launch_mma2<MT, false>(p, rt, grid, cpt, err, stream, pdl);
}

}  // namespace

// Tiles of 16 rows per CTA: the fewest (1, 2, 4 or 8; at least 2 for SwiGLU) that keep the
// grid within one CTA per SM, the chunks per lane within the largest instantiation and the
// shared memory (weight rows, quantised tokens) within a CTA's; where no count keeps the grid
// within the SMs, the largest that fits.
constexpr size_t kMmaSmemMax = 200 * 1024;

bool gemv_mma_plan(const GemvParams& p, int sms, int* rt, int* grid, int* cpt) {
    if (p.M < 1 || p.M > 8 || p.K > int64_t(kMaxPieceIters) * kMmaThreads * 8) return false;
    const int64_t C = p.K >> 6;
    const int mt = p.M <= 1 ? 1 : p.M <= 2 ? 2 : p.M <= 4 ? 4 : 8;
    const int64_t rows = p.swiglu ? 2 * p.total_rows : p.total_rows;
    const int64_t tiles = (rows + 15) / 16;
    int best = 0;
    for (int r : {1, 2, 4, 8}) {
        if (p.swiglu && r < 2) continue;
        const int ks = kMmaWarps / r;
        const int64_t need = ((C + ks - 1) / ks + 3) / 4;
        if (need > kMmaMaxCpt || mma_smem_bytes(mt, r, p.K) > kMmaSmemMax) continue;
        best = r;
        if ((tiles + r - 1) / r <= sms) break;
    }
    if (best == 0) return false;
    const int ks = kMmaWarps / best;
    const int64_t need = ((C + ks - 1) / ks + 3) / 4;
    int c = kMmaMaxCpt;
    for (int v : kMmaCpt)
        if (v >= need) {
            c = v;
            break;
        }
    *rt = best;
    *grid = static_cast<int>((tiles + best - 1) / best);
    *cpt = c;
    return true;
}

cudaError_t launch_gemv_mma(const GemvParams& p, int rt, int grid, int cpt, int32_t* err,
                            cudaStream_t stream, bool pdl) {
    if (p.M <= 1) return launch_mma1<1>(p, rt, grid, cpt, err, stream, pdl);
    if (p.M <= 2) return launch_mma1<2>(p, rt, grid, cpt, err, stream, pdl);
    if (p.M <= 4) return launch_mma1<4>(p, rt, grid, cpt, err, stream, pdl);
    return launch_mma1<8>(p, rt, grid, cpt, err, stream, pdl);
}

}  // namespace bitnet
