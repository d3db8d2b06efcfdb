// Grid-stride one-token GEMV for large weight matrices: the MLP's interleaved gate/up matrix with
// SwiGLU in the 2-bit format, and plain projections in the base-3 format (page "BitNet-Triton",
// section "技术架构：融合内核的三重优化", items 1 and 3: weights unpacked in the kernel,
// activation quantiser fused; page "将 BitNet 三元查找表集成到自定义 Triton 内核中", step 1: 4-5
// ternary values per byte). Plain 2-bit projections take the streaming kernel, which measured
// faster for them.
//
// At one token the product reads every weight byte once, so for a large matrix it runs at the
// rate bytes arrive; that rate is set by the bytes each SM keeps in flight. Here every warp
// keeps a ring of NB row pairs in registers: while it reduces pair i, the loads of pairs
// i + 1 .. i + NB - 1 are in flight. One 16-warp CTA per SM walks the rows (or, for the
// MLP's interleaved gate/up matrix, the output pairs) with a grid stride; lanes hold the
// 16-byte chunks l, l + 32, ... of a row. x is quantised once per CTA into shared memory in
// the permuted in-group order, against which a 2-bit word unpacks with one shift and mask per
// four weights (dp4a on codes t + 1; sum q t = sum q c - sum q). A base-3 chunk (80 weights)
// is first decoded into the five 2-bit words of its groups (decode_b3_chunk).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"
#include "swiglu_device.cuh"

namespace bitnet {
namespace {

constexpr int kGsWarps = 16;
constexpr int kGsThreads = kGsWarps * 32;

// One base-3 chunk (16 bytes, 80 weights: byte p holds k = 16d + p of the chunk, d = 0..4, as
// sum_d (t + 1) 3^d) -> the five 2-bit-format words of its 16-weight groups (code of position
// 4b + i of group d in bits 2i of byte b of word d). Two bytes per register in 16-bit lanes:
// for x < 256, floor(x / 3) = (x * 171) >> 9 exactly and x * 171 < 2^16, so one multiply,
// shift and mask give both quotients and the digit is x - 3 floor(x / 3); four steps and the
// last quotient give the five digits; a shift-or packs four bytes' digits into one byte.
__device__ __forceinline__ void decode_b3_chunk(const uint4 v, uint32_t (&w)[5]) {
#pragma unroll
    for (int d = 0; d < 5; ++d) w[d] = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t s = b == 0 ? v.x : b == 1 ? v.y : b == 2 ? v.z : v.w;
        uint32_t lo = s & 0x00FF00FFu;         // bytes 4b and 4b + 2 of the chunk
        uint32_t hi = (s >> 8) & 0x00FF00FFu;  // bytes 4b + 1 and 4b + 3
#pragma unroll
        for (int d = 0; d < 5; ++d) {
            uint32_t dl = lo, dh = hi;  // the last digit is the remaining quotient
            if (d < 4) {
                const uint32_t ql = ((lo * 171u) >> 9) & 0x007F007Fu;
                const uint32_t qh = ((hi * 171u) >> 9) & 0x007F007Fu;
                dl = lo - 3u * ql;
                dh = hi - 3u * qh;
                lo = ql;
                hi = qh;
            }
            // bits 0-1: byte 4b, 2-3: byte 4b + 1, 4-5: byte 4b + 2, 6-7: byte 4b + 3
            const uint32_t m = dl | (dh << 2);
            w[d] |= ((m | (m >> 12)) & 0xFFu) << (8 * b);
        }
    }
}

// One row of a pair in flight: this lane's chunks and, for lane 0, the row's scale.
template <int CPL>
struct RowBuf {
    uint4 w[CPL];
    float sw;
};

// CPL: chunks per lane. B3: base-3 weights. SW: interleaved gate/up matrix, output h = SwiGLU.
// NB: row pairs in the register ring (NB - 1 in flight while one is reduced).
template <int CPL, bool B3, bool SW, int NB>
__global__ void __launch_bounds__(kGsThreads, 1) gemv_gs_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ uint4 s_q[];
    __shared__ uint32_t s_red[kGsWarps];
    __shared__ int32_t s_qs[kGsWarps];
    constexpr int G = B3 ? 5 : 4;  // 16-weight groups per chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int64_t rb = B3 ? b3_row_bytes(K) : (K >> 2);
    const int C = static_cast<int>(rb >> 4);  // chunks per row
    const int groups = static_cast<int>(K >> 4);
    const int64_t S = int64_t(gridDim.x) * kGsWarps;  // warps in the grid
    const int64_t w0 = int64_t(blockIdx.x) * kGsWarps + warp;
    const int64_t units = p.total_rows;  // rows, or output pairs for SwiGLU

    // Pair k of this warp: rows (a, b) and whether the pair exists.
    auto pair_rows = [&](int64_t k, int64_t* a, int64_t* b) -> bool {
        if constexpr (SW) {
            const int64_t j = w0 + k * S;  // output pair: gate row and up row
            *a = (j / kSwigluBlock) * (2 * kSwigluBlock) + j % kSwigluBlock;
            *b = *a + kSwigluBlock;
            return j < units;
        } else {
            *a = w0 + 2 * k * S;
            *b = *a + S;
            return *a < units;
        }
    };
    auto load_row = [&](int64_t r, RowBuf<CPL>& buf) {
        const uint8_t* base = nullptr;
        float sw = 0.0f;
        if (SW ? r < 2 * units : r < units) {
            int pj = 0;
            if constexpr (!SW) {
#pragma unroll
                for (int j = 1; j < kMaxProj; ++j)
                    if (j < p.nproj && r >= p.proj[j].row_begin) pj = j;
            }
            const GemvProj& pr = p.proj[pj];
            const int64_t n = r - pr.row_begin;
            base = pr.packed + n * rb;
            if (lane == 0 && p.out_kind != 2)
                sw = pr.per_row ? pr.s_w[n] : pr.s_w[SW ? (r / kSwigluBlock) & 1 : 0];
        }
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            buf.w[i] = (base && c < C) ? ldg_stream_v4(base + int64_t(c) * 16)
                                       : make_uint4(0u, 0u, 0u, 0u);
        }
        buf.sw = sw;
    };

    RowBuf<CPL> ra[NB], rbuf[NB];
#pragma unroll
    for (int s = 0; s < NB - 1; ++s) {
        int64_t a, b;
        pair_rows(s, &a, &b);
        load_row(a, ra[s]);
        load_row(b, rbuf[s]);
    }
    pdl_trigger();
    pdl_wait();

    // ---- quantise the token (amax over the CTA, then permuted q into shared memory)
    const int pieces = static_cast<int>(K >> 3);
    uint32_t mx = 0;
    for (int c = threadIdx.x; c < pieces; c += kGsThreads)
        mx = max(mx, absmax8_bits(reinterpret_cast<const uint4*>(p.x)[c]));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    uint32_t all = s_red[0];
#pragma unroll
    for (int i = 1; i < kGsWarps; ++i) all = max(all, s_red[i]);
    const float s = __fdiv_rn(127.0f, fmaxf(bf16_lo(all), kActEps));
    int qs = 0;
    uint8_t* sq = reinterpret_cast<uint8_t*>(s_q);
    for (int base = warp * 32; base < pieces; base += kGsThreads) {  // warp-uniform trips
        const int c = base + lane;
        uint2 nat = make_uint2(0u, 0u);
        if (c < pieces) nat = quant8(reinterpret_cast<const uint4*>(p.x)[c], s);
        qs += bytesum(nat.x) + bytesum(nat.y);
        const uint2 out = permute_group_half(nat, lane & 1);
        if (c < pieces) {
            const int u = c >> 1;  // group u at (u % G) C + u / G
            *reinterpret_cast<uint2*>(sq + (int64_t(u % G) * C + u / G) * 16 + (c & 1) * 8) = out;
        }
    }
    qs = __reduce_add_sync(0xFFFFFFFFu, qs);
    if (lane == 0) s_qs[warp] = qs;
    __syncthreads();
    int32_t qtot = 0;
#pragma unroll
    for (int i = 0; i < kGsWarps; ++i) qtot += s_qs[i];
    const float rx = __frcp_rn(s);

    auto row_dot = [&](const RowBuf<CPL>& buf) -> int {
        int4 a0 = make_int4(0, 0, 0, 0), a1 = make_int4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < C) {
                uint32_t wd[G];
                if constexpr (B3) {
                    decode_b3_chunk(buf.w[i], wd);
                } else {
                    wd[0] = buf.w[i].x;
                    wd[1] = buf.w[i].y;
                    wd[2] = buf.w[i].z;
                    wd[3] = buf.w[i].w;
                }
#pragma unroll
                for (int d = 0; d < G; ++d) {
                    if (!B3 || G * c + d < groups) {  // base-3 padding groups carry no q
                        const uint4 q = s_q[d * C + c];
                        code_dot_acc(wd[d], q, (d & 1) ? a1 : a0);
                    }
                }
            }
        }
        return code_dot_total(a0) + code_dot_total(a1);
    };
    auto store_row = [&](int64_t r, int32_t acc, float sw) {
        int pj = 0;
#pragma unroll
        for (int j = 1; j < kMaxProj; ++j)
            if (j < p.nproj && r >= p.proj[j].row_begin) pj = j;
        const GemvProj& pr = p.proj[pj];
        const int64_t n = r - pr.row_begin;
        if (p.out_kind == 2) {
            static_cast<int32_t*>(pr.y)[n] = acc;
        } else {
            const float yv = __fmul_rn(__int2float_rn(acc), __fmul_rn(sw, rx));
            if (p.out_kind == 0)
                static_cast<__nv_bfloat16*>(pr.y)[n] = __float2bfloat16_rn(yv);
            else
                static_cast<float*>(pr.y)[n] = yv;
        }
    };
    auto process = [&](int64_t k, const RowBuf<CPL>& A, const RowBuf<CPL>& B) {
        int64_t a, b;
        pair_rows(k, &a, &b);
        const int da = row_dot(A);
        const int db = row_dot(B);
        const int32_t ta = __reduce_add_sync(0xFFFFFFFFu, da) - qtot;
        const int32_t tb = __reduce_add_sync(0xFFFFFFFFu, db) - qtot;
        if (lane == 0) {
            if constexpr (SW) {
                const float g = __fmul_rn(__int2float_rn(ta), __fmul_rn(A.sw, rx));
                const float u = __fmul_rn(__int2float_rn(tb), __fmul_rn(B.sw, rx));
                static_cast<uint16_t*>(p.proj[0].y)[w0 + k * S] = swiglu_bf16_bits(g, u);
            } else {
                store_row(a, ta, A.sw);
                if (b < units) store_row(b, tb, B.sw);
            }
        }
    };

    // The ring: pair k sits in slot k % NB; before pair k is reduced, pair k + NB - 1 is loaded
    // into the slot pair k - 1 left.
    for (int64_t k0 = 0;; k0 += NB) {
#pragma unroll
        for (int s = 0; s < NB; ++s) {
            const int64_t k = k0 + s;
            int64_t a, b;
            if (!pair_rows(k, &a, &b)) return;  // warp-uniform
            int64_t na, nb;
            pair_rows(k + NB - 1, &na, &nb);
            load_row(na, ra[(s + NB - 1) % NB]);
            load_row(nb, rbuf[(s + NB - 1) % NB]);
            process(k, ra[s], rbuf[s]);
        }
    }
}

template <int CPL, bool B3, bool SW>
cudaError_t launch_gs3(const GemvParams& p, int sms, cudaStream_t stream, bool pdl) {
    constexpr int NB = CPL <= 2 ? 4 : 2;
    auto kern = gemv_gs_kernel<CPL, B3, SW, NB>;
    const int64_t rb = B3 ? b3_row_bytes(p.K) : (p.K >> 2);
    const size_t smem = size_t((B3 ? 5 : 4) * (rb >> 4)) * 16;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t per_cta = SW ? kGsWarps : 2 * kGsWarps;  // units in a CTA's first pass
    const int64_t want = (p.total_rows + per_cta - 1) / per_cta;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(want < sms ? want : sms));
    cfg.blockDim = dim3(kGsThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <bool B3, bool SW>
cudaError_t launch_gs2(const GemvParams& p, int sms, cudaStream_t stream, bool pdl) {
    const int64_t rb = B3 ? b3_row_bytes(p.K) : (p.K >> 2);
    const int cpl = static_cast<int>(((rb >> 4) + 31) / 32);
    if (cpl <= 1) return launch_gs3<1, B3, SW>(p, sms, stream, pdl);
    if (cpl <= 2) return launch_gs3<2, B3, SW>(p, sms, stream, pdl);
    if (cpl <= 4) return launch_gs3<4, B3, SW>(p, sms, stream, pdl);
    return launch_gs3<8, B3, SW>(p, sms, stream, pdl);
}

}  // namespace

bool gemv_gs_supported(const GemvParams& p, bool b3) {
    return p.M == 1 && p.q_in == nullptr && p.K >= 64 && p.K <= 16384 && p.K % 64 == 0 &&
           (b3 ? !p.swiglu : p.swiglu != 0);
}

cudaError_t launch_gemv_gs(const GemvParams& p, bool b3, int sms, cudaStream_t stream, bool pdl) {
    if (b3) return launch_gs2<true, false>(p, sms, stream, pdl);
    if (p.swiglu) return launch_gs2<false, true>(p, sms, stream, pdl);
    return cudaErrorNotSupported;  // plain 2-bit projections take the streaming kernel
}

}  // namespace bitnet
