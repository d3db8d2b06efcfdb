// Base-3 weight format, five ternary weights per byte (page "将 BitNet 三元查找表集成到自定义
// Triton 内核中", step 1 of its recipe: ternary values packed into uint8 bitmaps, 4-5 per byte;
// 3^5 = 243 <= 256, so 1.6 bits per weight against the 2-bit format's 2): a packing kernel and
// a one-token GEMV that reads it.
//
// Layout: a row is cut into chunks of 80 weights (16 bytes); byte p of chunk c holds weights
// k = 80c + 16d + p (d = 0..4) as sum_d (t + 1) 3^d; weights past K count as 0; a row takes
// 16 ceil(K / 80) bytes. Byte p of a chunk thus carries position p of the chunk's five
// 16-weight groups, and decoding a chunk yields five 32-bit words in the 2-bit format (code of
// k = 16u + 4b + i in bits 2i of byte b of word u), which feed the same permuted-q dp4a
// product as the 2-bit GEMV.
//
// Decoding without a divide: within 16-bit lanes (two bytes per 32-bit register), for x < 256
// floor(x / 3) = (x * 171) >> 9 exactly and x * 171 < 2^16, so one multiply, shift and mask
// give two quotients at once and the digit is x - 3 floor(x / 3). Four digit steps and the
// last quotient give the five digits; a shift-or packs four bytes' digits into one 2-bit byte.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr int kB3Warps = 16;
constexpr int kB3Threads = kB3Warps * 32;

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

// One 16-byte chunk (80 weights) -> the five 2-bit-format words of its groups.
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

// sum over the 16 weights of one 2-bit-format word of code * q (q permuted, one uint4).
__device__ __forceinline__ int word_dot(uint32_t word, const uint4 q, int acc) {
    acc = __dp4a(int(word & 0x03030303u), int(q.x), acc);
    acc = __dp4a(int((word >> 2) & 0x03030303u), int(q.y), acc);
    acc = __dp4a(int((word >> 4) & 0x03030303u), int(q.z), acc);
    return __dp4a(int((word >> 6) & 0x03030303u), int(q.w), acc);
}

// One token. Each warp takes rows warp_id, warp_id + total warps, ... (two at a time, the next
// pair's chunks loaded before the current pair is reduced); lane l holds chunks l + 32 i.
// q of the token lives in shared memory as [5][C3] uint4: group u at (u % 5) C3 + u / 5, so
// lanes reading consecutive chunks read consecutive addresses.
template <int CPL>
__global__ void __launch_bounds__(kB3Threads, CPL <= 4 ? 2 : 1) gemv_b3_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ uint4 s_q[];
    __shared__ uint32_t s_red[kB3Warps];
    __shared__ int32_t s_qs[kB3Warps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int64_t rb = b3_row_bytes(K);
    const int C3 = static_cast<int>(rb >> 4);  // 80-weight chunks per row
    const int groups = static_cast<int>(K >> 4);
    const GemvProj& pr = p.proj[0];
    const int64_t N = pr.N;
    const int64_t wstride = int64_t(gridDim.x) * kB3Warps;
    int64_t row = int64_t(blockIdx.x) * kB3Warps + warp;

    auto load_row = [&](int64_t r, uint4 (&w)[CPL]) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            w[i] = (r < N && c < C3) ? ldg_stream_v4(pr.packed + r * rb + int64_t(c) * 16)
                                     : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 wa[CPL], wb[CPL];
    load_row(row, wa);
    load_row(row + wstride, wb);
    pdl_trigger();
    pdl_wait();

    // ---- quantise the token (amax over the CTA, then permuted q into shared memory)
    const int pieces = static_cast<int>(K >> 3);
    uint32_t mx = 0;
    for (int c = threadIdx.x; c < pieces; c += kB3Threads)
        mx = max(mx, absmax8_bits(reinterpret_cast<const uint4*>(p.x)[c]));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    uint32_t all = s_red[0];
#pragma unroll
    for (int i = 1; i < kB3Warps; ++i) all = max(all, s_red[i]);
    const float s = __fdiv_rn(127.0f, fmaxf(bf16_lo(all), kActEps));
    int qs = 0;
    uint8_t* sq = reinterpret_cast<uint8_t*>(s_q);
    for (int base = warp * 32; base < pieces; base += kB3Threads) {  // warp-uniform trips
        const int c = base + lane;
        uint2 nat = make_uint2(0u, 0u);
        if (c < pieces) nat = quant8(reinterpret_cast<const uint4*>(p.x)[c], s);
        qs += bytesum(nat.x) + bytesum(nat.y);
        const uint2 out = permute_group_half(nat, lane & 1);
        if (c < pieces) {
            const int u = c >> 1;
            *reinterpret_cast<uint2*>(sq + (int64_t(u % 5) * C3 + u / 5) * 16 + (c & 1) * 8) = out;
        }
    }
    qs = __reduce_add_sync(0xFFFFFFFFu, qs);
    if (lane == 0) s_qs[warp] = qs;
    __syncthreads();
    int32_t qtot = 0;
#pragma unroll
    for (int i = 0; i < kB3Warps; ++i) qtot += s_qs[i];
    const float rx = __frcp_rn(s);

    auto row_dot = [&](const uint4 (&w)[CPL]) -> int {
        int a0 = 0, a1 = 0;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < C3) {
                uint32_t wd[5];
                decode_b3_chunk(w[i], wd);
#pragma unroll
                for (int d = 0; d < 5; ++d) {
                    const int u = 5 * c + d;
                    if (u < groups) {  // padding groups past K carry no q
                        const uint4 q = s_q[d * C3 + c];
                        if (d & 1)
                            a1 = word_dot(wd[d], q, a1);
                        else
                            a0 = word_dot(wd[d], q, a0);
                    }
                }
            }
        }
        return a0 + a1;
    };
    auto finish = [&](int64_t r, int dot) {
        const int32_t acc = __reduce_add_sync(0xFFFFFFFFu, dot) - qtot;
        if (lane == 0 && r < N) {
            if (p.out_kind == 2) {
                static_cast<int32_t*>(pr.y)[r] = acc;
            } else {
                const float sw = pr.per_row ? pr.s_w[r] : pr.s_w[0];
                const float yv = __fmul_rn(__int2float_rn(acc), __fmul_rn(sw, rx));
                if (p.out_kind == 0)
                    static_cast<__nv_bfloat16*>(pr.y)[r] = __float2bfloat16_rn(yv);
                else
                    static_cast<float*>(pr.y)[r] = yv;
            }
        }
    };
    while (row < N) {  // warp-uniform
        const int da = row_dot(wa);
        const int db = row_dot(wb);
        const int64_t r0 = row;
        row += 2 * wstride;
        load_row(row, wa);
        load_row(row + wstride, wb);
        finish(r0, da);
        finish(r0 + wstride, db);
    }
}

template <int CPL>
cudaError_t launch_b3_cpl(const GemvParams& p, int sms, cudaStream_t stream, bool pdl) {
    auto kern = gemv_b3_kernel<CPL>;
    const int64_t C3 = b3_row_bytes(p.K) >> 4;
    const size_t smem = size_t(5 * C3) * 16;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t want = (p.proj[0].N + kB3Warps - 1) / kB3Warps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(want < 2 * sms ? want : 2 * sms));
    cfg.blockDim = dim3(kB3Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t launch_pack_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                           cudaStream_t stream) {
    const int64_t total = N * b3_row_bytes(K);
    pack_b3_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(t, N, K, packed);
    return cudaGetLastError();
}

bool gemv_b3_supported(int64_t K) { return K >= 64 && K <= 16384 && K % 64 == 0; }

cudaError_t launch_gemv_b3(const GemvParams& p, int sms, cudaStream_t stream, bool pdl) {
    const int64_t C3 = b3_row_bytes(p.K) >> 4;
    const int cpl = static_cast<int>((C3 + 31) / 32);
    if (cpl <= 1) return launch_b3_cpl<1>(p, sms, stream, pdl);
    if (cpl <= 2) return launch_b3_cpl<2>(p, sms, stream, pdl);
    if (cpl <= 4) return launch_b3_cpl<4>(p, sms, stream, pdl);
    return launch_b3_cpl<8>(p, sms, stream, pdl);
}

}  // namespace bitnet
