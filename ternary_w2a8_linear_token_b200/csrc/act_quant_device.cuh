// Device helpers of the per-token absmax int8 activation quantiser, shared by the standalone
// quantiser (kernels_quant.cu) and the GEMVs that fuse it (page "BitNet-Triton", section
// "技术架构：融合内核的三重优化", item 3 "融合激活量化"; page "BitNet 1-bit LLM推理优化",
// section 3.2 "激活量化策略"):
//   amax = max_k |x[m,k]|,  s_x = 127 / max(amax, 1e-5),  q = clamp(rint(x * s_x), -128, 127).
//
// Permuted in-group order (the operand layout of every contraction here): inside each group
// of 16 values along K, byte 4i + b holds k = 4b + i. A packed 32-bit weight word covers 16
// weights, and its 2-bit fields for k = i, 4+i, 8+i, 12+i sit in bits 2i..2i+1 of its four
// bytes, so against q in this order the weights unpack with one mask per four weights.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace bitnet {

constexpr float kActEps = 1e-5f;

// The two bf16 values of a 32-bit word as binary32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// q = clamp(rint(x * s_x), -128, 127) for one value, as the bits of a binary32 whose low byte
// is q. The clamp never acts: s_x = RN(127 / a) with a = max(amax, 1e-5) >= |x|, so
// |x * s_x| <= 127 (1 + 2^-24)^2 < 127.5. Adding 1.5 * 2^23 to the rounded product lands in
// [2^23, 2^24), where the binary32 spacing is 1, so that sum is rint(x * s_x) + 1.5 * 2^23
// (round half to even) and its low mantissa byte is q in two's complement. Both steps are
// separately rounded intrinsics, so nothing is contracted into an FMA.
__device__ __forceinline__ uint32_t qbits(float xv, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(xv, s), 12582912.0f));
}

// Low bytes of a, b, c, d -> one word (byte 0 = a).
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// 8 bf16 (one uint4, natural order) -> 8 int8 as two words (values k..k+3, k+4..k+7).
__device__ __forceinline__ uint2 quant8(const uint4 v, float s) {
    uint2 r;
    r.x = pack4(qbits(bf16_lo(v.x), s), qbits(bf16_hi(v.x), s), qbits(bf16_lo(v.y), s),
                qbits(bf16_hi(v.y), s));
    r.y = pack4(qbits(bf16_lo(v.z), s), qbits(bf16_hi(v.z), s), qbits(bf16_lo(v.w), s),
                qbits(bf16_hi(v.w), s));
    return r;
}

// Sum of the four signed bytes of w.
__device__ __forceinline__ int bytesum(uint32_t w) { return __dp4a(int(w), 0x01010101, 0); }

// max |x| over the 8 bf16 of v, as the bit pattern of |x| (bf16 magnitudes order as unsigned
// integers, so the maximum is exact).
__device__ __forceinline__ uint32_t absmax8_bits(const uint4 v) {
    const uint32_t a = max(max(v.x & 0x7FFFu, v.x >> 16 & 0x7FFFu), max(v.y & 0x7FFFu, v.y >> 16 & 0x7FFFu));
    const uint32_t b = max(max(v.z & 0x7FFFu, v.z >> 16 & 0x7FFFu), max(v.w & 0x7FFFu, v.w >> 16 & 0x7FFFu));
    return max(a, b);
}

// Turns the natural-order words (lo = k..k+3, hi = k+4..k+7) held by lane pair
// (2p, 2p+1) of one 16-group into that lane's 8 bytes of the permuted group. Both lanes of
// the pair must execute it (one shuffle).
__device__ __forceinline__ uint2 permute_group_half(uint2 nat, int h) {
    const uint32_t p01 = __byte_perm(nat.x, nat.y, 0x5140);  // pieces for words 0 and 1
    const uint32_t p23 = __byte_perm(nat.x, nat.y, 0x7362);  // pieces for words 2 and 3
    const uint32_t own = h ? p23 : p01;
    const uint32_t send = h ? p01 : p23;
    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
    const uint32_t lo = h ? recv : own;  // pieces from the first 8 values of the group
    const uint32_t hi = h ? own : recv;  // pieces from the last 8 values of the group
    return make_uint2(__byte_perm(lo, hi, 0x5410), __byte_perm(lo, hi, 0x7632));
}

}  // namespace bitnet

// Sum over one packed weight word (16 codes c = t + 1) times the token's permuted q (one
// uint4, word i against the codes at bits 2i..2i+1 of every byte). The codes are masked in
// place instead of shifted down: byte values c * 4^i with c in {0, 1, 2}, unsigned, against
// signed q, so acc.{x, y, z, w} collect 4^i * sum c q for i = 0 .. 3 with one AND and one dp4a
// per four weights; code_dot_total divides the factors back out, exactly (each sum is a
// multiple of its 4^i; |64 sum c q| stays far inside int32 for a lane's share of a row).
__device__ __forceinline__ int dp4a_u8s8(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void code_dot_acc(uint32_t word, const uint4 q, int4& acc) {
    acc.x = dp4a_u8s8(word & 0x03030303u, q.x, acc.x);
    acc.y = dp4a_u8s8(word & 0x0C0C0C0Cu, q.y, acc.y);
    acc.z = dp4a_u8s8(word & 0x30303030u, q.z, acc.z);
    acc.w = dp4a_u8s8(word & 0xC0C0C0C0u, q.w, acc.w);
}

__device__ __forceinline__ int code_dot_total(const int4 acc) {
    return (acc.x + (acc.y >> 2)) + ((acc.z >> 4) + (acc.w >> 6));
}
