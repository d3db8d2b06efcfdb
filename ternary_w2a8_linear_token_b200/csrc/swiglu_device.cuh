// SwiGLU of the MLP for one output ("BitNet 深度实战", section 3.2, BitLlamaMLP: the down
// projection's input is silu(gate_proj(x)) * up_proj(x)), shared by the GEMV and the
// tensor-core epilogue. The rounding points are those of the page's module run in bf16:
// the gate and up projections each return bf16, silu returns bf16, and so does the product.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace bitnet {

// silu(z) = z * sigmoid(z) in binary32, branch-free and without overflow: with
// e = exp(-|z|) in (0, 1], silu(z) = z / (1 + e) for z >= 0 and z e / (1 + e) for z < 0.
// expf is CUDA's (within 2 binary32 steps); the divisor lies in [1, 2], where __fdividef is
// within 2 steps, so the result is within a few binary32 steps of the exact value, far
// below the bf16 step it is rounded to next. Below z = -104 e underflows to 0 and the
// result is -0, as is the exactly rounded bf16 value there (|silu(z)| < 2^-134).
__device__ __forceinline__ float silu_f32(float z) {
    const float e = expf(-fabsf(z));
    const float num = z >= 0.0f ? z : __fmul_rn(z, e);
    return __fdividef(num, __fadd_rn(1.0f, e));
}

__device__ __forceinline__ float bf16_round_f32(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}

// g, u: the binary32 dequantised gate and up outputs (acc * f, before any bf16 rounding).
// Returns the bf16 bits of h = bf16(bf16(silu(bf16(g))) * bf16(u)); the product of two
// bf16 values is exact in binary32 above 2^-126, so h is rounded once.
__device__ __forceinline__ uint16_t swiglu_bf16_bits(float g, float u) {
    const float gb = bf16_round_f32(g);
    const float sb = bf16_round_f32(silu_f32(gb));
    const float ub = bf16_round_f32(u);
    return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(sb, ub)));
}

}  // namespace bitnet
