/*
 * Plain CPU oracle for the BitNet b1.58 W2A8 BitLinear forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
 * this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header, table or helper with the CUDA
 * library; the two meet only through the seeded input generators.
 *
 * Every function is a slow, literal restatement of one step of the method, with
 * no blocking, fusion or reordering beyond what the step's definition states.
 * Build flags: -O1 -ffp-contract=off (no FMA contraction), no -ffast-math, so
 * every float operation below is one IEEE-754 binary32 or binary64 operation
 * rounded to nearest-even (the default rounding mode, which is never changed).
 *
 * Sources (web pages on BitNet b1.58):
 *  [P5-2.4] "BitNet 深度实战", section 2.4 "量化函数的细节": the absmean weight
 *           quantiser (scale = mean |W| along the row, clamped at eps = 1e-5;
 *           t = clamp(round(W / scale), -1, 1)) and its worked example.
 *  [P5-3.2] same page, section 3.2: BitLinear uses the same quantiser and the
 *           float product linear(x, t * scale); its BitLlamaMLP feeds the down
 *           projection silu(gate(x)) * up(x) (SwiGLU).
 *  [P5-4.3] same page, section 4.3 "位打包（Bit Packing）存储": four 2-bit codes
 *           per byte, the first weight in bits 0-1 up to the fourth in bits 6-7.
 *  [P5-4.4] same page, section 4.4 "查找表加速": the int8 x ternary product with
 *           an int32 accumulator where +1 adds, -1 subtracts and 0 is skipped.
 *  [P1-arch] "BitNet-Triton：消费级GPU上的1.58-bit大模型推理加速方案", section
 *           "技术架构：融合内核的三重优化": weights stored (N, K/4) uint8, four per
 *           byte; activations quantised to int8 for an int8 matmul.
 *  [P2-3.2] "BitNet 1-bit LLM推理优化：内存布局、量化策略与硬件加速", section 3.2
 *           "激活量化策略": int8 activations with an absmax-style scale, per-tensor
 *           or per-channel.
 *  [P2-2.2] same page, section 2.2 "I2_S（Int2 with Scale）内核": follows the
 *           per-tensor int8 activation quantisation BitNet b1.58 was trained with.
 *  [P3-1]   "将 BitNet 三元查找表集成到自定义 Triton 内核中", step 1 of its recipe:
 *           ternary values packed into uint8 bitmaps, 4-5 of them per byte.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - code = t + 1 (00 = -1, 01 = 0, 10 = +1); code 11 never appears. Section 4.3
 *    of [P5] prints a different map (11 = +1, 00 = 0, 01 = -1); the packed
 *    format of this library uses t + 1.
 *  - Activation quantiser, per token m: amax = max_k |x[m,k]|,
 *    s_x = 127 / max(amax, 1e-5) (binary32 divide), q = clamp(rint(x * s_x),
 *    -128, 127) with a binary32 multiply. The pages print no formula; the eps is
 *    the weight quantiser's.
 *  - Weight scale: mean |W| is the binary64 sum of |W| taken in index order
 *    (row by row, k ascending), divided in binary64 by the count and rounded to
 *    binary32, then clamped below at 1e-5f. Per-row (the page's dim=-1) or
 *    per-tensor (one scale for the matrix).
 *  - Output: y[m,n] = acc[m,n] * s_w / s_x[m], the exact real value, evaluated
 *    in binary64 (error < 2^-52 relative); rounding to bf16 is round-to-nearest-
 *    even of that value.
 *  - SwiGLU: g and u are the bf16 outputs of the gate and up projections;
 *    silu(g) is rounded to bf16, then the product with u is rounded to bf16, the
 *    rounding points of the page's module run in bf16 (each op returns bf16).
 *
 * Return codes: 0 = ok, 1 = bad argument, 2 = invalid data (a weight outside
 * {-1,0,+1}, or a packed code 3).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs FLT_EVAL_METHOD == 0 (each float operation rounded to its own type)"
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_DATA 2

static const float ORACLE_EPS = 1e-5f; /* clamp of both scales, [P5-2.4] */

static float bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ---------------------------------------------------------------------------
 * Weight scale, [P5-2.4]: scale = mean(|W|) along the row (per_row = 1) or over
 * the whole matrix (per_row = 0), clamped below at eps.
 * ------------------------------------------------------------------------- */
int oracle_absmean_scale(const float* W, int64_t N, int64_t K, int per_row, float* s_w) {
    if (!W || !s_w || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double row_sum = 0.0;
        for (int64_t k = 0; k < K; ++k) row_sum += (double)fabsf(W[n * K + k]);
        if (per_row) {
            float mean = (float)(row_sum / (double)K);
            s_w[n] = mean < ORACLE_EPS ? ORACLE_EPS : mean;
        } else {
            total += row_sum;
        }
    }
    if (!per_row) {
        float mean = (float)(total / ((double)N * (double)K));
        s_w[0] = mean < ORACLE_EPS ? ORACLE_EPS : mean;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Ternary weights, [P5-2.4]: t = clamp(round(W / scale), -1, 1). round() is
 * half-to-even (torch.round), W / scale is one binary32 divide. `rounded`
 * (nullable) receives round(W / scale) before the clamp, the "pre-clip" row of
 * the worked example.
 * ------------------------------------------------------------------------- */
int oracle_ternarize(const float* W, int64_t N, int64_t K, int per_row, const float* s_w,
                     int8_t* t, int32_t* rounded) {
    if (!W || !s_w || !t || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    for (int64_t n = 0; n < N; ++n) {
        float scale = per_row ? s_w[n] : s_w[0];
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(W[n * K + k] / scale);
            if (rounded) rounded[n * K + k] = (int32_t)r;
            if (r > 1.0f) r = 1.0f;
            if (r < -1.0f) r = -1.0f;
            t[n * K + k] = (int8_t)r;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * 2-bit packing, [P5-4.3] bit order and [P1-arch] (N, K/4) uint8 shape:
 * weight k of row n lands in byte k/4 of that row at bit 2*(k%4); its code is
 * t + 1.
 * ------------------------------------------------------------------------- */
int oracle_pack(const int8_t* t, int64_t N, int64_t K, uint8_t* packed) {
    if (!t || !packed || N <= 0 || K <= 0 || K % 4 != 0) return ORACLE_BAD_ARG;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < K / 4; ++j) {
            unsigned byte = 0;
            for (int i = 0; i < 4; ++i) {
                int w = t[n * K + 4 * j + i];
                if (w < -1 || w > 1) return ORACLE_BAD_DATA;
                unsigned code = (unsigned)(w + 1);
                byte |= code << (2 * i);
            }
            packed[n * (K / 4) + j] = (uint8_t)byte;
        }
    }
    return ORACLE_OK;
}

/* Inverse of oracle_pack. A code of 3 has no weight and is reported as bad data. */
int oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* t) {
    if (!t || !packed || N <= 0 || K <= 0 || K % 4 != 0) return ORACLE_BAD_ARG;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = packed[n * (K / 4) + k / 4];
            unsigned code = (byte >> (2 * (k % 4))) & 3u;
            if (code == 3u) return ORACLE_BAD_DATA;
            t[n * K + k] = (int8_t)((int)code - 1);
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Base-3 packing, five weights per byte ([P3-1] "每个 8-bit 字节存储 4-5 个三元值":
 * 3^5 = 243 <= 256, 1.6 bits per weight). The digit of a weight is its code t + 1,
 * least significant digit first. The pages fix no layout; the one read here: a row
 * is cut into chunks of 80 weights (16 bytes), and byte p (0..15) of chunk c holds
 * the weights k = 80c + 16d + p for d = 0..4 as sum_d (t + 1) * 3^d. Weights past
 * K count as t = 0. A row takes 16 * ceil(K / 80) bytes.
 * ------------------------------------------------------------------------- */
static int64_t b3_row_bytes(int64_t K) { return 16 * ((K + 79) / 80); }

int oracle_pack_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed) {
    if (!t || !packed || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    const int64_t rb = b3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < rb; ++j) {
            const int64_t c = j / 16, p = j % 16;
            unsigned byte = 0, place = 1;
            for (int d = 0; d < 5; ++d) {
                const int64_t k = 80 * c + 16 * d + p;
                int w = 0;
                if (k < K) {
                    w = t[n * K + k];
                    if (w < -1 || w > 1) return ORACLE_BAD_DATA;
                }
                byte += (unsigned)(w + 1) * place;
                place *= 3u;
            }
            packed[n * rb + j] = (uint8_t)byte;
        }
    }
    return ORACLE_OK;
}

/* Inverse of oracle_pack_b3. A byte above 242 (no five digits), or a padding weight
 * that is not 0, is reported as bad data. */
int oracle_unpack_b3(const uint8_t* packed, int64_t N, int64_t K, int8_t* t) {
    if (!t || !packed || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    const int64_t rb = b3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < rb; ++j) {
            const int64_t c = j / 16, p = j % 16;
            unsigned byte = packed[n * rb + j];
            if (byte > 242u) return ORACLE_BAD_DATA;
            for (int d = 0; d < 5; ++d) {
                const int w = (int)(byte % 3u) - 1;
                byte /= 3u;
                const int64_t k = 80 * c + 16 * d + p;
                if (k < K)
                    t[n * K + k] = (int8_t)w;
                else if (w != 0)
                    return ORACLE_BAD_DATA;
            }
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Per-token absmax int8 activation quantiser ([P1-arch] int8 activations,
 * [P2-3.2] absmax scale; granularity per token). x is bf16 bit patterns.
 * ------------------------------------------------------------------------- */
int oracle_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s_x) {
    if (!x || !q || !s_x || M <= 0 || K <= 0) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(x[m * K + k]));
            if (a > amax) amax = a;
        }
        float denom = amax < ORACLE_EPS ? ORACLE_EPS : amax;
        float s = 127.0f / denom;
        s_x[m] = s;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_float(x[m * K + k]) * s;
            float r = rintf(v);
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            q[m * K + k] = (int8_t)r;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Per-tensor absmax int8 activation quantiser ([P2-2.2] I2_S keeps BitNet
 * b1.58's per-tensor int8 activation setting; [P2-3.2] lists per-tensor scales):
 * one scale for the whole (M, K) input, amax = max over every m and k, then the
 * same s = 127 / max(amax, eps) and q = clamp(rint(x * s), -128, 127) as the
 * per-token quantiser. s_x receives s in each of its M entries.
 * ------------------------------------------------------------------------- */
int oracle_quant_act_per_tensor(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s_x) {
    if (!x || !q || !s_x || M <= 0 || K <= 0) return ORACLE_BAD_ARG;
    float amax = 0.0f;
    for (int64_t i = 0; i < M * K; ++i) {
        float a = fabsf(bf16_to_float(x[i]));
        if (a > amax) amax = a;
    }
    float denom = amax < ORACLE_EPS ? ORACLE_EPS : amax;
    float s = 127.0f / denom;
    for (int64_t m = 0; m < M; ++m) {
        s_x[m] = s;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_float(x[m * K + k]) * s;
            float r = rintf(v);
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            q[m * K + k] = (int8_t)r;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * int8 x ternary contraction with an int32 accumulator, [P5-4.4] and [P5-2.2]:
 * for every output (m, n) walk k; a +1 weight adds the activation, a -1 weight
 * subtracts it, a 0 weight is skipped. No multiply takes place.
 * ------------------------------------------------------------------------- */
int oracle_ternary_matmul(const int8_t* q, const int8_t* t, int64_t M, int64_t N, int64_t K,
                          int32_t* acc) {
    if (!q || !t || !acc || M <= 0 || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int32_t sum = 0;
            for (int64_t k = 0; k < K; ++k) {
                int w = t[n * K + k];
                if (w == 0) continue;
                int a = q[m * K + k];
                if (w == 1) sum += a;
                else if (w == -1) sum -= a;
                else return ORACLE_BAD_DATA;
            }
            acc[m * N + n] = sum;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Dequantisation, [P5-3.2] (the float result is linear(x, t * scale)) with the
 * per-token activation scale divided out: y = acc * s_w / s_x, binary64.
 * ------------------------------------------------------------------------- */
int oracle_dequant(const int32_t* acc, const float* s_x, const float* s_w, int per_row,
                   int64_t M, int64_t N, double* y) {
    if (!acc || !s_x || !s_w || !y || M <= 0 || N <= 0) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double sw = per_row ? (double)s_w[n] : (double)s_w[0];
            y[m * N + n] = (double)acc[m * N + n] * sw / (double)s_x[m];
        }
    }
    return ORACLE_OK;
}

/* Round binary64 values to bf16 (8 significant bits), round-half-even, with
 * overflow to infinity. The result is returned as bf16 bit patterns. */
void oracle_round_bf16(const double* y, int64_t count, uint16_t* out) {
    for (int64_t i = 0; i < count; ++i) {
        double v = y[i];
        float f;
        if (v == 0.0 || isnan(v) || isinf(v)) {
            f = (float)v;
        } else {
            int e;
            double m = frexp(v, &e);            /* v = m * 2^e, 0.5 <= |m| < 1 */
            if (e < -125) {                     /* bf16 subnormal range: fixed quantum 2^-133 */
                double r = nearbyint(ldexp(v, 133));
                f = (float)ldexp(r, -133);
            } else {
                double r = nearbyint(ldexp(m, 8)); /* 8 significant bits */
                double rv = ldexp(r, e - 8);
                f = (fabs(rv) > 3.3895313892515355e38) ? (float)(v > 0 ? INFINITY : -INFINITY)
                                                       : (float)rv;
            }
        }
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        out[i] = (uint16_t)(u >> 16);
    }
}

/* ---------------------------------------------------------------------------
 * The whole BitLinear forward on packed weights, restricted to the sampled
 * token rows m_idx[0..Ms) and output columns n_idx[0..Ns): unpack, quantise
 * the sampled tokens, contract, dequantise. y is (Ms, Ns) binary64. Optional
 * outputs: acc (Ms, Ns) int32, q (Ms, K) int8 and s_x (Ms).
 * ------------------------------------------------------------------------- */
int oracle_bitlinear_sampled(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                             const float* s_w, int per_row, int64_t N,
                             const int64_t* m_idx, int64_t Ms, const int64_t* n_idx, int64_t Ns,
                             double* y, int32_t* acc_out, int8_t* q_out, float* sx_out,
                             int8_t* scratch_t /* K bytes */, int8_t* scratch_q /* Ms*K bytes */,
                             float* scratch_sx /* Ms */) {
    if (!x || !packed || !s_w || !m_idx || !n_idx || !y || !scratch_t || !scratch_q ||
        !scratch_sx || M <= 0 || N <= 0 || K <= 0 || K % 4 != 0 || Ms <= 0 || Ns <= 0)
        return ORACLE_BAD_ARG;
    for (int64_t a = 0; a < Ms; ++a) {
        int64_t m = m_idx[a];
        if (m < 0 || m >= M) return ORACLE_BAD_ARG;
        int rc = oracle_quant_act(x + m * K, 1, K, scratch_q + a * K, scratch_sx + a);
        if (rc) return rc;
    }
    for (int64_t b = 0; b < Ns; ++b) {
        int64_t n = n_idx[b];
        if (n < 0 || n >= N) return ORACLE_BAD_ARG;
        int rc = oracle_unpack(packed + n * (K / 4), 1, K, scratch_t);
        if (rc) return rc;
        for (int64_t a = 0; a < Ms; ++a) {
            int32_t acc;
            rc = oracle_ternary_matmul(scratch_q + a * K, scratch_t, 1, 1, K, &acc);
            if (rc) return rc;
            float sw = per_row ? s_w[n] : s_w[0];
            double yv;
            rc = oracle_dequant(&acc, scratch_sx + a, &sw, 0, 1, 1, &yv);
            if (rc) return rc;
            y[a * Ns + b] = yv;
            if (acc_out) acc_out[a * Ns + b] = acc;
        }
    }
    if (q_out) memcpy(q_out, scratch_q, (size_t)(Ms * K));
    if (sx_out) memcpy(sx_out, scratch_sx, (size_t)Ms * sizeof(float));
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * SwiGLU of the MLP, [P5-3.2] BitLlamaMLP: the down projection's input is
 * silu(gate(x)) * up(x), silu(z) = z * sigmoid(z) = z / (1 + e^-z). g and u are
 * the bf16 outputs of the gate and up BitLinears. As in the page's module, where
 * each op returns a bf16 tensor, every op rounds its result to bf16:
 *   s = bf16(silu(g))   evaluated in binary64 with libm exp, rounded once to bf16;
 *   h = bf16(s * u)     the product of two bf16 values is exact in binary64.
 * s_out (optional) receives s. All arrays hold bf16 bit patterns.
 * ------------------------------------------------------------------------- */
int oracle_swiglu(const uint16_t* g, const uint16_t* u, int64_t count, uint16_t* s_out,
                  uint16_t* h) {
    if (!g || !u || !h || count < 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < count; ++i) {
        double gv = (double)bf16_to_float(g[i]);
        double silu = gv / (1.0 + exp(-gv));
        uint16_t s;
        oracle_round_bf16(&silu, 1, &s);
        double prod = (double)bf16_to_float(s) * (double)bf16_to_float(u[i]);
        oracle_round_bf16(&prod, 1, &h[i]);
        if (s_out) s_out[i] = s;
    }
    return ORACLE_OK;
}
