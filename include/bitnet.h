/*
 * bitnet.h — C ABI of the B200 (sm_100a) W2A8 BitLinear library (libbitnet.so).
 *
 * The operation is the BitNet b1.58 BitLinear forward:
 *   y[m, n] = (sum_k q[m, k] * t[n, k]) * s_w / s_x[m]
 * with ternary weights t in {-1, 0, +1} and absmean scale s_w (page "BitNet 深度实战：
 * 微软 32K Star 的 1-bit LLM 推理框架", section 2.4 "量化函数的细节" and section 3.2, where
 * BitLinear computes linear(x, t * s_w)), weights stored 2-bit packed as (N, K/4) uint8
 * with four weights per byte (page "BitNet-Triton：消费级GPU上的1.58-bit大模型推理加速方案",
 * section "技术架构：融合内核的三重优化", item 1; bit order from "BitNet 深度实战" section
 * 4.3 "位打包（Bit Packing）存储"), int8 activations quantised per token (BitNet-Triton,
 * items 2 and 3; "BitNet 1-bit LLM推理优化：内存布局、量化策略与硬件加速", section 3.2
 * "激活量化策略"), and an int32 accumulator ("BitNet 深度实战" section 4.4 "查找表加速").
 *
 * Conventions shared by every call:
 *  - Data pointers are DEVICE pointers in the current CUDA context, owned by the
 *    caller. The library keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Every call is asynchronous on that stream and returns once the work is queued.
 *  - Arguments are checked on the host before anything is launched; a call that
 *    returns an error status has launched nothing (except BITNET_ERR_CUDA, which
 *    reports a failed launch).
 *  - Layouts are dense row-major. bf16 values are passed as their uint16 bit
 *    patterns. Base addresses of x, packed, q, y and t must be 16-byte aligned and
 *    `workspace` 256-byte aligned (BITNET_ERR_ALIGN otherwise).
 *  - Shapes: M, N >= 1; K >= 64 and K % 64 == 0 (BITNET_ERR_SHAPE if K % 4 != 0,
 *    BITNET_ERR_UNSUPPORTED for other K); M, N, K < 2^31.
 *  - NaN or Inf in x or W give unspecified (but memory-safe) results.
 *  - Rounding: every float step is IEEE binary32 round-to-nearest-even, with no
 *    contraction into FMA where the order below is stated.
 *  - Thread safety: calls may be made from several host threads. The library holds two
 *    pieces of device state per device: the watchdog word read by
 *    bitnet_check_device_errors(), and the fixed scratch array of bitnet_linear_noalloc
 *    (the only call that uses it). Their device addresses are looked up on first use on
 *    each device and cached, so the library must not be used on a device again after
 *    cudaDeviceReset of that device. Every other call keeps its scratch in the caller's
 *    workspace.
 */
#ifndef BITNET_H
#define BITNET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_NULL = 1,        /* a required pointer is NULL                                   */
    BITNET_ERR_SHAPE = 2,       /* M, N or K out of range, or K not a multiple of 4             */
    BITNET_ERR_ALIGN = 3,       /* a pointer is not aligned as stated above                     */
    BITNET_ERR_UNSUPPORTED = 4, /* valid by the method but not by these kernels (e.g. K % 64)   */
    BITNET_ERR_CUDA = 5,        /* a CUDA launch or query failed                                */
    BITNET_ERR_TIMEOUT = 6,     /* a kernel's bounded wait expired (see bitnet_check_device_errors) */
    BITNET_ERR_WORKSPACE = 7    /* workspace missing or smaller than bitnet_linear_workspace_size() */
} bitnet_status;

typedef enum {
    BITNET_SCALE_PER_TENSOR = 0, /* s_w has 1 element (the BitNet b1.58 layout)                 */
    BITNET_SCALE_PER_ROW = 1     /* s_w has N elements (mean along dim=-1, "BitNet 深度实战" 2.4) */
} bitnet_scale_mode;

typedef enum {
    BITNET_OUT_BF16 = 0, /* y is (M, N) bf16, round-to-nearest-even of the fp32 value */
    BITNET_OUT_F32 = 1   /* y is (M, N) fp32                                          */
} bitnet_out_dtype;

/* Granularity of the activation scale s_x. Per token is the default of every call without
 * an `act` argument; per tensor is one scale for the whole (M, K) input, the setting the I2_S
 * kernel keeps from BitNet b1.58's training ("BitNet 1-bit LLM推理优化" section 2.2; section 3.2
 * lists per-tensor and per-channel scales). A scale per K channel is not offered: it would
 * sit inside the sum over k, so the contraction could no longer run in integers. */
typedef enum {
    BITNET_ACT_PER_TOKEN = 0, /* s_x[m] = 127 / max(max_k |x[m,k]|, 1e-5)                   */
    BITNET_ACT_PER_TENSOR = 1 /* one s = 127 / max(max_{m,k} |x[m,k]|, 1e-5) for every token */
} bitnet_act_mode;

typedef enum {
    BITNET_PATH_AUTO = 0, /* GEMV for M <= BITNET_GEMV_AUTO_M; for M up to                */
                          /* BITNET_GEMV_MAX_M the tensor-core GEMM when the workspace    */
                          /* holds it, else the GEMV; tensor-core GEMM above, and for     */
                          /* rows longer than the GEMV takes (K > 32768 at one token,     */
                          /* bitnet_linear_plan tells). Among the GEMVs, the kernel       */
                          /* measured fastest for the size.                               */
    BITNET_PATH_GEMV = 1, /* force the dp4a GEMV with fused activation quantisation (the  */
                          /* streaming variant at one token from 12 MiB of weights)       */
    BITNET_PATH_TC = 2,   /* force the tcgen05 GEMM (needs the workspace)                 */
    BITNET_PATH_MMA = 3   /* force the warp-level tensor-core GEMV (mma.sync), M <= 8     */
} bitnet_path;

#define BITNET_GEMV_MAX_M 8
#define BITNET_GEMV_AUTO_M 4
#define BITNET_MAX_PROJ 8

/*
 * bitnet_pack_weights — the offline weight step ("BitNet 深度实战" section 2.4, packing
 * per section 4.3): absmean scale, ternarise, pack.
 *   W       [in]  (N, K) fp32 latent weights, device.
 *   mode          BITNET_SCALE_PER_TENSOR or BITNET_SCALE_PER_ROW.
 *   packed  [out] (N, K/4) uint8, device. Byte j of row n holds weights 4j..4j+3, weight
 *                 4j+i in bits 2i..2i+1, code = t + 1 (00 = -1, 01 = 0, 10 = +1; 11 unused).
 *                 Also used as scratch for the per-row sums before it is written.
 *   s_w     [out] fp32, 1 element (per tensor) or N (per row), device.
 * Order of operations (fixed, so results are bit-reproducible): r_n = binary64 sum of
 * |W[n,k]| for k ascending; per row s_n = (float)(r_n / K); per tensor
 * s = (float)((r_0 + r_1 + ... + r_{N-1}) / (N*K)) summed for n ascending; then
 * s = max(s, 1e-5f). t = clamp(rint(W / s), -1, 1) with a binary32 divide, ties to even.
 */
bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, bitnet_scale_mode mode,
                                  uint8_t* packed, float* s_w, void* stream);

/*
 * bitnet_pack_ternary — pack weights that are already ternary (synthetic workloads draw
 * t directly). t is (N, K) int8 with values in {-1, 0, +1} (other values give
 * unspecified codes); packed is (N, K/4) uint8 in the layout above. No scale is made.
 */
bitnet_status bitnet_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                  void* stream);

/*
 * bitnet_quant_act — per-token absmax int8 activation quantiser (BitNet-Triton item 3
 * "融合激活量化"; "BitNet 1-bit LLM推理优化" section 3.2). For each token m:
 *   amax = max_k |x[m,k]|;  s_x[m] = 127 / max(amax, 1e-5)  (binary32 divide);
 *   q[m,k] = clamp(rint(x[m,k] * s_x[m]), -128, 127)          (binary32 multiply).
 *   x   [in]  (M, K) bf16 bits, device.   q [out] (M, K) int8.   s_x [out] (M) fp32.
 * |q| <= 127 always (-128 is unreachable); every non-zero token has max |q| = 127.
 */
bitnet_status bitnet_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s_x,
                               void* stream);

/*
 * bitnet_quant_act_ex — bitnet_quant_act with a choice of scale granularity. With
 * BITNET_ACT_PER_TENSOR all M entries of s_x receive the one scale, and the call needs
 * `workspace` (device, 4-byte aligned) of at least BITNET_QUANT_WORKSPACE_BYTES bytes for the
 * partial maxima of |x|; per token it may be NULL. Two kernels run per tensor: partial maxima
 * of |x|, then the quantiser reducing them.
 */
#define BITNET_QUANT_WORKSPACE_BYTES 4096
bitnet_status bitnet_quant_act_ex(const uint16_t* x, int64_t M, int64_t K, bitnet_act_mode act,
                                  int8_t* q, float* s_x, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * Workspace bytes the tensor-core path of bitnet_linear / bitnet_linear_batch needs for
 * M tokens of width K (quantised activations, per-token scales, the partial maxima of a
 * per-tensor activation scale, and room for split-K partial tiles). The GEMV path uses
 * none: under BITNET_PATH_AUTO, calls with M <= BITNET_GEMV_MAX_M may pass workspace =
 * NULL and then run the GEMV (for 5 <= M <= 8 a sufficient workspace selects the faster
 * tensor-core path instead).
 */
size_t bitnet_linear_workspace_size(int64_t M, int64_t K);

/*
 * bitnet_linear — the BitLinear forward: per-token quantisation of x (as in
 * bitnet_quant_act), unpacking of the 2-bit codes, int8 x ternary contraction with an
 * int32 accumulator, and the dequant epilogue, all on the device.
 *   x        [in]  (M, K) bf16 bits.        packed [in] (N, K/4) uint8 (layout above).
 *   s_w      [in]  fp32, 1 or N elements by `mode`.
 *   y        [out] (M, N) bf16 or fp32 by `out_dtype`.
 *   workspace, workspace_bytes: device scratch of at least bitnet_linear_workspace_size(M, K)
 *            bytes when the tensor-core path runs (M > BITNET_GEMV_AUTO_M); its contents
 *            on entry are ignored, and it must not be shared by calls that may overlap.
 * Kernels, chosen per call (results identical): the dp4a GEMV with the quantiser fused for
 * few tokens (a shared-memory streaming variant at one token and >= 12 MiB of packed weights
 * per call), otherwise the quantiser followed by the tcgen05 GEMM.
 * Epilogue arithmetic: acc = exact int32 sum; r = 1/s_x[m] (binary32, rounded);
 * y = (float)acc * (s_w[n or 0] * r), each product rounded; bf16 is RNE of that fp32
 * value. The result differs from the exact acc * s_w / s_x by at most 3 binary32
 * roundings (relative error < 2^-22), before the bf16 rounding.
 */
bitnet_status bitnet_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                            const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                            bitnet_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                            void* stream);

/* bitnet_linear with an explicit choice of kernel path (testing and benchmarking). */
bitnet_status bitnet_linear_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                               const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                               bitnet_out_dtype out_dtype, void* workspace,
                               size_t workspace_bytes, bitnet_path path, void* stream);

/* One projection of a batch: its own packed weights, scale, width N and output (M, N). */
typedef struct {
    const uint8_t* packed; /* (N, K/4) uint8, device                  */
    const float* s_w;      /* 1 or N fp32, device                      */
    int32_t mode;          /* bitnet_scale_mode                        */
    int32_t reserved;      /* must be 0                                */
    int64_t N;             /* output width of this projection          */
    void* y;               /* (M, N) output, device                    */
} bitnet_proj;

/*
 * bitnet_linear_batch — several projections of one input x, e.g. q/k/v of one hidden
 * state or gate/up of the MLP ("BitNet 深度实战" section 3.2, BitLlamaAttention and
 * BitLlamaMLP). x is quantised once and all projections run in one GEMM/GEMV launch.
 *   projs [in] HOST array of nproj (1..BITNET_MAX_PROJ) descriptors; all share K and M.
 * Results equal nproj separate bitnet_linear calls bit for bit.
 */
bitnet_status bitnet_linear_batch(const uint16_t* x, int64_t M, int64_t K,
                                  const bitnet_proj* projs, int32_t nproj,
                                  bitnet_out_dtype out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* bitnet_linear_batch with an explicit kernel path. */
bitnet_status bitnet_linear_batch_ex(const uint16_t* x, int64_t M, int64_t K,
                                     const bitnet_proj* projs, int32_t nproj,
                                     bitnet_out_dtype out_dtype, void* workspace,
                                     size_t workspace_bytes, bitnet_path path, void* stream);

/*
 * bitnet_linear_batch_act — bitnet_linear_batch_ex with a choice of activation scale
 * granularity (bitnet_act_mode). Per tensor: the quantiser uses one scale for all M tokens
 * (the tensor-core path adds one small kernel for the partial maxima of |x|; the GEMV takes
 * the maximum over its tokens in the same launch), and the epilogue divides by that scale.
 */
bitnet_status bitnet_linear_batch_act(const uint16_t* x, int64_t M, int64_t K,
                                      const bitnet_proj* projs, int32_t nproj,
                                      bitnet_out_dtype out_dtype, bitnet_act_mode act,
                                      void* workspace, size_t workspace_bytes, bitnet_path path,
                                      void* stream);

/*
 * bitnet_linear_i32 — the contraction alone, for bit-exact checks: acc[m, n] =
 * sum_k q[m, k] * t[n, k] in int32 from int8 q (M, K) and packed weights (N, K/4).
 * Runs the same GEMV / tensor-core main loops as bitnet_linear (chosen by `path`).
 */
bitnet_status bitnet_linear_i32(const int8_t* q, int64_t M, int64_t K, const uint8_t* packed,
                                int64_t N, int32_t* acc, void* workspace, size_t workspace_bytes,
                                bitnet_path path, void* stream);

/*
 * Fused MLP gate/up projections with SwiGLU ("BitNet 深度实战" section 3.2, BitLlamaMLP:
 * the down projection's input is silu(gate_proj(x)) * up_proj(x)). Two calls:
 *
 * bitnet_interleave_gate_up — offline layout step, like packing. It writes the gate and
 * up projections of one MLP (each packed (I, K/4) with its scale) as one matrix of 2I rows
 * in blocks of 16: rows 32b .. 32b+15 are gate rows 16b .. 16b+15 and rows 32b+16 ..
 * 32b+31 are up rows 16b .. 16b+15. Per-row scales are interleaved the same way (2I
 * floats); per-tensor scales become {s_gate, s_up} (2 floats). Both projections use `mode`.
 *   I: intermediate width, a multiple of 16.  K: as for packing (a multiple of 64).
 *   packed_gu [out] (2I, K/4) uint8, 16-byte aligned.  s_w_gu [out] 2 or 2I floats.
 *   All pointers device; outputs must not overlap inputs. Asynchronous on `stream`.
 */
bitnet_status bitnet_interleave_gate_up(const uint8_t* packed_gate, const float* s_w_gate,
                                        const uint8_t* packed_up, const float* s_w_up,
                                        bitnet_scale_mode mode, int64_t I, int64_t K,
                                        uint8_t* packed_gu, float* s_w_gu, void* stream);

/*
 * bitnet_linear_swiglu — h = SwiGLU of the gate and up projections of x, with no (M, 2I)
 * intermediate in memory. Per token m and output j:
 *   g = bf16 output of gate row j for x (the arithmetic of bitnet_linear, bit for bit);
 *   u = the same for up row j;
 *   s = bf16(silu(g)), silu evaluated in binary32 with e = expf(-|g|): g / (1 + e) for
 *       g >= 0 and g e / (1 + e) for g < 0 (a fast divide: the divisor lies in [1, 2]);
 *   h = bf16(s * u) (the product of two bf16 values, exact in binary32 above 2^-126).
 *   x [in] (M, K) bf16 bits.  packed_gu, s_w_gu [in] from bitnet_interleave_gate_up.
 *   h [out] (M, I) bf16 bits, 16-byte aligned.
 *   workspace, workspace_bytes, path: as bitnet_linear_ex (the GEMV path for M <=
 *   BITNET_GEMV_AUTO_M under BITNET_PATH_AUTO, needing no workspace).
 * s differs from the exactly rounded silu(g) by at most one bf16 step, and only where the
 * binary32 value falls within a few binary32 steps of a bf16 rounding boundary.
 */
bitnet_status bitnet_linear_swiglu(const uint16_t* x, int64_t M, int64_t K,
                                   const uint8_t* packed_gu, const float* s_w_gu,
                                   bitnet_scale_mode mode, int64_t I, uint16_t* h,
                                   void* workspace, size_t workspace_bytes, bitnet_path path,
                                   void* stream);

/*
 * The SwiGLU -> down projection hand-off (page "BitNet-Triton", section "技术架构：融合内核的
 * 三重优化", item 3 "融合激活量化": the activation quantiser belongs with the producer of its
 * input; "BitNet 深度实战" section 3.2, BitLlamaMLP: down(silu(gate(x)) * up(x))).
 * The down projection quantises h per token, and a token's amax runs over all I outputs of h,
 * which the gate/up kernel computes in different CTAs. So the gate/up epilogue writes, beside
 * h, the maxima of |h| over every block of 16 outputs, and the down projection's quantiser
 * takes each token's amax from those I/16 values instead of reducing the row of h.
 *
 * hmax / xmax layout: (M, K/16) uint16, row-major; entry [m, b] holds the bf16 bit pattern,
 * sign cleared, of max |x[m, 16b .. 16b + 15]|. |x| ordered as an unsigned integer is exact,
 * so the amax, and therefore q, s_x and y, equal the plain per-token path's bit for bit.
 *
 * bitnet_linear_swiglu_hmax — bitnet_linear_swiglu that also writes hmax (M, I/16), 2-byte
 *   aligned. Always runs the tensor-core path (workspace as bitnet_linear_ex for that path;
 *   any M); BITNET_ERR_NULL for a null hmax, other errors as bitnet_linear_swiglu.
 * bitnet_linear_hmax — bitnet_linear on the tensor-core path whose quantiser reads xmax
 *   (M, K/16, 8-byte aligned) for each token's amax. xmax must be the block maxima of this x:
 *   the library does not check them, and other values give other scales.
 * bitnet_quant_act_hmax — bitnet_quant_act with the amax taken from xmax: q (M, K) int8
 *   natural layout, s_x (M) fp32.
 */
bitnet_status bitnet_linear_swiglu_hmax(const uint16_t* x, int64_t M, int64_t K,
                                        const uint8_t* packed_gu, const float* s_w_gu,
                                        bitnet_scale_mode mode, int64_t I, uint16_t* h,
                                        uint16_t* hmax, void* workspace, size_t workspace_bytes,
                                        void* stream);
bitnet_status bitnet_linear_hmax(const uint16_t* x, const uint16_t* xmax, int64_t M, int64_t K,
                                 const uint8_t* packed, const float* s_w, bitnet_scale_mode mode,
                                 int64_t N, void* y, bitnet_out_dtype out_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream);
bitnet_status bitnet_quant_act_hmax(const uint16_t* x, const uint16_t* xmax, int64_t M,
                                    int64_t K, int8_t* q, float* s_x, void* stream);

/*
 * bitnet_linear_noalloc — bitnet_linear for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for callers such as a serving
 * loop in which cudaMalloc could synchronise the device and stall other streams, or a
 * plug-in whose host runtime owns all device memory and forbids allocations of its own.
 * It takes the same arguments as bitnet_linear minus the workspace: the tensor-core path's
 * scratch is a fixed device array of BITNET_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.
 *  - Calls that run the tensor-core path (every M > BITNET_GEMV_AUTO_M, since the array
 *    is always there to serve as the workspace) and whose bitnet_linear_workspace_size(M, K)
 *    exceeds the array are rejected with BITNET_ERR_WORKSPACE before anything is launched.
 *    M <= BITNET_GEMV_AUTO_M runs the GEMV, which needs no scratch.
 *  - The first call on each device looks the array's address up (cudaGetSymbolAddress) and
 *    caches it for the process; make that first call before any stream capture on that
 *    device, and do not use the library on a device after cudaDeviceReset of it.
 *  - All calls share the one array and it keeps the last call's contents (each call writes
 *    or clears every part it reads). Calls that may overlap on the GPU — on different
 *    streams, or from different threads without ordering — race on it and give wrong results.
 *  - It calls no cudaMalloc, cudaFree or allocating library routine.
 * Results equal bitnet_linear's bit for bit (the same kernels on the same inputs).
 */
#define BITNET_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
bitnet_status bitnet_linear_noalloc(const uint16_t* x, int64_t M, int64_t K,
                                    const uint8_t* packed, const float* s_w,
                                    bitnet_scale_mode mode, int64_t N, void* y,
                                    bitnet_out_dtype out_dtype, void* stream);

/*
 * Base-3 weight format, five ternary weights per byte (page "将 BitNet 三元查找表集成到自定义
 * Triton 内核中", step 1: 4-5 ternary values per 8-bit byte; 3^5 = 243 <= 256, so 1.6 bits
 * per weight against 2). Row n is cut into chunks of 80 weights (16 bytes); byte p of chunk c
 * holds weights k = 80c + 16d + p, d = 0..4, as sum_d (t + 1) * 3^d; weights past K count as
 * 0. A row takes bitnet_b3_row_bytes(K) = 16 * ceil(K / 80) bytes.
 *
 * bitnet_pack_ternary_b3 — t (N, K) int8 in {-1, 0, +1} -> packed (N, bitnet_b3_row_bytes(K))
 *   uint8, 16-byte aligned; K as for the other calls (a multiple of 64).
 * bitnet_linear_b3 — bitnet_linear for one token (M = 1; BITNET_ERR_UNSUPPORTED otherwise)
 *   on base-3 weights, K <= 16384: the same quantiser, contraction and epilogue arithmetic,
 *   so its output equals bitnet_linear on the 2-bit packing of the same weights bit for bit.
 *   y (1, N) 16-byte aligned. No workspace. Asynchronous on `stream`.
 */
int64_t bitnet_b3_row_bytes(int64_t K);
bitnet_status bitnet_pack_ternary_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                     void* stream);
bitnet_status bitnet_linear_b3(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_b3,
                               const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                               bitnet_out_dtype out_dtype, void* stream);

/*
 * Tensor-parallel steps ("BitNet：1-bit LLM推理框架技术实战指南", section on the distributed
 * engine: a model split by layer or by tensor across devices). When a projection's K range is
 * split over ranks (rank r holds x[:, k0:k1] and packed[:, k0/4 : k1/4], k0 and k1 multiples
 * of 64), the per-token scale needs the amax of the whole row and the int32 accumulator the
 * sum over all slices. A rank runs: bitnet_act_amax on its slice; an all-reduce (max) of amax
 * over the ranks; bitnet_quant_act_amax with that amax; bitnet_linear_i32 on its slices; an
 * all-reduce (sum) of the int32 accumulators (exact in any order); bitnet_dequant. The result
 * equals bitnet_linear on the whole row bit for bit. A split over N needs none of these: each
 * rank runs bitnet_linear on its rows and the outputs are gathered.
 *
 * bitnet_act_amax — amax[m] = max_k |x[m, k]| (exact; the value a bf16 element has).
 *   x [in] (M, K) bf16 bits, 16-byte aligned.  amax [out] (M) fp32.
 * bitnet_quant_act_amax — bitnet_quant_act with the amax supplied: s_x[m] = 127 /
 *   max(amax[m], 1e-5) (binary32 divide), q = clamp(rint(x * s_x), -128, 127), natural order.
 *   amax must be at least max_k |x[m, k]| of this x (as the all-reduced maximum is), so the
 *   clamp never acts. x, q 16-byte aligned; amax, s_x (M) fp32.
 * bitnet_dequant — the epilogue alone: y[m, n] = RN(RN(acc[m, n]) * RN(s_w[n or 0] *
 *   RN(1 / s_x[m]))) in binary32, bf16 by RNE: the rounding steps of bitnet_linear.
 *   acc (M, N) int32, s_x (M), s_w (1 or N by mode), y (M, N) bf16 or fp32.
 * All asynchronous on `stream`; argument errors as for the other calls (M * K / 8 and M * N
 * below 2^39).
 */
bitnet_status bitnet_act_amax(const uint16_t* x, int64_t M, int64_t K, float* amax, void* stream);
bitnet_status bitnet_quant_act_amax(const uint16_t* x, int64_t M, int64_t K, const float* amax,
                                    int8_t* q, float* s_x, void* stream);
bitnet_status bitnet_dequant(const int32_t* acc, int64_t M, int64_t N, const float* s_x,
                             const float* s_w, bitnet_scale_mode mode, void* y,
                             bitnet_out_dtype out_dtype, void* stream);

/*
 * bitnet_linear_plan — which kernels a call would run, without running anything (a host-only
 * query for tests and tuning; the pages have no counterpart). It reports the choices
 * bitnet_linear_batch_ex makes for nproj projections of widths Ns[0 .. nproj) at M tokens of
 * width K with a 256-byte aligned workspace of workspace_bytes (0 = no workspace) on path
 * `path`, or, with swiglu = 1 (nproj = 1, Ns[0] = 2I), those of bitnet_linear_swiglu. It
 * reads the current device's SM count (148 when no device can be queried). Argument errors
 * are those of the call it describes.
 */
#define BITNET_KERNEL_GEMV 1   /* dp4a GEMV with the quantiser fused, up to 8 tokens          */
#define BITNET_KERNEL_MMA_GEMV 2 /* warp-level tensor-core GEMV (mma.sync), up to 8 tokens  */
#define BITNET_KERNEL_STREAM 3 /* one-token streaming GEMV through a shared-memory ring      */
#define BITNET_KERNEL_TC 4     /* quantiser kernel, then the tcgen05 tensor-core GEMM         */
#define BITNET_KERNEL_GS 5     /* one-token grid-stride GEMV for large matrices               */
typedef struct {
    int32_t kernel;        /* BITNET_KERNEL_*                                               */
    int32_t grid;          /* CTAs of the main kernel                                       */
    int32_t tile_tokens;   /* tensor-core path: tokens per tile (16 .. 192), else 0         */
    int32_t splits;        /* tensor-core path: K splits per tile (1 = none), else 0        */
    int32_t tile_rows;     /* GEMV and warp-MMA GEMV: weight rows per CTA, else 0            */
    int32_t reserved[3];
} bitnet_plan;
bitnet_status bitnet_linear_plan(int64_t M, int64_t K, const int64_t* Ns, int32_t nproj,
                                 int32_t swiglu, size_t workspace_bytes, bitnet_path path,
                                 bitnet_plan* plan);

/*
 * bitnet_check_device_errors — synchronises the current device, returns the library's
 * watchdog word in *flags (0 = no kernel gave up a bounded wait since the last check)
 * and clears it. Returns BITNET_ERR_TIMEOUT when the word was non-zero. The word is an OR
 * of the BITNET_WATCHDOG_* bits of the waits that expired.
 */
#define BITNET_WATCHDOG_TMA_FULL (1 << 0)   /* a stage's TMA load never completed */
#define BITNET_WATCHDOG_UNPACK (1 << 1)     /* unpacked weights never arrived */
#define BITNET_WATCHDOG_EMPTY (1 << 2)      /* a ring slot was never released */
#define BITNET_WATCHDOG_ACCUM (1 << 3)      /* an accumulator handoff never happened */
#define BITNET_WATCHDOG_DRAIN (1 << 4)      /* copies or MMAs in flight at exit never completed */
#define BITNET_WATCHDOG_SELFTEST (1 << 6)   /* bitnet_selftest_wait_timeout's wait */
bitnet_status bitnet_check_device_errors(int32_t* flags);

/*
 * bitnet_selftest_wait_timeout — test hook for the failure detection, not on the hot path
 * (the pages have no counterpart). Launches one thread that waits on an mbarrier nothing
 * completes, through the same bounded wait every tensor-core kernel wait uses, with a limit
 * of limit_ns nanoseconds of %globaltimer. On expiry the kernel ORs
 * BITNET_WATCHDOG_SELFTEST into the watchdog word and returns (no trap, the context stays
 * usable), so a following bitnet_check_device_errors returns BITNET_ERR_TIMEOUT.
 * limit_ns must lie in [1e6, 2e9] (BITNET_ERR_UNSUPPORTED otherwise). Asynchronous on
 * `stream`.
 */
bitnet_status bitnet_selftest_wait_timeout(int64_t limit_ns, void* stream);

/*
 * Arithmetic rate probes for the roofline of the one-token GEMV (diagnostics; the pages have
 * no counterpart). bitnet_probe_int_rate launches `blocks` CTAs of 256 threads that issue only
 * dp4a (BITNET_PROBE_DP4A: eight independent chains per thread) or only warp-level
 * mma.sync m16n8k32 s8 x s8 -> s32 (BITNET_PROBE_MMA_S8: four independent accumulator tiles
 * per warp), `iters` rounds each; out receives one int32 per CTA (blocks elements, device).
 * Asynchronous on `stream`: the caller times the launch (CUDA events) and divides
 * bitnet_probe_int_ops(kind, blocks, iters) integer operations (2 per multiply-add) by it.
 * Errors: BITNET_ERR_UNSUPPORTED for another kind, BITNET_ERR_SHAPE for blocks outside
 * [1, 65535] or iters outside [1, 2^24], BITNET_ERR_NULL for a null out.
 */
#define BITNET_PROBE_DP4A 0
#define BITNET_PROBE_MMA_S8 1
bitnet_status bitnet_probe_int_rate(int32_t kind, int32_t blocks, int64_t iters, int32_t* out,
                                    void* stream);
int64_t bitnet_probe_int_ops(int32_t kind, int32_t blocks, int64_t iters);

/* Human-readable name of a status code (static storage). */
const char* bitnet_status_string(bitnet_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t bitnet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_H */
