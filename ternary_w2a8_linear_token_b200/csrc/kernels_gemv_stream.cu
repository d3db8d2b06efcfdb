// Streaming decode GEMV for one token and large weight matrices: the same product as
// gemv_w2a8_kernel (page "BitNet-Triton", section "技术架构：融合内核的三重优化", items 1 and 3:
// 2-bit weights unpacked in the kernel, activation quantiser fused; page "BitNet 1-bit LLM推理
// 优化", section 4.2: packed decode to 8-bit and dp4a dot products), laid out for matrices too
// large for one wave of the register-resident kernel (the layer-wide batched projections of
// the 2B-4T and 8B-class models at M = 1).
//
// At M = 1 the product reads each packed weight byte once and does four multiply-adds with
// it, so it runs at the rate bytes arrive from HBM. That rate is set by the bytes each SM
// keeps in flight; registers cannot hold enough of them, so here a producer warp keeps a
// shared-memory ring of weight stages filled with bulk async copies (no multicast), while
// sixteen consumer warps take one weight row (or one SwiGLU gate/up pair) each per stage:
//  - one CTA per SM, persistent over stages s = blockIdx.x, blockIdx.x + gridDim.x, ...;
//    a stage is 16 * UPW consecutive rows of one projection (16 * UPW output pairs, 32 * UPW
//    interleaved rows, for SwiGLU), one contiguous span of the (N, K/4) packed matrix, and
//    each consumer warp takes UPW of its units: at one token the consumers' instruction
//    stream bounds the kernel (8 instructions per 16 weights: the codes are masked in place,
//    see code_dot_acc, and issued at about one instruction every other cycle per scheduler),
//    so the per-stage bookkeeping is spread over several rows, which are summed as
//    independent chains;
//  - full/empty mbarriers per ring slot, every wait bounded (the library's watchdog);
//  - the consumers quantise x once per CTA into shared memory in the permuted in-group
//    order (see kernels_quant.cu) and keep their lanes' share of q in registers (K <= 4096)
//    or read it from shared memory, so the per-stage shared-memory traffic is the weights.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "act_quant_device.cuh"
#include "bitnet_device.cuh"
#include "bitnet_internal.h"
#include "swiglu_device.cuh"

namespace bitnet {
namespace {

constexpr float kEps = kActEps;
constexpr int kConsumers = 16;                     // consumer warps, one unit per stage each
constexpr int kStreamThreads = (kConsumers + 1) * 32;  // warp 0 produces
constexpr int kConsumerThreads = kConsumers * 32;
constexpr int kMaxPiecesPerThread = 4;             // K <= 4 * 512 * 8 = 16384
constexpr int kMaxDepth = 8;
constexpr int kRingMax = 180 * 1024;

// Barrier among the 16 consumer warps (named barrier 1); the producer never joins it.
__device__ __forceinline__ void consumer_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}

struct Stage {
    int proj;
    int64_t row0;   // first packed row of the stage within its projection
    int rows;       // packed rows in the stage (fewer than the full stage at a ragged end)
};

// Stage s of the whole problem: projections are cut into stages of 16 * upw rows in order;
// SwiGLU (one interleaved projection of 2I rows) into stages of 32 * upw rows.
__device__ __forceinline__ Stage stage_of(const GemvParams& p, int64_t s, int upw) {
    Stage st;
    if (p.swiglu) {
        const int64_t rows = int64_t(2 * kSwigluBlock) * upw;
        st.proj = 0;
        st.row0 = s * rows;
        const int64_t left = 2 * p.total_rows - st.row0;  // total_rows counts output pairs
        st.rows = static_cast<int>(left < rows ? left : rows);
        return st;
    }
    const int64_t rows = int64_t(kConsumers) * upw;
    int64_t first = 0;
    st.proj = 0;
    for (int j = 0; j < p.nproj; ++j) {
        const int64_t n_st = (p.proj[j].N + rows - 1) / rows;
        if (s < first + n_st) {
            st.proj = j;
            break;
        }
        first += n_st;
    }
    st.row0 = (s - first) * rows;
    const int64_t left = p.proj[st.proj].N - st.row0;
    st.rows = static_cast<int>(left < rows ? left : rows);
    return st;
}

// CPL: 16-byte chunks per lane (K <= CPL * 2048). QREG: keep this lane's q in registers.
// UPW: units (rows, or SwiGLU pairs) per consumer warp per stage.
template <int CPL, bool QREG, int UPW>
__global__ void __launch_bounds__(kStreamThreads, 1)
    gemv_stream_kernel(const __grid_constant__ GemvParams p, int64_t n_stages, int depth,
                       uint32_t stage_bytes, int32_t* err) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* ring = smem;                                               // depth x stage_bytes
    uint4* s_q = reinterpret_cast<uint4*>(smem + int64_t(depth) * stage_bytes);  // K bytes
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s_q) + p.K);
    uint64_t* empty = full + kMaxDepth;
    __shared__ uint32_t s_red[kConsumers];
    __shared__ int32_t s_qsum[kConsumers];
    __shared__ int32_t s_abort;
    volatile int32_t* abort_flag = &s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t K = p.K;
    const int C = static_cast<int>(K >> 6);  // 16-byte chunks per packed row
    const int64_t row_bytes = K >> 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < depth; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers);
        }
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();

    if (warp == 0) {
        // ---------------- producer: weight stages never depend on earlier grids, so they
        // stream from the start, ahead of the wait on the previous grid.
        if (lane == 0) {
            int i = 0;
            for (int64_t s = blockIdx.x; s < n_stages; s += gridDim.x, ++i) {
                const int slot = i % depth;
                const uint32_t phase = uint32_t(i / depth) & 1u;
                if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, err, kErrWaitEmpty, abort_flag))
                    break;
                const Stage st = stage_of(p, s, UPW);
                const uint32_t bytes = uint32_t(st.rows * row_bytes);
                mbar_arrive_expect_tx(&full[slot], bytes);
                bulk_load_1d(ring + int64_t(slot) * stage_bytes,
                             p.proj[st.proj].packed + st.row0 * row_bytes, bytes, &full[slot]);
            }
            // Every issued copy lands before the CTA may exit (also after an abort).
            for (int k = i > depth ? i - depth : 0; k < i; ++k)
                mbar_wait_bounded(&full[k % depth], uint32_t(k / depth) & 1u, err, kErrWaitDrain,
                                  nullptr);
        }
        return;
    }

    // ---------------- consumers
    const int cw = warp - 1;
    const int ct = threadIdx.x - 32;
    pdl_wait();

    // Quantise the token once: absmax, one consumer barrier, permuted q to shared memory.
    const int64_t pieces = K >> 3;
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x);
    uint4 xv[kMaxPiecesPerThread];
    uint32_t mx = 0;
#pragma unroll
    for (int t = 0; t < kMaxPiecesPerThread; ++t) {
        const int64_t c = ct + int64_t(t) * kConsumerThreads;
        xv[t] = c < pieces ? x4[c] : make_uint4(0u, 0u, 0u, 0u);
        mx = max(mx, absmax8_bits(xv[t]));
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) s_red[cw] = mx;
    consumer_bar();
    uint32_t all = s_red[0];
#pragma unroll
    for (int w = 1; w < kConsumers; ++w) all = max(all, s_red[w]);
    const float s_tok = __fdiv_rn(127.0f, fmaxf(__uint_as_float(all << 16), kEps));
    uint8_t* sq_bytes = reinterpret_cast<uint8_t*>(s_q);
    int qs = 0;
#pragma unroll
    for (int t = 0; t < kMaxPiecesPerThread; ++t) {
        const int64_t c = ct + int64_t(t) * kConsumerThreads;  // lane pairs share a 16-group
        uint2 nat;
        nat.x = pack4(qbits(bf16_lo(xv[t].x), s_tok), qbits(bf16_hi(xv[t].x), s_tok),
                      qbits(bf16_lo(xv[t].y), s_tok), qbits(bf16_hi(xv[t].y), s_tok));
        nat.y = pack4(qbits(bf16_lo(xv[t].z), s_tok), qbits(bf16_hi(xv[t].z), s_tok),
                      qbits(bf16_lo(xv[t].w), s_tok), qbits(bf16_hi(xv[t].w), s_tok));
        qs += bytesum(nat.x) + bytesum(nat.y);  // padding pieces quantise to 0
        const uint2 out = permute_group_half(nat, lane & 1);
        if (c < pieces) {
            const int64_t g = c >> 1;  // group g = c / 2 lives in chunk g / 4, slot g % 4
            const int64_t idx16 = (g & 3) * C + (g >> 2);
            *reinterpret_cast<uint2*>(sq_bytes + idx16 * 16 + (c & 1) * 8) = out;
        }
    }
    qs = __reduce_add_sync(0xFFFFFFFFu, qs);
    if (lane == 0) s_qsum[cw] = qs;
    consumer_bar();
    int32_t qs_tot = 0;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) qs_tot += s_qsum[w];
    const float rx = __frcp_rn(s_tok);

    uint4 qreg[QREG ? CPL : 1][4];
    if constexpr (QREG) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int chunk = lane + 32 * c;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                qreg[c][j] = chunk < C ? s_q[j * C + chunk] : make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // Sum over this lane's chunks of one packed row in shared memory: sum_k q * code.
    auto row_dot = [&](const uint8_t* row) -> int32_t {
        int4 acc = make_int4(0, 0, 0, 0);  // four independent dp4a chains
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int chunk = lane + 32 * c;
            if (chunk < C) {
                const uint4 wv = *reinterpret_cast<const uint4*>(row + int64_t(chunk) * 16);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t word = j == 0 ? wv.x : j == 1 ? wv.y : j == 2 ? wv.z : wv.w;
                    const uint4 qv = QREG ? qreg[QREG ? c : 0][j] : s_q[j * C + chunk];
                    code_dot_acc(word, qv, acc);
                }
            }
        }
        return code_dot_total(acc);
    };

    int i = 0;
    for (int64_t s = blockIdx.x; s < n_stages; s += gridDim.x, ++i) {
        const int slot = i % depth;
        const uint32_t phase = uint32_t(i / depth) & 1u;
        const bool ok = mbar_wait_bounded(&full[slot], phase, err, kErrWaitTmaFull, abort_flag);
        const Stage st = stage_of(p, s, UPW);
        const GemvProj& pr = p.proj[st.proj];
        const uint8_t* base = ring + int64_t(slot) * stage_bytes;
        // This warp's units: non-SwiGLU row cw + 16 u of the stage; SwiGLU pair cw of the
        // stage's 32-row block u (gate row 32 u + cw, up row 32 u + 16 + cw). The scales are
        // loaded first, so their latency hides behind the dot products.
        float sa[UPW], sb[UPW];
        bool valid[UPW];
#pragma unroll
        for (int u = 0; u < UPW; ++u) {
            const int lr = p.swiglu ? 2 * kSwigluBlock * u + cw : kConsumers * u + cw;
            valid[u] = lr < st.rows;
            sa[u] = sb[u] = 0.0f;
            if (lane == 0 && valid[u] && p.out_kind != 2) {
                const int64_t r = st.row0 + lr;
                sa[u] = pr.per_row ? pr.s_w[r] : pr.s_w[0];
                if (p.swiglu) sb[u] = pr.per_row ? pr.s_w[r + kSwigluBlock] : pr.s_w[1];
            }
        }
        // All of this warp's row sums first, as independent chains (the dp4a chains of one
        // row alone leave most issue slots idle), then the warp reductions. A unit past the
        // end of a short last stage reads stale bytes of its slot and is discarded.
        int32_t part[UPW], part2[UPW];
#pragma unroll
        for (int u = 0; u < UPW; ++u) {
            const int lr = p.swiglu ? 2 * kSwigluBlock * u + cw : kConsumers * u + cw;
            part[u] = row_dot(base + lr * row_bytes);
            part2[u] = p.swiglu ? row_dot(base + (lr + kSwigluBlock) * row_bytes) : 0;
        }
        int32_t tot[UPW], tot2[UPW];
#pragma unroll
        for (int u = 0; u < UPW; ++u) {
            tot[u] = __reduce_add_sync(0xFFFFFFFFu, part[u]) - qs_tot;
            tot2[u] = p.swiglu ? __reduce_add_sync(0xFFFFFFFFu, part2[u]) - qs_tot : 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done reading the slot
        if (!ok) break;
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < UPW; ++u) {
                if (!valid[u]) continue;
                if (p.swiglu) {
                    const float g = __fmul_rn(__int2float_rn(tot[u]), __fmul_rn(sa[u], rx));
                    const float uu = __fmul_rn(__int2float_rn(tot2[u]), __fmul_rn(sb[u], rx));
                    const int64_t j = (st.row0 >> 1) + kSwigluBlock * u + cw;  // output pair
                    static_cast<uint16_t*>(pr.y)[j] = swiglu_bf16_bits(g, uu);
                } else {
                    const int64_t n = st.row0 + kConsumers * u + cw;
                    if (p.out_kind == 2) {
                        static_cast<int32_t*>(pr.y)[n] = tot[u];
                    } else {
                        const float yv = __fmul_rn(__int2float_rn(tot[u]), __fmul_rn(sa[u], rx));
                        if (p.out_kind == 0)
                            static_cast<__nv_bfloat16*>(pr.y)[n] = __float2bfloat16_rn(yv);
                        else
                            static_cast<float*>(pr.y)[n] = yv;
                    }
                }
            }
        }
    }
}

template <int CPL, int UPW>
cudaError_t launch_stream_cpl(const GemvParams& p, int64_t n_stages, int depth,
                              uint32_t stage_bytes, int sms, int32_t* err, cudaStream_t stream,
                              bool pdl) {
    constexpr bool kQreg = CPL <= 2;
    auto kern = gemv_stream_kernel<CPL, kQreg, UPW>;
    const size_t smem = size_t(depth) * stage_bytes + size_t(p.K) + 2 * kMaxDepth * 8;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_stages < sms ? n_stages : sms));
    cfg.blockDim = dim3(kStreamThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p, n_stages, depth, stage_bytes, err);
}

template <int UPW>
cudaError_t launch_stream_upw(const GemvParams& p, int64_t n_stages, int depth,
                              uint32_t stage_bytes, int sms, int32_t* err, cudaStream_t stream,
                              bool pdl) {
    const int cpl = static_cast<int>(((p.K >> 6) + 31) / 32);
    if (cpl <= 1)
        return launch_stream_cpl<1, UPW>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
    if (cpl <= 2)
        return launch_stream_cpl<2, UPW>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
    if (cpl <= 4)
        return launch_stream_cpl<4, UPW>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
    return launch_stream_cpl<8, UPW>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
}

// Units per warp per stage: the most (4, 2, 1) whose stage is at most kStageMax bytes and
// leaves a ring of at least two stages.
constexpr int64_t kStageMax = 64 * 1024;

int stream_upw(const GemvParams& p) {
    const int64_t unit_bytes = (p.swiglu ? 2 : 1) * int64_t(kConsumers) * (p.K / 4);
    for (int upw : {4, 2, 1})
        if (unit_bytes * upw <= kStageMax && kRingMax / (unit_bytes * upw) >= 2) return upw;
    return 0;
}

}  // namespace

bool gemv_stream_plan(const GemvParams& p, int64_t* n_stages, int* depth, uint32_t* stage_bytes) {
    if (p.M != 1 || p.q_in != nullptr || p.K > int64_t(kMaxPiecesPerThread) * kConsumerThreads * 8)
        return false;
    const int upw = stream_upw(p);
    if (upw == 0) return false;
    const int64_t sb = (p.swiglu ? 2 : 1) * int64_t(kConsumers) * upw * (p.K / 4);
    const int64_t d = kRingMax / sb < kMaxDepth ? kRingMax / sb : kMaxDepth;
    int64_t ns = 0;
    if (p.swiglu) {
        const int64_t pairs = int64_t(kConsumers) * upw;  // total_rows counts output pairs
        ns = (p.total_rows + pairs - 1) / pairs;
    } else {
        const int64_t rows = int64_t(kConsumers) * upw;
        for (int j = 0; j < p.nproj; ++j) ns += (p.proj[j].N + rows - 1) / rows;
    }
    *n_stages = ns;
    *depth = static_cast<int>(d);
    *stage_bytes = static_cast<uint32_t>(sb);
    return true;
}

cudaError_t launch_gemv_stream(const GemvParams& p, int64_t n_stages, int depth,
                               uint32_t stage_bytes, int sms, int32_t* err, cudaStream_t stream,
                               bool pdl) {
    const int upw = stream_upw(p);
    if (upw == 4) return launch_stream_upw<4>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
    if (upw == 2) return launch_stream_upw<2>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
    return launch_stream_upw<1>(p, n_stages, depth, stage_bytes, sms, err, stream, pdl);
}

}  // namespace bitnet
