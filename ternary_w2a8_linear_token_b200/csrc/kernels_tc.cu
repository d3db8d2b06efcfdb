// Tensor-core W2A8 GEMM for sm_100a (tcgen05 + TMA + TMEM).
//
// The contraction acc[m, n] = sum_k q[m, k] t[n, k] ("BitNet 深度实战", section 4.4
// "查找表加速": int8 activations, ternary weights, int32 accumulation) runs as an int8
// tensor-core product, since ternary weights are just int8 values in {-1, 0, +1}
// (page "BitNet-Triton", section "技术架构：融合内核的三重优化", item 2 "INT8张量核心加速").
//
// Operand roles are swapped so that the weight rows fill the 128-row MMA dimension and
// the tokens are the MMA N dimension (16 ... 256): D[n, m] in TMEM = T[n, :] . Q[m, :].
// That keeps small token counts efficient and re-unpacks each weight tile once per
// token tile of up to 256 tokens.
//
// Per CTA: one 128 x BN output tile (weight rows x tokens), K streamed in 128-byte stages.
//  warp 0      TMEM allocation; lane 0 issues TMA loads of the packed weight tile
//              (128 rows x 32 bytes) and the quantised token tile (BN rows x 128 bytes,
//              128-byte swizzle) for each stage;
//  warp 1      lane 0 issues 4 tcgen05.mma.kind::i8 (K = 32 each) per stage and commits
//              them to the stage's "empty" barrier;
//  warps 2-9   unpack each packed stage into the int8 A tile in shared memory (128-byte
//              swizzled K-major, codes - 1 per byte), then run the epilogue: TMEM -> regs,
//              y = acc * (s_w * 1/s_x), store.
// The activation tile arrives already in the permuted in-group K order produced by the
// quantiser, which is the order a packed word unpacks into with shifts and masks alone.
//
// Every mbarrier wait is bounded (bitnet_device.cuh): on expiry the kernel records a
// watchdog code and runs on to its end, so it always returns and frees its TMEM.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"

namespace bitnet {
namespace {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 128;          // K bytes per stage
constexpr int kUnpackWarps = 8;
constexpr int kThreads = 64 + kUnpackWarps * 32;  // 320

template <int BN>
struct TcLayout {
    static constexpr int kA = kBM * kBK;        // unpacked weights, 16 KB
    static constexpr int kB = BN * kBK;         // token tile
    static constexpr int kP = kBM * kBK / 4;    // packed weights, 4 KB
    static constexpr int kStage = kA + kB + kP;  // multiple of 1024
    static constexpr int kStages = (200 * 1024) / kStage > 6 ? 6 : (200 * 1024) / kStage;
    static constexpr int kBarOff = kStages * kStage;
    static constexpr int kBarBytes = (3 * kStages + 1) * 8 + 16;  // + TMEM slot, abort flag
    static constexpr int kRxOff = kBarOff + kBarBytes;             // BN floats: 1/s_x of the tile
    static constexpr int kSmem = kRxOff + BN * 4 + 1024;           // + alignment slack
    static_assert(BN * kBM * 4 <= kStages * kStage, "output staging must fit the stage area");
    static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
    static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kStages >= 2, "need at least two stages");
};

// Barrier among the 8 unpack/epilogue warps only (named barrier 1).
__device__ __forceinline__ void epilogue_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kUnpackWarps * 32) : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]) {
    static_assert(N % 8 == 0, "columns in multiples of 8");
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        uint32_t (&r)[8] = *reinterpret_cast<uint32_t(*)[8]>(&v[8 * i]);
        tmem_ld_32x32b_x8(taddr + uint32_t(8 * i), r);
    }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
    using L = TcLayout<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* full_unp = full_tma + L::kStages;
    uint64_t* empty = full_unp + L::kStages;
    uint64_t* acc_full = empty + L::kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // tile -> (projection, weight-row block, token block)
    int j = 0;
#pragma unroll
    for (int jj = 1; jj < kMaxProj; ++jj)
        if (jj < p.nproj && int(blockIdx.x) >= p.proj[jj].tile_begin) j = jj;
    const int n0 = (int(blockIdx.x) - p.proj[j].tile_begin) * kBM;
    const int m0 = int(blockIdx.y) * BN;
    const int num_k = static_cast<int>((p.K + kBK - 1) / kBK);

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < L::kStages; ++s) {
                mbar_init(&full_tma[s], 1);
                mbar_init(&full_unp[s], kUnpackWarps);
                mbar_init(&empty[s], 1);
            }
            mbar_init(acc_full, 1);
            *abort_flag = 0;
            fence_mbar_init();
            tma_prefetch_desc(&p.tmap_w[j]);
            tma_prefetch_desc(&p.tmap_q);
        }
        __syncwarp();
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            pdl_wait();  // the token tile is written by the quantiser grid
            for (int kt = 0; kt < num_k; ++kt) {
                const int s = kt % L::kStages;
                const uint32_t ph = (kt / L::kStages) & 1;
                mbar_wait_bounded(&empty[s], ph ^ 1, p.err, kErrWaitEmpty, abort_flag);
                uint8_t* st = smem + s * L::kStage;
                mbar_arrive_expect_tx(&full_tma[s], L::kB + L::kP);
                tma_load_2d(st + L::kA + L::kB, &p.tmap_w[j], &full_tma[s], kt * (kBK / 4), n0);
                tma_load_2d(st + L::kA, &p.tmap_q, &full_tma[s], kt * kBK, m0);
            }
            // Drain: every issued stage must have landed before the CTA may exit.
            for (int kt = num_k > L::kStages ? num_k - L::kStages : 0; kt < num_k; ++kt) {
                mbar_wait_bounded(&full_tma[kt % L::kStages], (kt / L::kStages) & 1, p.err,
                                  kErrWaitDrain, nullptr);
            }
        }
        __syncwarp();  // lanes 1-31 wait for the producer lane: the CTA barrier below is aligned
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            for (int kt = 0; kt < num_k; ++kt) {
                const int s = kt % L::kStages;
                const uint32_t ph = (kt / L::kStages) & 1;
                mbar_wait_bounded(&full_tma[s], ph, p.err, kErrWaitTmaFull, abort_flag);
                mbar_wait_bounded(&full_unp[s], ph, p.err, kErrWaitUnpack, abort_flag);
                tc_fence_after();
                const uint32_t a_base = smem_addr(smem + s * L::kStage);
                const uint32_t b_base = a_base + L::kA;
#pragma unroll
                for (int kk = 0; kk < kBK / 32; ++kk) {
                    const uint64_t ad = smem_desc_k_sw128(a_base + kk * 32);
                    const uint64_t bd = smem_desc_k_sw128(b_base + kk * 32);
                    mma_i8(tmem_d, ad, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(acc_full);
            // Drain: no tensor-core operation may still be running when TMEM is freed.
            mbar_wait_bounded(acc_full, 0, p.err, kErrWaitDrain, nullptr);
        }
        __syncwarp();  // reconverge before the aligned CTA barrier below
    } else {
        // ---------------- unpack warps
        const int ut = threadIdx.x - 64;  // 0 .. 255
        const int row = ut >> 1;         // weight row of the tile
        const int half = ut & 1;         // which 16 packed bytes (64 weights) of the stage
        for (int kt = 0; kt < num_k; ++kt) {
            const int s = kt % L::kStages;
            const uint32_t ph = (kt / L::kStages) & 1;
            mbar_wait_bounded(&full_tma[s], ph, p.err, kErrWaitTmaFull, abort_flag);
            uint8_t* st = smem + s * L::kStage;
            const uint4 pk = *reinterpret_cast<const uint4*>(st + L::kA + L::kB + row * 32 +
                                                             half * 16);
            const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
            uint8_t* arow = st + row * kBK;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t wv = words[c];
                uint4 t;
                t.x = codes_to_ternary_s8x4(wv & 0x03030303u);
                t.y = codes_to_ternary_s8x4((wv >> 2) & 0x03030303u);
                t.z = codes_to_ternary_s8x4((wv >> 4) & 0x03030303u);
                t.w = codes_to_ternary_s8x4((wv >> 6) & 0x03030303u);
                const int chunk = half * 4 + c;  // 16-byte chunk of the 128-byte row
                *reinterpret_cast<uint4*>(arow + ((chunk ^ (row & 7)) << 4)) = t;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_unp[s]);
        }

        // ---------------- epilogue
        // 1/s_x of the tile's tokens -> shared memory while the last MMAs run.
        pdl_wait();  // r_x comes from the quantiser grid; y may be read by earlier grids
        const int et = threadIdx.x - 64;  // 0 .. 255
        float* s_rx = reinterpret_cast<float*>(smem + L::kRxOff);
        for (int i = et; i < BN; i += kUnpackWarps * 32) {
            const int64_t m = int64_t(m0) + i;
            s_rx[i] = (p.out_kind != 2 && m < p.M) ? p.r_x[m] : 0.0f;
        }
        epilogue_bar_sync();
        mbar_wait_bounded(acc_full, 0, p.err, kErrWaitAccum, abort_flag);
        tc_fence_after();

        // TMEM (lane = weight row, column = token) -> registers -> dequantised values staged in
        // the idle stage area as rows of the output: stage[token][weight row].
        const int quarter = warp & 3;         // TMEM lanes 32*quarter ... +31
        const int colhalf = (warp - 2) >> 2;  // which half of the BN columns
        const int n_local = quarter * 32 + lane;
        const TcProj& pr = p.proj[j];
        const int64_t n = int64_t(n0) + n_local;
        const bool nvalid = n < pr.N;
        // s_w is absent (nullptr) when the raw int32 accumulator is the output.
        const float sw = p.out_kind == 2 ? 0.0f
                         : pr.per_row   ? (nvalid ? pr.s_w[n] : 0.0f)
                                        : pr.s_w[0];
        const int esz = p.out_kind == 0 ? 2 : 4;
        uint8_t* stage = smem;
        constexpr int kHalfCols = BN / 2;
        constexpr int kLd = kHalfCols >= 32 ? 32 : kHalfCols;  // columns per TMEM load
#pragma unroll 1
        for (int cc = 0; cc < kHalfCols; cc += kLd) {
            const int col0 = colhalf * kHalfCols + cc;
            uint32_t v[kLd];
            tmem_ld_cols<kLd>(tmem_d + (uint32_t(quarter * 32) << 16) + uint32_t(col0), v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < kLd; ++i) {
                const int col = col0 + i;
                const int32_t a = static_cast<int32_t>(v[i]);
                uint8_t* dst = stage + (size_t(col) * kBM + n_local) * esz;
                if (p.out_kind == 2) {
                    *reinterpret_cast<int32_t*>(dst) = a;
                } else {
                    const float yv = __fmul_rn(__int2float_rn(a), __fmul_rn(sw, s_rx[col]));
                    if (p.out_kind == 0)
                        *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(yv);
                    else
                        *reinterpret_cast<float*>(dst) = yv;
                }
            }
        }
        epilogue_bar_sync();

        // Coalesced copy-out: each token row of the tile is 128 contiguous outputs.
        const int row_bytes = kBM * esz;
        const int chunks_per_row = row_bytes / 16;
        const int vals_per_chunk = 16 / esz;
        const bool vec_ok = ((pr.N * esz) % 16) == 0;  // every row start 16-byte aligned
        uint8_t* ybase = static_cast<uint8_t*>(pr.y);
        for (int c = et; c < BN * chunks_per_row; c += kUnpackWarps * 32) {
            const int row = c / chunks_per_row;
            const int ch = c - row * chunks_per_row;
            const int64_t m = int64_t(m0) + row;
            if (m >= p.M) continue;
            const int64_t nn = int64_t(n0) + int64_t(ch) * vals_per_chunk;
            const uint8_t* src = stage + size_t(row) * row_bytes + size_t(ch) * 16;
            uint8_t* dst = ybase + (m * pr.N + nn) * esz;
            if (vec_ok && nn + vals_per_chunk <= pr.N) {
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
            } else {
                for (int e = 0; e < vals_per_chunk; ++e) {
                    if (nn + e >= pr.N) break;
                    if (esz == 2)
                        reinterpret_cast<uint16_t*>(dst)[e] = reinterpret_cast<const uint16_t*>(src)[e];
                    else
                        reinterpret_cast<uint32_t*>(dst)[e] = reinterpret_cast<const uint32_t*>(src)[e];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tmem_dealloc(tmem_d, L::kTmemCols);
    }
}

template <int BN>
cudaError_t launch_bn(const TcParams& p, cudaStream_t stream, bool pdl) {
    using L = TcLayout<BN>;
    auto kern = tc_gemm_kernel<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.n_tiles_total),
                       static_cast<unsigned>((p.M + BN - 1) / BN));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int tc_pick_bn(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

cudaError_t launch_tc_gemm(const TcParams& p, int bn, cudaStream_t stream, bool pdl) {
    switch (bn) {
        case 16: return launch_bn<16>(p, stream, pdl);
        case 32: return launch_bn<32>(p, stream, pdl);
        case 64: return launch_bn<64>(p, stream, pdl);
        case 128: return launch_bn<128>(p, stream, pdl);
        default: return launch_bn<256>(p, stream, pdl);
    }
}

}  // namespace bitnet
