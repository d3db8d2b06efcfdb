// Tensor-core W2A8 GEMM for sm_100a (tcgen05 + TMA + TMEM), persistent.
//
// The contraction acc[m, n] = sum_k q[m, k] t[n, k] ("BitNet 深度实战", section 4.4
// "查找表加速": int8 activations, ternary weights, int32 accumulation) runs as an int8
// tensor-core product, since ternary weights are just int8 values in {-1, 0, +1}
// (page "BitNet-Triton", section "技术架构：融合内核的三重优化", item 2 "INT8张量核心加速").
//
// Operand roles are swapped so that the weight rows fill the 128-row MMA dimension and
// the tokens are the MMA N dimension (16 ... 192): D[n, m] in TMEM = T[n, :] . Q[m, :].
// That keeps small token counts efficient and re-unpacks each weight tile once per
// token tile of up to 192 tokens.
//
// The unpacked weights go from registers straight into TMEM and feed the MMA as its A
// operand from there, so the weight operand never takes a shared-memory round trip (on B200
// this removed the unpack warps' shared-memory stores and the tensor core's reads of them
// from the main loop); TMEM holds two accumulators and a weight ring of 2 (BN = 192), 3
// (BN = 160) or 4 stages, which caps the token tile at 192.
//
// One CTA per SM walks a static list of 128 x BN output tiles. Two shared-memory rings and
// the TMEM weight ring decouple the stages of the main loop, and two TMEM accumulators let
// the epilogue of one tile overlap the main loop of the next:
//  warp 0      TMEM allocation; lane 0 loads token tiles (two BN-row x 128-byte boxes per
//              256-byte K stage, 128-byte swizzle, no multicast) into ring B with TMA;
//  warps 1, 19 lane 0 of each issues 8 tcgen05.mma.kind::i8 (K = 32 each) per 256-byte K
//              stage, the two threads taking alternate stages, and commits them to the A/B
//              slots they read and, per tile, to the accumulator (barrier round trips of a
//              single issuing thread, not the tensor core, set the main-loop cadence on B200,
//              hence the wide stage and the second issuer);
//  warp 2      lane 0 loads packed weight tiles (128 rows x 64 bytes, 64-byte swizzle) into
//              ring P with TMA;
//  warps 3-10  epilogue, two warps per TMEM lane quarter splitting the columns; they zero
//              each accumulator as they read it (every MMA accumulates): TMEM ->
//              registers -> acc = D - sum_k q -> y = acc * (s_w * 1/s_x) -> a per-warp
//              staging tile in shared memory -> TMA store (the tensor map clips ragged
//              edges); the dequantisation factors and sum_k q of the tile's tokens sit in a
//              shared table filled before the accumulator is ready, and the accumulator goes
//              back to the MMA warps as soon as its last columns are in registers. For the
//              MLP's interleaved gate/up matrix the epilogue instead pairs lanes l and l + 16
//              (gate and up rows of one output) and stores h = SwiGLU(g, u);
//  warps 11-18 unpack ring P into the TMEM weight ring: the codes t + 1 themselves (the
//              MMA's A operand is unsigned; the epilogue removes sum_k q), one row per TMEM
//              lane, four K bytes per column.
// The token tile arrives in the permuted in-group K order produced by the quantiser, which
// is the order a packed word unpacks into with shifts and masks alone.
//
// Under programmatic dependent launch the weight producer and the unpack warps start
// before the quantiser grid has finished; only the token producer and the epilogue wait.
// Every mbarrier wait is bounded (bitnet_device.cuh): on expiry the kernel records a
// watchdog code, the other waits return at once, and the CTA drains its copies and MMAs
// and frees its TMEM before it exits.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "bitnet_device.cuh"
#include "bitnet_internal.h"
#include "swiglu_device.cuh"

namespace bitnet {
namespace {

constexpr int kBM = 128;  // weight rows per tile (MMA M)
constexpr int kSub = 128;  // K bytes per token sub-tile (TMA box width, 128-byte swizzle atom)
constexpr int kWarpB = 0, kWarpMma = 1, kWarpP = 2, kEpiWarp0 = 3, kEpiWarps = 8,
              kUnpWarp0 = 11, kUnpWarps = 8, kWarpMma2 = 19;
constexpr int kMmaIssuers = 2;                  // warps kWarpMma and kWarpMma2
constexpr int kThreads = (kWarpMma2 + 1) * 32;  // 640
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kHalfCols = 16;                           // columns per epilogue warp per round

template <int BN>
struct TcLayout {
    // K bytes per stage: 8 MMAs between barrier round trips, 16 for token tiles of at most
    // 64, where the round trip rather than the MMAs sets the stage's pace (measured on B200).
    static constexpr int kBK = BN <= 64 ? 512 : 256;
    static constexpr int kB = BN * kBK;       // token tile: kBK / kSub sub-tiles of BN x kSub
    static constexpr int kP = kBM * kBK / 4;  // packed weights, 8 or 16 KB
    static constexpr int kPBoxes = kBK / 256;        // 64-byte-wide packed TMA boxes per stage
    static constexpr int kChunksPerWarp = kBK / 128; // 16-byte packed chunks per unpack warp
    // Ring depths. The unpacked weights live in TMEM (kDA stages of 64 columns), so shared
    // memory carries only the token and packed-weight rings and the epilogue staging.
    // The two MMA issuers take the global K stages by parity. The token ring has an even
    // depth, so each of its slots is always consumed by the same issuer, in order: its TMA
    // fills may land out of order, and an issuer must never wait on a slot whose previous
    // fill has not landed (a parity wait cannot tell the two phases apart). The weight ring
    // needs no such rule: the unpack warps arrive in stage order, so when an issuer has
    // consumed its previous stage g - 2, every stage up to g - 2 >= g - kDA has completed.
    static constexpr int kDA = BN > 160 ? 2 : BN > 128 ? 3 : kBK == 512 ? 3 : 4;
    static constexpr int kDB = BN > 32 ? 4 : 6;
    static constexpr int kDP = BN > 160 ? 2 : 4;
    static_assert(kDB % 2 == 0, "one issuer per token-ring slot");
    static constexpr int kStage = 2048;  // per epilogue warp: 32 rows x 16 tokens x 4 bytes
    static constexpr int kOffB = 0;
    static constexpr int kOffP = kOffB + kDB * kB;
    static constexpr int kOffStage = kOffP + kDP * kP;
    static constexpr int kOffTab = kOffStage + kEpiWarps * kStage;  // BN floats, then BN int32
    static constexpr int kOffBar = kOffTab + (2 * BN * 4 + 15) / 16 * 16;
    static constexpr int kNumBars = 2 * (kDA + kDB + kDP) + 4;
    static constexpr int kSmem = kOffBar + kNumBars * 8 + 16 + 1024;  // + slot, flag, align
    // TMEM: two accumulators of BN columns, then the unpacked-weight ring.
    static constexpr uint32_t kAccCols = BN;
    static constexpr uint32_t kACol0 = 2 * BN;
    static constexpr uint32_t kAStageCols = kBK / 4;
    static constexpr uint32_t kTmemNeed = 2 * BN + kDA * kAStageCols;
    static constexpr uint32_t kTmemCols = kTmemNeed <= 32    ? 32
                                          : kTmemNeed <= 64  ? 64
                                          : kTmemNeed <= 128 ? 128
                                          : kTmemNeed <= 256 ? 256
                                                             : 512;
    static_assert(kTmemNeed <= 512, "TMEM budget");
    static_assert(kB % 1024 == 0, "swizzled tiles need 1024-byte alignment");
    static_assert(kSmem <= 232448, "shared memory budget");
};

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]) {
    static_assert(N % 8 == 0, "columns in multiples of 8");
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        uint32_t(&r)[8] = *reinterpret_cast<uint32_t(*)[8]>(&v[8 * i]);
        tmem_ld_32x32b_x8(taddr + uint32_t(8 * i), r);
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[N]) {
    static_assert(N % 8 == 0, "columns in multiples of 8");
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
        tmem_st_32x32b_x8(taddr + uint32_t(8 * i), *reinterpret_cast<const uint32_t(*)[8]>(&v[8 * i]));
}

struct TileCoord {
    int proj;
    int n0;   // first weight row of the tile within its projection
    int m0;   // first token of the tile
    int kt0;  // first K stage of the tile's main loop
};

__device__ __forceinline__ TileCoord tile_coord(const TcParams& p, int t, int bn, int num_k) {
    const int nt = t % p.n_tiles_total;
    TileCoord c;
    c.proj = 0;
#pragma unroll
    for (int jj = 1; jj < kMaxProj; ++jj)
        if (jj < p.nproj && nt >= p.proj[jj].tile_begin) c.proj = jj;
    c.n0 = (nt - p.proj[c.proj].tile_begin) * kBM;
    c.m0 = (t / p.n_tiles_total) * bn;
    // Tiles that share a token tile run at the same time on different SMs; starting their K
    // loops at different stages spreads their reads of that tile over L2. The int32 sum is
    // exact, so the order of the K stages does not change the result.
    c.kt0 = static_cast<int>((int64_t(nt) * 7) % num_k);
    return c;
}

// Barrier among the 8 epilogue warps only (named barrier 1).
__device__ __forceinline__ void epilogue_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

// rx[c] = 1/s_x of column c of round r: lane l of rx_pre holds slot q*32 + l = r*kHC + c.
template <int kHC, int kPre>
__device__ __forceinline__ void spread_rx(const float (&rx_pre)[kPre], int r, float (&rx)[kHC]) {
#pragma unroll
    for (int c = 0; c < kHC; ++c) {
        const int slot = r * kHC + c;
        float mine = 0.0f;
#pragma unroll
        for (int q = 0; q < kPre; ++q)
            if (q == slot / 32) mine = rx_pre[q];
        rx[c] = __shfl_sync(0xFFFFFFFFu, mine, slot % 32);
    }
}

// Stores kHC columns of outputs (tokens m0 .. m0 + kHC - 1, weight row n) from registers:
// y = acc * f[c], where f[c] is the column's dequantisation factor s_w * (1/s_x); lanes hold
// adjacent rows n, so each store writes 32 adjacent outputs of one token. Structured
// branch: the warp reconverges before the caller's next aligned TMEM load.
template <int kHC>
__device__ __forceinline__ void store_cols(const TcParams& p, const TcProj& pr, int m0, int64_t n,
                                           bool nvalid, const float (&f)[kHC],
                                           const uint32_t (&v)[kHC]) {
    if (nvalid) {
        const int64_t mbase = m0;
        if (p.out_kind == 2) {
            int32_t* yp = static_cast<int32_t*>(pr.y) + mbase * pr.N + n;
#pragma unroll
            for (int c = 0; c < kHC; ++c)
                if (mbase + c < p.M) yp[int64_t(c) * pr.N] = int32_t(v[c]);
        } else if (p.out_kind == 0) {
            __nv_bfloat16* yp = static_cast<__nv_bfloat16*>(pr.y) + mbase * pr.N + n;
#pragma unroll
            for (int c = 0; c < kHC; ++c)
                if (mbase + c < p.M)
                    yp[int64_t(c) * pr.N] =
                        __float2bfloat16_rn(__fmul_rn(__int2float_rn(int32_t(v[c])), f[c]));
        } else {
            float* yp = static_cast<float*>(pr.y) + mbase * pr.N + n;
#pragma unroll
            for (int c = 0; c < kHC; ++c)
                if (mbase + c < p.M) yp[int64_t(c) * pr.N] = __fmul_rn(__int2float_rn(int32_t(v[c])), f[c]);
        }
    }
    __syncwarp();
}

// Writes this warp's kHC x 32 output block into its staging tile, laid out [token][row] as
// the TMA store box expects (a row of 32 outputs per token; lanes write adjacent elements).
template <int kHC>
__device__ __forceinline__ void stage_cols(int out_kind, uint8_t* buf, int lane,
                                           const float (&f)[kHC], const uint32_t (&v)[kHC]) {
    if (out_kind == 0) {
        __nv_bfloat16* b = reinterpret_cast<__nv_bfloat16*>(buf) + lane;
#pragma unroll
        for (int c = 0; c < kHC; ++c)
            b[c * 32] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(int32_t(v[c])), f[c]));
    } else if (out_kind == 1) {
        float* b = reinterpret_cast<float*>(buf) + lane;
#pragma unroll
        for (int c = 0; c < kHC; ++c) b[c * 32] = __fmul_rn(__int2float_rn(int32_t(v[c])), f[c]);
    } else {
        int32_t* b = reinterpret_cast<int32_t*>(buf) + lane;
#pragma unroll
        for (int c = 0; c < kHC; ++c) b[c * 32] = int32_t(v[c]);
    }
}

// Column maxima over a half warp: lanes 16h .. 16h + 15 each hold N values (one per column)
// of 16-bit magnitudes (bf16 bits, sign cleared here). Each exchange step halves the columns a
// lane keeps, swapping the other half with its partner, until one column is left; the
// remaining steps reduce it. On return v[0] holds the maximum of column c over the 16 lanes
// (the returned c); lanes that differ only in their low 4 - log2(N) bits hold the same column.
template <int N>
__device__ __forceinline__ int half_warp_column_max(uint32_t* v, int lane) {
    static_assert(N >= 1 && N <= 16 && (N & (N - 1)) == 0, "N is a power of two up to 16");
#pragma unroll
    for (int c = 0; c < N; ++c) v[c] &= 0x7FFFu;
    int col = 0;
#pragma unroll
    for (int step = 0; step < 4; ++step) {
        const int o = 8 >> step;
        const int n = N >> step;  // columns still held
        if (n > 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const uint32_t send = upper ? v[i] : v[i + n / 2];
                const uint32_t keep = upper ? v[i + n / 2] : v[i];
                v[i] = max(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
            }
            if (upper) col += n / 2;
        } else {
            v[0] = max(v[0], __shfl_xor_sync(0xFFFFFFFFu, v[0], o));
        }
    }
    return col;
}

// Dequantisation factors of kHC consecutive tokens from the tile's shared table (a
// broadcast read: every lane reads the same addresses). The table holds s_w * (1/s_x) for
// a per-tensor scale and 1/s_x for per-row scales, where this lane's row scale sw is
// applied here: f = s_w * (1/s_x) rounded once either way.
template <int kHC>
__device__ __forceinline__ void table_factors(const float* tab, bool per_row, float sw,
                                              float (&f)[kHC]) {
    const float4* t4 = reinterpret_cast<const float4*>(tab);
#pragma unroll
    for (int q = 0; q < kHC / 4; ++q) {
        const float4 t = t4[q];
        f[4 * q + 0] = t.x;
        f[4 * q + 1] = t.y;
        f[4 * q + 2] = t.z;
        f[4 * q + 3] = t.w;
    }
    if (per_row) {
#pragma unroll
        for (int c = 0; c < kHC; ++c) f[c] = __fmul_rn(sw, f[c]);
    }
}

// Position in a ring of D slots: the slot and the parity of its current phase, advanced
// without divisions.
template <int D>
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next() {
        if (++slot == D) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// Work unit u = (tile t, K split sp): K stages [kb, kb + ns) of tile t.
struct Unit {
    int t, sp, kb, ns;
};

__device__ __forceinline__ Unit unit_of(int u, int splits, int num_k) {
    Unit w;
    if (splits == 1) {  // whole tiles: no divisions
        w.t = u;
        w.sp = 0;
        w.kb = 0;
        w.ns = num_k;
        return w;
    }
    w.t = u / splits;
    w.sp = u - w.t * splits;
    w.kb = (w.sp * num_k) / splits;
    w.ns = ((w.sp + 1) * num_k) / splits - w.kb;
    return w;
}

// K stage of the i-th stage of a unit: a whole tile rotates its start (see tile_coord); a
// split unit walks its own K range.
__device__ __forceinline__ int stage_k(const Unit& w, const TileCoord& tc, int i, int splits,
                                       int num_k) {
    return splits == 1 ? (tc.kt0 + i) % num_k : w.kb + i;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
    using L = TcLayout<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* p_full = bars;
    uint64_t* p_empty = p_full + L::kDP;
    uint64_t* a_full = p_empty + L::kDP;
    uint64_t* a_empty = a_full + L::kDA;
    uint64_t* b_full = a_empty + L::kDA;
    uint64_t* b_empty = b_full + L::kDB;
    uint64_t* acc_full = b_empty + L::kDB;  // [2]
    uint64_t* acc_empty = acc_full + 2;     // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_k = static_cast<int>((p.K + L::kBK - 1) / L::kBK);
    const int m_tiles = (p.M + BN - 1) / BN;
    const int num_tiles = m_tiles * p.n_tiles_total;
    const int splits = p.splits;
    const int num_units = num_tiles * splits;

    if (warp == kWarpB) {
        if (lane == 0) {
            for (int s = 0; s < L::kDP; ++s) {
                mbar_init(&p_full[s], 1);
                mbar_init(&p_empty[s], kUnpWarps);
            }
            for (int s = 0; s < L::kDA; ++s) {
                mbar_init(&a_full[s], kUnpWarps);
                mbar_init(&a_empty[s], 1);
            }
            for (int s = 0; s < L::kDB; ++s) {
                mbar_init(&b_full[s], 1);
                mbar_init(&b_empty[s], 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(&acc_full[b], kMmaIssuers);
                mbar_init(&acc_empty[b], kEpiWarps);
            }
            *abort_flag = 0;
            fence_mbar_init();
            tma_prefetch_desc(&p.tmap_q);
        }
        __syncwarp();
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();

    if (warp == kWarpB) {
        if (lane == 0) {
            // ---------------- token tiles (written by the quantiser grid)
            pdl_wait();
            Ring<L::kDB> rb;
            int kc = 0;
            for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
                const Unit w = unit_of(u, splits, num_k);
                const TileCoord tc = tile_coord(p, w.t, BN, num_k);
                for (int kt = 0; kt < w.ns; ++kt, ++kc, rb.next()) {
                    mbar_wait_bounded(&b_empty[rb.slot], rb.phase ^ 1, p.err, kErrWaitEmpty, abort_flag);
                    mbar_arrive_expect_tx(&b_full[rb.slot], L::kB);
                    const int kr = stage_k(w, tc, kt, splits, num_k);
#pragma unroll
                    for (int h = 0; h < L::kBK / kSub; ++h)
                        tma_load_2d(smem + L::kOffB + rb.slot * L::kB + h * BN * kSub, &p.tmap_q,
                                    &b_full[rb.slot], kr * L::kBK + h * kSub, tc.m0);
                }
            }
            for (int k = kc > L::kDB ? kc - L::kDB : 0; k < kc; ++k)  // drain
                mbar_wait_bounded(&b_full[k % L::kDB], (k / L::kDB) & 1, p.err, kErrWaitDrain, nullptr);
        }
        __syncwarp();
    } else if (warp == kWarpP) {
        if (lane == 0) {
            // ---------------- packed weight tiles (independent of earlier grids)
            for (int j = 0; j < p.nproj; ++j) tma_prefetch_desc(&p.tmap_w[j]);
            Ring<L::kDP> rp;
            int kc = 0;
            for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
                const Unit w = unit_of(u, splits, num_k);
                const TileCoord tc = tile_coord(p, w.t, BN, num_k);
                for (int kt = 0; kt < w.ns; ++kt, ++kc, rp.next()) {
                    mbar_wait_bounded(&p_empty[rp.slot], rp.phase ^ 1, p.err, kErrWaitEmpty, abort_flag);
                    mbar_arrive_expect_tx(&p_full[rp.slot], L::kP);
                    const int kr = stage_k(w, tc, kt, splits, num_k);
#pragma unroll
                    for (int b = 0; b < L::kPBoxes; ++b)  // 64-byte boxes, [box][row][64 bytes]
                        tma_load_2d(smem + L::kOffP + rp.slot * L::kP + b * (kBM * 64),
                                    &p.tmap_w[tc.proj], &p_full[rp.slot],
                                    kr * (L::kBK / 4) + b * 64, tc.n0);
                }
            }
            for (int k = kc > L::kDP ? kc - L::kDP : 0; k < kc; ++k)  // drain
                mbar_wait_bounded(&p_full[k % L::kDP], (k / L::kDP) & 1, p.err, kErrWaitDrain, nullptr);
        }
        __syncwarp();
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        if (lane == 0) {
            // ---------------- MMA issuers: two threads take alternate K stages of each tile,
            // so one thread's barrier waits and commits overlap the other's MMAs (one issuing
            // thread left the tensor pipe idle between stages, measured on B200). Every MMA
            // accumulates into an accumulator the epilogue zeroed; the int32 sums are exact in
            // any order. The token descriptor is advanced by adding the encoded start-address
            // offsets (bytes / 16) of the ring slot and the 32-byte K step; the weight operand
            // is read from its TMEM ring slot, 8 columns per K step.
            const int issuer = warp == kWarpMma ? 0 : 1;
            constexpr uint32_t idesc = idesc_i8(kBM, BN, /*a_unsigned=*/true);
            const uint32_t a_tmem0 = tmem_base + L::kACol0;
            const uint64_t b_desc0 = smem_desc_k_sw128(smem_addr(smem + L::kOffB));
            Ring<L::kDA> ra;
            Ring<L::kDB> rb;
            int i = 0;
            uint32_t g = 0;  // K stages of this CTA so far, over all its units
            for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++i) {
                const Unit w = unit_of(u, splits, num_k);
                const int buf = i & 1;
                // The epilogue released both accumulators once after zeroing them at start.
                mbar_wait_bounded(&acc_empty[buf], (i >> 1) & 1, p.err, kErrWaitAccum, abort_flag);
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(buf) * L::kAccCols;
                for (int kt = 0; kt < w.ns; ++kt, ++g, ra.next(), rb.next()) {
                    if (int(g & 1u) != issuer) continue;  // the other issuer's stage
                    mbar_wait_bounded(&a_full[ra.slot], ra.phase, p.err, kErrWaitUnpack, abort_flag);
                    mbar_wait_bounded(&b_full[rb.slot], rb.phase, p.err, kErrWaitTmaFull, abort_flag);
                    tc_fence_after();
                    const uint32_t at = a_tmem0 + uint32_t(ra.slot) * L::kAStageCols;
                    const uint64_t bd = b_desc0 + uint64_t(rb.slot * (L::kB >> 4));
#pragma unroll
                    for (int kk = 0; kk < L::kBK / 32; ++kk) {
                        const int h = kk / (kSub / 32), k32 = kk % (kSub / 32);
                        mma_i8_tmem_a(d, at + uint32_t(8 * kk),
                                      bd + uint64_t((h * BN * kSub) >> 4) + uint64_t(2 * k32), idesc,
                                      1u);
                    }
                    mma_commit(&a_empty[ra.slot]);
                    mma_commit(&b_empty[rb.slot]);
                }
                mma_commit(&acc_full[buf]);
            }
            if (i > 0)  // drain: no tensor-core operation may run when TMEM is freed
                mbar_wait_bounded(&acc_full[(i - 1) & 1], ((i - 1) >> 1) & 1, p.err, kErrWaitDrain,
                                  nullptr);
        }
        __syncwarp();
    } else if (warp >= kUnpWarp0) {
        // ---------------- unpack: ring P (shared memory) -> ring A (TMEM). A warp may only
        // reach its own TMEM lane quarter (warp % 4); the two warps of a quarter take the two
        // 128-weight halves of each row's 256-weight stage.
        const int quarter = warp & 3;
        const int half = (warp - kUnpWarp0) >> 2;
        const int row = quarter * 32 + lane;  // weight row of the tile = TMEM lane
        const uint32_t a_lane = tmem_base + (uint32_t(quarter * 32) << 16) + L::kACol0 +
                                uint32_t(half * (L::kAStageCols / 2));
        Ring<L::kDP> rp;
        Ring<L::kDA> ra;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
            const Unit w = unit_of(u, splits, num_k);
            for (int kt = 0; kt < w.ns; ++kt, rp.next(), ra.next()) {
                mbar_wait_bounded(&p_full[rp.slot], rp.phase, p.err, kErrWaitTmaFull, abort_flag);
                // The packed tile arrives in 64-byte-wide TMA boxes with the 64-byte swizzle:
                // 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3) of its box, so the
                // 32 lanes' reads (one row each) spread over all banks instead of four rows
                // sharing each bank. This warp takes chunks kChunksPerWarp * half ... of the row.
                const uint8_t* pslot = smem + L::kOffP + rp.slot * L::kP;
                const int sw = (row >> 1) & 3;
                uint4 pk[L::kChunksPerWarp];
#pragma unroll
                for (int i = 0; i < L::kChunksPerWarp; ++i) {
                    const int gc = L::kChunksPerWarp * half + i;  // chunk of the row's stage
                    pk[i] = *reinterpret_cast<const uint4*>(pslot + (gc >> 2) * (kBM * 64) +
                                                            row * 64 + (((gc & 3) ^ sw) << 4));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_empty[rp.slot]);
                // The MMA multiplies the codes c = t + 1 in {0, 1, 2} themselves (unsigned A
                // operand); the epilogue removes sum_k q once per token (sum q t = sum q c -
                // sum q). Packed word c holds 16 weights; its shifts by 0, 2, 4, 6 give the
                // four 32-bit columns in the permuted in-group K order of the token operand.
                // Two chunks (8 words) fill 32 TMEM columns.
#pragma unroll
                for (int g2 = 0; g2 < L::kChunksPerWarp / 2; ++g2) {
                    const uint32_t words[8] = {pk[2 * g2].x,     pk[2 * g2].y,     pk[2 * g2].z,
                                               pk[2 * g2].w,     pk[2 * g2 + 1].x, pk[2 * g2 + 1].y,
                                               pk[2 * g2 + 1].z, pk[2 * g2 + 1].w};
                    uint32_t t[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        t[4 * c + 0] = words[c] & 0x03030303u;
                        t[4 * c + 1] = (words[c] >> 2) & 0x03030303u;
                        t[4 * c + 2] = (words[c] >> 4) & 0x03030303u;
                        t[4 * c + 3] = (words[c] >> 6) & 0x03030303u;
                    }
                    if (g2 == 0) {  // the ring slot must be free before the first store
                        mbar_wait_bounded(&a_empty[ra.slot], ra.phase ^ 1, p.err, kErrWaitEmpty,
                                          abort_flag);
                        tc_fence_after();
                    }
                    tmem_st_32x32b_x32(a_lane + uint32_t(ra.slot) * L::kAStageCols +
                                           uint32_t(32 * g2),
                                       t);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[ra.slot]);
            }
        }
    } else {
        // ---------------- epilogue (warps 3-10: TMEM lane quarter warp % 4, column half)
        pdl_wait();  // r_x and split counters come from the quantiser grid; y may be read earlier
        const int quarter = warp & 3;
        const int colhalf = (warp - kEpiWarp0) >> 2;
        const int n_local = quarter * 32 + lane;
        const int et = threadIdx.x - kEpiWarp0 * 32;  // 0 .. 255
        volatile int32_t* last_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 2);
        uint8_t* stage = smem + L::kOffStage + (warp - kEpiWarp0) * L::kStage;
        float* tab = reinterpret_cast<float*>(smem + L::kOffTab);
        int32_t* qtab = reinterpret_cast<int32_t*>(tab + BN);  // sum_k q of the tile's tokens
        constexpr int kHC = BN / 2 < kHalfCols ? BN / 2 : kHalfCols;  // columns per warp per round
        constexpr int kRounds = BN / (2 * kHC);
        constexpr int kPre = (kRounds * kHC + 31) / 32;
        static_assert(kHC == 8 || kHC == 16, "store box width");
        static_assert(BN % (2 * kHC) == 0, "whole epilogue rounds");
        uint32_t staged_stores = 0;  // selects the half of the staging tile (2-byte outputs)
        // Every MMA accumulates, so an accumulator starts at zero: zero both now, and each
        // one again as its columns are read out, before it goes back to the MMA warps.
        uint32_t zeros[kHC];
#pragma unroll
        for (int c = 0; c < kHC; ++c) zeros[c] = 0u;
        {
            const uint32_t lane_base = tmem_base + (uint32_t(quarter * 32) << 16);
#pragma unroll 1
            for (int b = 0; b < 2; ++b)
#pragma unroll 1
                for (int r = 0; r < kRounds; ++r)
                    tmem_st_cols<kHC>(lane_base + uint32_t(b) * L::kAccCols +
                                          uint32_t(r * 2 * kHC + colhalf * kHC),
                                      zeros);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[0]);
                mbar_arrive(&acc_empty[1]);
            }
        }
        int i = 0;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++i) {
            const Unit w = unit_of(u, splits, num_k);
            const TileCoord tc = tile_coord(p, w.t, BN, num_k);
            const TcProj& pr = p.proj[tc.proj];
            const int64_t n = int64_t(tc.n0) + n_local;
            const bool nvalid = n < pr.N;
            // s_w is absent (nullptr) when the raw int32 accumulator is the output. SwiGLU
            // with per-tensor scales: lanes 0-15 hold gate rows (s_gate), 16-31 up rows (s_up).
            const float sw = p.out_kind == 2 ? 0.0f
                             : pr.sw_pair   ? pr.s_w[(lane >> 4) & 1]
                             : pr.per_row   ? (nvalid ? pr.s_w[n] : 0.0f)
                                            : pr.s_w[0];
            const int buf = i & 1;
            if (splits == 1) {
                // Dequantisation factors of the tile's tokens, filled while the main loop runs.
                epilogue_bar_sync();  // every warp is done with the previous tile's table
                if (et < BN) {
                    const int64_t m = int64_t(tc.m0) + et;
                    float fv = 0.0f;
                    if (p.out_kind != 2 && m < p.M) {
                        fv = p.r_x[m];
                        if (!pr.per_row) fv = __fmul_rn(sw, fv);
                    }
                    tab[et] = fv;
                    qtab[et] = m < p.M ? p.qsum[m] : 0;
                }
                epilogue_bar_sync();
                mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1, p.err, kErrWaitAccum, abort_flag);
                tc_fence_after();
                const uint32_t d =
                    tmem_base + uint32_t(buf) * L::kAccCols + (uint32_t(quarter * 32) << 16);
                const bool staged = pr.tma_store != 0;
#pragma unroll 1
                for (int r = 0; r < kRounds; ++r) {
                    const int col0 = r * 2 * kHC + colhalf * kHC;  // this warp's first column
                    uint32_t v[kHC];
                    tmem_ld_cols<kHC>(d + uint32_t(col0), v);
                    tmem_ld_wait();
                    tmem_st_cols<kHC>(d + uint32_t(col0), zeros);
                    if (r == kRounds - 1) {
                        // accumulator read out and zeroed: hand it back to the MMA warps
                        tmem_st_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc_empty[buf]);
                    }
                    {  // acc = sum q c - sum q (exact int32)
                        const int4* q4 = reinterpret_cast<const int4*>(qtab + col0);
#pragma unroll
                        for (int c4 = 0; c4 < kHC / 4; ++c4) {
                            const int4 qq = q4[c4];
                            v[4 * c4 + 0] = uint32_t(int32_t(v[4 * c4 + 0]) - qq.x);
                            v[4 * c4 + 1] = uint32_t(int32_t(v[4 * c4 + 1]) - qq.y);
                            v[4 * c4 + 2] = uint32_t(int32_t(v[4 * c4 + 2]) - qq.z);
                            v[4 * c4 + 3] = uint32_t(int32_t(v[4 * c4 + 3]) - qq.w);
                        }
                    }
                    float f[kHC];
                    table_factors<kHC>(tab + col0, pr.per_row != 0, sw, f);
                    if (p.swiglu) {
                        // Interleaved gate/up rows: lane l < 16 holds gate row j, lane l + 16
                        // the up row of the same output j = n0 / 2 + 16 quarter + l. Both
                        // dequantise as in the plain epilogue. Partner lanes (l, l + 16) then
                        // split the columns: one shuffle per column pair gives lane l the up
                        // value of column c and lane l + 16 the gate value of column
                        // c + kHC / 2, so every lane computes SwiGLU for half of the columns.
                        constexpr int kHalf = kHC / 2;
                        const bool gate_lane = lane < kSwigluBlock;
#pragma unroll
                        for (int c = 0; c < kHalf; ++c) {
                            const float y0 = __fmul_rn(__int2float_rn(int32_t(v[c])), f[c]);
                            const float y1 =
                                __fmul_rn(__int2float_rn(int32_t(v[c + kHalf])), f[c + kHalf]);
                            const float other =
                                __shfl_xor_sync(0xFFFFFFFFu, gate_lane ? y1 : y0, kSwigluBlock);
                            // lane l: column c; lane l + 16: column c + kHalf
                            const float g = gate_lane ? y0 : other;
                            const float u = gate_lane ? other : y1;
                            v[c] = swiglu_bf16_bits(g, u);
                        }
                        uint8_t* sb = stage + (staged_stores & 1u) * 1024u;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        {  // staging tile [token][16 outputs]
                            uint16_t* b = reinterpret_cast<uint16_t*>(sb) +
                                          (gate_lane ? lane : kHalf * kSwigluBlock + lane - kSwigluBlock);
#pragma unroll
                            for (int c = 0; c < kHalf; ++c) b[c * kSwigluBlock] = uint16_t(v[c]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        const int x = (tc.n0 >> 1) + quarter * kSwigluBlock, y = tc.m0 + col0;
                        if (lane == 0 && x < (pr.N >> 1) && y < p.M) {
                            tma_store_2d(&p.tmap_y[tc.proj], sb, x, y);
                            bulk_commit_group();
                        }
                        ++staged_stores;
                        if (p.hmax && x < (pr.N >> 1)) {  // warp-uniform
                            // Maxima of |h| over this warp's 16 outputs, per token: half-warp
                            // column maxima, stored as bf16 bits at hmax[token][x / 16].
                            const int c = half_warp_column_max<kHalf>(v, lane);
                            const int64_t m = int64_t(y) + c + (gate_lane ? 0 : kHalf);
                            if ((lane & (kSwigluBlock / kHalf - 1)) == 0 && m < p.M)
                                p.hmax[m * (pr.N >> 5) + (x >> 4)] = uint16_t(v[0]);
                        }
                    } else if (staged) {
                        // 2-byte outputs alternate between the two 1 KB halves of the staging
                        // tile; 4-byte outputs use all 2 KB, so the previous store must have
                        // read it out first.
                        uint8_t* sb = stage + (p.out_kind == 0 ? (staged_stores & 1u) * 1024u : 0u);
                        if (lane == 0) {
                            if (p.out_kind == 0)
                                bulk_wait_group_read<1>();
                            else
                                bulk_wait_group_read<0>();
                        }
                        __syncwarp();
                        stage_cols<kHC>(p.out_kind, sb, lane, f, v);
                        fence_proxy_async_smem();
                        __syncwarp();
                        const int x = tc.n0 + quarter * 32, y = tc.m0 + col0;
                        if (lane == 0 && x < pr.N && y < p.M) {
                            tma_store_2d(&p.tmap_y[tc.proj], sb, x, y);
                            bulk_commit_group();
                        }
                        ++staged_stores;
                    } else {
                        store_cols<kHC>(p, pr, tc.m0 + col0, n, nvalid, f, v);
                    }
                }
            } else {
                // 1/s_x of this warp's columns, fetched before the accumulator is ready: lane l
                // holds token (round r, column l % kHC) for r = l / kHC (+ rounds of 32 / kHC).
                float rx_pre[kPre];
#pragma unroll
                for (int q = 0; q < kPre; ++q) {
                    const int slot = q * 32 + lane;  // = round * kHC + column
                    const int rr = slot / kHC, cc = slot % kHC;
                    const int64_t m = int64_t(tc.m0) + rr * 2 * kHC + colhalf * kHC + cc;
                    rx_pre[q] = (p.out_kind != 2 && rr < kRounds && m < p.M) ? p.r_x[m] : 0.0f;
                }
                mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1, p.err, kErrWaitAccum, abort_flag);
                tc_fence_after();
                const uint32_t d =
                    tmem_base + uint32_t(buf) * L::kAccCols + (uint32_t(quarter * 32) << 16);
                // Split unit: this CTA adds its int32 partial tile into the tile's accumulation
                // tile, [tile][token][row]; a warp adds 32 adjacent rows per reduction.
                int32_t* acc = p.split_acc + size_t(w.t) * BN * kBM;
#pragma unroll 1
                for (int r = 0; r < kRounds; ++r) {
                    const int col0 = r * 2 * kHC + colhalf * kHC;
                    uint32_t v[kHC];
                    tmem_ld_cols<kHC>(d + uint32_t(col0), v);
                    tmem_ld_wait();
                    tmem_st_cols<kHC>(d + uint32_t(col0), zeros);
#pragma unroll
                    for (int c = 0; c < kHC; ++c)
                        atomicAdd(acc + size_t(col0 + c) * kBM + n_local, int32_t(v[c]));
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
                // The last unit of the tile to arrive reads the summed tile (exact int32 adds,
                // so the arrival order does not matter) and writes the outputs; no CTA waits
                // for another.
                __threadfence();
                epilogue_bar_sync();
                if (et == 0) *last_flag = atomicAdd(&p.split_cnt[w.t], 1) == splits - 1 ? 1 : 0;
                epilogue_bar_sync();
                if (*last_flag) {
                    __threadfence();
#pragma unroll 1
                    for (int r = 0; r < kRounds; ++r) {
                        const int col0 = r * 2 * kHC + colhalf * kHC;
                        uint32_t v[kHC];
#pragma unroll
                        for (int c = 0; c < kHC; ++c) {
                            const int64_t m = int64_t(tc.m0) + col0 + c;
                            v[c] = uint32_t(__ldcg(acc + size_t(col0 + c) * kBM + n_local) -
                                            (m < p.M ? p.qsum[m] : 0));
                        }
                        float rx[kHC];
                        spread_rx<kHC, kPre>(rx_pre, r, rx);
                        float f[kHC];
#pragma unroll
                        for (int c = 0; c < kHC; ++c) f[c] = __fmul_rn(sw, rx[c]);
                        store_cols<kHC>(p, pr, tc.m0 + col0, n, nvalid, f, v);
                    }
                }
                epilogue_bar_sync();  // last_flag is reused by the next unit
            }
        }
        // Staged stores must be complete before the CTA exits (their source is this CTA's
        // shared memory, and the next grid reads y).
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpB) {
        __syncwarp();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

int num_sms_cached() {
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

template <int BN>
cudaError_t launch_bn(const TcParams& p, cudaStream_t stream, bool pdl) {
    using L = TcLayout<BN>;
    auto kern = tc_gemm_kernel<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    const int units = ((p.M + BN - 1) / BN) * p.n_tiles_total * p.splits;
    const int grid = units < num_sms_cached() ? units : num_sms_cached();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
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

int tc_num_sms() { return num_sms_cached(); }

int tc_pick_bn(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 192;
}

cudaError_t launch_tc_gemm(const TcParams& p, int bn, cudaStream_t stream, bool pdl) {
    switch (bn) {
        case 16: return launch_bn<16>(p, stream, pdl);
        case 32: return launch_bn<32>(p, stream, pdl);
        case 64: return launch_bn<64>(p, stream, pdl);
        case 128: return launch_bn<128>(p, stream, pdl);
        case 160: return launch_bn<160>(p, stream, pdl);
        default: return launch_bn<192>(p, stream, pdl);
    }
}

}  // namespace bitnet
