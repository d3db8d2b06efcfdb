// Internal declarations shared by the kernel translation units and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "bitnet.h"

namespace bitnet {

constexpr int kMaxProj = BITNET_MAX_PROJ;

// ----------------------------------------------------------------------------- workspace
// Tensor-core path scratch: q (M, K) int8 in the in-group permuted K order, s_x (M),
// r_x = 1/s_x (M) and qsum (M, int32: the sum of each token's q), each region 256-byte
// aligned.
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline size_t ws_q_bytes(int64_t M, int64_t K) { return align256(size_t(M) * size_t(K)); }
inline size_t ws_scale_bytes(int64_t M) { return align256(size_t(M) * 4); }
// Then the partial maxima of |x| for a per-tensor activation scale (kMaxAmaxParts words).
constexpr int kMaxAmaxParts = 1024;
inline size_t ws_parts_bytes() { return size_t(kMaxAmaxParts) * 4; }
inline size_t ws_total_bytes(int64_t M, int64_t K) {
    return ws_q_bytes(M, K) + 3 * ws_scale_bytes(M) + ws_parts_bytes();
}

// SwiGLU of the MLP: interleaved gate/up weight rows come in blocks of this many rows.
constexpr int kSwigluBlock = 16;

// Optional split-K area after the base workspace: one int32 arrival counter and one int32
// accumulation tile (128 weight rows x BN tokens) per split tile; the quantiser zeroes the
// area on every call. Split-K runs only when the caller's workspace holds it.
constexpr int kMaxSplitTiles = 80;
int tc_pick_bn(int64_t M);
inline size_t ws_split_cnt_bytes() { return align256(size_t(kMaxSplitTiles) * 4); }
// Split-K runs only with token tiles of at most 64.
inline size_t ws_split_tile_bytes(int64_t M) {
    return size_t(128) * size_t(tc_pick_bn(M) < 64 ? tc_pick_bn(M) : 64) * 4;
}
inline size_t ws_split_bytes(int64_t M) {
    return ws_split_cnt_bytes() + size_t(kMaxSplitTiles) * ws_split_tile_bytes(M);
}

// ----------------------------------------------------------------------------- GEMV
struct GemvProj {
    const uint8_t* packed;
    const float* s_w;
    void* y;
    int64_t N;
    int64_t row_begin;  // first global row of this projection
    int32_t per_row;
    int32_t pad;
};

struct GemvParams {
    const uint16_t* x;   // (M, K) bf16 bits, or nullptr when q_in is used
    const int8_t* q_in;  // (M, K) int8 natural order (contraction-only mode)
    int64_t K;
    int64_t total_rows;
    int32_t M;
    int32_t nproj;
    int32_t out_kind;  // 0 bf16, 1 f32, 2 int32 accumulator
    int32_t stage_x;   // set by the launcher: stage x in shared memory
    int32_t swiglu;    // 1: proj[0] is an interleaved gate/up matrix, total_rows counts
                       // output pairs, y = SwiGLU (bf16, (M, proj[0].N))
    int32_t act_per_tensor;  // 1: one activation scale for all M tokens
    GemvProj proj[kMaxProj];
};

cudaError_t launch_gemv(const GemvParams& p, cudaStream_t stream, bool pdl);
bool gemv_supported(int64_t M, int64_t K);
// Rows per warp the dp4a GEMV takes for this call on a GPU of `sms` SMs (SwiGLU: 2 per
// gate/up pair): the launch's choice, also reported by the plan query.
int gemv_rows_per_warp(const GemvParams& p, int sms);
// The kernel-path choice of bitnet_linear / bitnet_linear_batch: true when a call with this
// token count, width, path and workspace runs the GEMV (which uses no workspace).
bool use_gemv(int64_t M, int64_t K, bitnet_path path, const void* ws, size_t ws_bytes);

// Decode GEMV on warp-level tensor-core MMA (mma.sync m16n8k32) for M <= 8 tokens: CTAs of 8
// warps own rt tiles of 16 weight rows, split over the warps by K. gemv_mma_plan returns false
// where it does not apply (M > 8, or q of the tokens too large for shared memory); otherwise
// the tiles per CTA, the grid and the packed chunks per lane.
bool gemv_mma_plan(const GemvParams& p, int sms, int* rt, int* grid, int* cpt);
// Where the warp-MMA GEMV runs under BITNET_PATH_AUTO: five to eight tokens (reached without a
// workspace) above 4 MiB of packed weights (chains of calls on B200: 6912 x 2560 at 8 tokens
// 14.1 against 20.1 us for the dp4a GEMV; 4096 x 4096, 4 MiB, 15.1 against 11.3). At one token
// it lost to the dp4a GEMV everywhere but in chains of 11 MB batched calls (7.0 against 8.2 us),
// and in the layer stacks, where it alternates with the dp4a GEMV, it lost there too (2B-4T
// stack at M = 1: 465 against 431 us per pass); BITNET_PATH_MMA still forces it.
constexpr int64_t kMmaMinBytesFewTokens = int64_t(4) << 20;
cudaError_t launch_gemv_mma(const GemvParams& p, int rt, int grid, int cpt, int32_t* err,
                            cudaStream_t stream, bool pdl);

// Streaming GEMV for one token and large matrices (a producer warp fills a shared-memory
// ring of 16-row weight stages with bulk copies; one CTA per SM). gemv_stream_plan returns
// false where it does not apply (M != 1, contraction-only input, K > 16384, or a ring of
// fewer than two stages). Used from kStreamMinBytes of packed weights per call: below that
// (measured on B200 in chains of calls) the register-resident kernel wins, because its
// grid leaves room for the next call's CTAs to start their weight loads early.
constexpr int64_t kStreamMinBytes = int64_t(12) << 20;
bool gemv_stream_plan(const GemvParams& p, int64_t* n_stages, int* depth, uint32_t* stage_bytes);
cudaError_t launch_gemv_stream(const GemvParams& p, int64_t n_stages, int depth,
                               uint32_t stage_bytes, int sms, int32_t* err, cudaStream_t stream,
                               bool pdl);

// ----------------------------------------------------------------------------- quantisation
// mode 0: natural-order q (public bitnet_quant_act); mode 1: permuted q + s_x + r_x for
// the tensor-core path. q_in != nullptr: copy-permute given int8 q (no scales).
// zero / zero_bytes: a 16-byte aligned region (multiple of 16 bytes) the launch clears, spread
// over its CTAs (the split-K area of the GEMM that follows), or null.
// amax_parts / n_parts: when set, every token uses the one scale of the whole input, whose
// amax is the maximum of these partial maxima (written by launch_amax_parts).
// tok_parts: when set, token m's amax is the maximum of tok_parts[m * K/16 .. + K/16), the
// maxima of |x| over its blocks of 16 values (bf16 bits) written by x's producer.
cudaError_t launch_quant(const uint16_t* x, const int8_t* q_in, int64_t M, int64_t K, int8_t* q,
                         float* s_x, float* r_x, int permuted, cudaStream_t stream, bool pdl,
                         void* zero = nullptr, int64_t zero_bytes = 0, int32_t* qsum = nullptr,
                         const uint32_t* amax_parts = nullptr, int n_parts = 0,
                         const uint16_t* tok_parts = nullptr);
// Partial maxima of |x| over all of x (M, K) into parts[0 .. amax_parts_count(M, K)).
int amax_parts_count(int64_t M, int64_t K);
cudaError_t launch_amax_parts(const uint16_t* x, int64_t M, int64_t K, uint32_t* parts,
                              cudaStream_t stream, bool pdl);

// ----------------------------------------------------------------------------- base-3 weights
// Five ternary weights per byte (kernels_b3.cu): bytes per row, 16 per started 80-weight chunk.
__host__ __device__ inline int64_t b3_row_bytes(int64_t K) { return 16 * ((K + 79) / 80); }
cudaError_t launch_pack_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                           cudaStream_t stream);
// Grid-stride one-token GEMV (kernels_gemv_gs.cu) for large matrices, 2-bit or base-3 (b3)
// weights: one 16-warp CTA per SM, each warp a ring of row pairs in registers.
bool gemv_gs_supported(const GemvParams& p, bool b3);
cudaError_t launch_gemv_gs(const GemvParams& p, bool b3, int sms, cudaStream_t stream, bool pdl);
// The grid-stride kernel replaces the streaming one for one-token SwiGLU calls from
// kStreamMinBytes with rows of at most this many K values (two chunks per lane, four row pairs
// in flight per warp). On B200 (µs per call): 8B-class gate/up + SwiGLU 28672 x 4096 12.3
// against 13.8; plain projections lost or tied (35.7 MB 8B q/k/v/gate/up batch 17.4 against
// 15.9; 50011 x 1024 17.4 against 14.7; 14336 x 4096 and a 14.6 MB 2B-4T batch equal).
constexpr int64_t kGsMaxK = 4096;

// ----------------------------------------------------------------------------- tensor parallel
// The steps a rank runs when a projection's K range is split across ranks (kernels_tp.cu).
cudaError_t launch_act_amax(const uint16_t* x, int64_t M, int64_t K, float* amax,
                            cudaStream_t stream);
cudaError_t launch_quant_amax(const uint16_t* x, const float* amax, int64_t M, int64_t K,
                              int8_t* q, float* s_x, cudaStream_t stream);
cudaError_t launch_dequant(const int32_t* acc, int64_t M, int64_t N, const float* s_x,
                           const float* s_w, int per_row, void* y, int out_kind,
                           cudaStream_t stream);

// ----------------------------------------------------------------------------- packing
cudaError_t launch_pack_weights(const float* W, int64_t N, int64_t K, int per_row,
                                uint8_t* packed, float* s_w, cudaStream_t stream);
cudaError_t launch_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                cudaStream_t stream);

// ----------------------------------------------------------------------------- tensor-core GEMM
struct TcProj {
    const float* s_w;
    void* y;
    int64_t N;
    int32_t per_row;
    int32_t tile_begin;  // first n-tile index of this projection in the flattened grid
    int32_t tma_store;   // 1: tmap_y is valid and the epilogue stores through it
    int32_t sw_pair;     // SwiGLU with per-tensor scales: s_w = {s_gate, s_up}
};

struct alignas(64) TcParams {
    CUtensorMap tmap_w[kMaxProj];  // packed weights (N, K/4) u8, box {64, 128}
    CUtensorMap tmap_q;            // workspace q (M, K) s8, box {128, BN}, 128-byte swizzle
    CUtensorMap tmap_y[kMaxProj];  // outputs (M, N), box {32 rows, tc_store_cols(BN) tokens}
    TcProj proj[kMaxProj];
    const float* r_x;     // (M) 1 / s_x
    const int32_t* qsum;  // (M) sum over k of q[m, k] (the MMA multiplies codes t + 1)
    int32_t* err;         // watchdog word
    int32_t* split_cnt;   // split-K: arrival counter per tile (zeroed by the quantiser)
    int32_t* split_acc;   // split-K: int32 accumulation tile per tile, [tile][token][row]
    int32_t splits;       // K splits per tile (1 = none)
    int32_t swiglu;       // 1: interleaved gate/up rows, outputs h = SwiGLU (bf16, M x N/2)
    uint16_t* hmax;       // SwiGLU: when set, (M, N/32) maxima of |h| over blocks of 16 outputs
    int64_t K;
    int32_t M;
    int32_t nproj;
    int32_t n_tiles_total;
    int32_t out_kind;  // 0 bf16, 1 f32, 2 int32
};

cudaError_t launch_tc_gemm(const TcParams& p, int bn, cudaStream_t stream, bool pdl);
int tc_num_sms();
// Tokens per epilogue store box for token-tile width bn.
inline int tc_store_cols(int bn) { return bn / 2 < 16 ? bn / 2 : 16; }

// Encodes the TMA descriptors (driver entry point fetched through the runtime).
// dtype: a CUtensorMapDataType value. swizzle_bytes: 0 (none), 64 or 128: the 16-byte chunks
// of each box row are permuted in shared memory as the hardware swizzle of that span.
bool encode_tmap_2d(CUtensorMap* map, int dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                    int swizzle_bytes);
inline bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                              int swizzle_bytes) {
    return encode_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer,
                          row_stride_bytes, box_inner, box_outer, swizzle_bytes);
}

// Device watchdog word of the current device.
int32_t* device_error_word();

}  // namespace bitnet
