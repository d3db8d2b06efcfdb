// C-ABI host layer of libbitnet: argument checks, kernel-path choice, TMA descriptor
// encoding and launches on the caller's stream. Declarations and contracts: include/bitnet.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "bitnet.h"
#include "bitnet_internal.h"

// The watchdog word every kernel reports bounded-wait expiries into.
__device__ int32_t g_bitnet_watchdog;

namespace bitnet {
namespace {

constexpr int kMaxDevices = 64;
int32_t* g_err_ptr[kMaxDevices] = {};
std::mutex g_err_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bitnet_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

// K, M, N shared checks.
bitnet_status check_mk(int64_t M, int64_t K) {
    if (M < 1 || K < 1 || M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return BITNET_ERR_SHAPE;
    if (K % 4 != 0) return BITNET_ERR_SHAPE;
    if (K % 64 != 0) return BITNET_ERR_UNSUPPORTED;
    return BITNET_OK;
}

bitnet_status check_n(int64_t N) {
    return (N < 1 || N >= (int64_t(1) << 31)) ? BITNET_ERR_SHAPE : BITNET_OK;
}

// Validated batch description shared by bitnet_linear and bitnet_linear_batch.
struct Batch {
    int nproj;
    bitnet_proj proj[kMaxProj];
};

bitnet_status validate_batch(const void* x, int64_t M, int64_t K, const bitnet_proj* projs,
                             int32_t nproj, int out_kind, Batch* b) {
    if (!x || !projs) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (nproj < 1 || nproj > kMaxProj) return BITNET_ERR_SHAPE;
    if (out_kind < 0 || out_kind > 2) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(x, 16)) return BITNET_ERR_ALIGN;
    b->nproj = nproj;
    for (int i = 0; i < nproj; ++i) {
        const bitnet_proj& pr = projs[i];
        if (!pr.packed || !pr.y || (out_kind != 2 && !pr.s_w)) return BITNET_ERR_NULL;
        if ((st = check_n(pr.N)) != BITNET_OK) return st;
        if (pr.mode != BITNET_SCALE_PER_TENSOR && pr.mode != BITNET_SCALE_PER_ROW)
            return BITNET_ERR_UNSUPPORTED;
        if (pr.reserved != 0) return BITNET_ERR_UNSUPPORTED;
        if (!aligned(pr.packed, 16) || !aligned(pr.y, 16) || (pr.s_w && !aligned(pr.s_w, 4)))
            return BITNET_ERR_ALIGN;
        b->proj[i] = pr;
    }
    return BITNET_OK;
}

bitnet_status check_workspace(void* ws, size_t bytes, int64_t M, int64_t K) {
    if (!ws || bytes < ws_total_bytes(M, K)) return BITNET_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return BITNET_ERR_ALIGN;
    return BITNET_OK;
}

}  // namespace

// Five to eight tokens take the tensor-core path when the caller's workspace holds it: the
// GEMV's per-CTA quantisation and dp4a work grow with the token count, and on B200 the
// tensor-core path with 16-token tiles is as fast or faster there (2B-4T shapes, 8 tokens:
// 10.7 / 8.7 / 20.9 / 27.2 us per GEMV call against about 10 / 9 / 11 / 15 us).
bool use_gemv(int64_t M, int64_t K, bitnet_path path, const void* ws, size_t ws_bytes) {
    if (path == BITNET_PATH_GEMV || path == BITNET_PATH_MMA) return true;
    if (path == BITNET_PATH_TC) return false;
    if (M > BITNET_GEMV_MAX_M || !gemv_supported(M, K)) return false;
    if (M <= BITNET_GEMV_AUTO_M) return true;
    return !(ws && ws_bytes >= ws_total_bytes(M, K) && aligned(ws, 256));
}

namespace {

// The launch decisions of one call, shared by run_batch and bitnet_linear_plan.
struct Plan {
    int kernel = 0;  // BITNET_KERNEL_*
    GemvParams gp;   // GEMV family: the kernel's parameters
    int rt = 0, grid = 0, cpt = 0;                       // warp-MMA decode GEMV
    int64_t n_stages = 0;                                // streaming GEMV
    int depth = 0;
    uint32_t stage_bytes = 0;
    int bn = 0, splits = 1, tiles = 0;                   // tensor-core GEMM
};

// Chooses the kernels of a validated batch (pointers are copied, never dereferenced).
bitnet_status plan_batch(const uint16_t* x_bf16, const int8_t* q_in, int64_t M, int64_t K,
                         const Batch& b, int out_kind, const void* workspace,
                         size_t workspace_bytes, bitnet_path path, bool swiglu,
                         bool act_per_tensor, Plan* pl) {
    if (use_gemv(M, K, path, workspace, workspace_bytes)) {
        if (!gemv_supported(M, K)) return BITNET_ERR_UNSUPPORTED;
        GemvParams& p = pl->gp;
        std::memset(&p, 0, sizeof(p));
        p.x = x_bf16;
        p.q_in = q_in;
        p.K = K;
        p.M = static_cast<int32_t>(M);
        p.nproj = b.nproj;
        p.out_kind = out_kind;
        p.act_per_tensor = act_per_tensor ? 1 : 0;
        int64_t rows = 0;
        for (int i = 0; i < b.nproj; ++i) {
            p.proj[i].packed = b.proj[i].packed;
            p.proj[i].s_w = b.proj[i].s_w;
            p.proj[i].y = b.proj[i].y;
            p.proj[i].N = b.proj[i].N;
            p.proj[i].per_row = b.proj[i].mode == BITNET_SCALE_PER_ROW;
            p.proj[i].row_begin = rows;
            rows += b.proj[i].N;
        }
        p.total_rows = rows;
        if (swiglu) {  // one output per gate/up row pair: I pairs, output width I
            p.swiglu = 1;
            p.total_rows = rows / 2;
            p.proj[0].N = rows / 2;
        }
        // One token and a matrix too large for one wave of register-resident rows: the
        // streaming kernel, or for the MLP's gate/up pairs with rows of at most kGsMaxK the
        // grid-stride kernel (measured faster there on B200, slower on plain projections).
        // The warp-MMA GEMV where it measured faster than the dp4a GEMV on B200 (five to
        // eight tokens above kMmaMinBytesFewTokens, reached without a workspace); the dp4a
        // GEMV otherwise.
        const int64_t wbytes = rows * (K / 4);
        if (path == BITNET_PATH_MMA) {
            if (!gemv_mma_plan(p, tc_num_sms(), &pl->rt, &pl->grid, &pl->cpt))
                return BITNET_ERR_UNSUPPORTED;
            pl->kernel = BITNET_KERNEL_MMA_GEMV;
            return BITNET_OK;
        }
        const bool mma_pays = path == BITNET_PATH_AUTO && M >= 5 && wbytes > kMmaMinBytesFewTokens;
        if (wbytes >= kStreamMinBytes && swiglu && K <= kGsMaxK && gemv_gs_supported(p, false)) {
            pl->kernel = BITNET_KERNEL_GS;
            const int64_t per_cta = swiglu ? 16 : 32;
            const int64_t want = (p.total_rows + per_cta - 1) / per_cta;
            pl->grid = static_cast<int>(want < tc_num_sms() ? want : tc_num_sms());
        } else if (wbytes >= kStreamMinBytes &&
                   gemv_stream_plan(p, &pl->n_stages, &pl->depth, &pl->stage_bytes)) {
            pl->kernel = BITNET_KERNEL_STREAM;
            pl->grid = static_cast<int>(pl->n_stages < tc_num_sms() ? pl->n_stages : tc_num_sms());
        } else if (mma_pays && gemv_mma_plan(p, tc_num_sms(), &pl->rt, &pl->grid, &pl->cpt)) {
            pl->kernel = BITNET_KERNEL_MMA_GEMV;
        } else {
            pl->kernel = BITNET_KERNEL_GEMV;
        }
        return BITNET_OK;
    }

    if (!workspace || workspace_bytes < ws_total_bytes(M, K)) return BITNET_ERR_WORKSPACE;
    pl->kernel = BITNET_KERNEL_TC;
    int tiles = 0;
    for (int i = 0; i < b.nproj; ++i) tiles += static_cast<int>((b.proj[i].N + 127) / 128);
    pl->tiles = tiles;
    // Token tile width: the widest that M needs; past 128 tokens, 192, 160 or 128, whichever
    // gives the shortest run of tile waves, a K stage of a BN-token tile costing about
    // BN + 264 units (fitted to per-call times measured on B200 at M = 512 ... 4096).
    const int sms = tc_num_sms();
    int bn = tc_pick_bn(M);
    if (bn > 128) {
        auto waves_cost = [&](int64_t w) {
            const int64_t t = int64_t(tiles) * ((M + w - 1) / w);
            return ((t + sms - 1) / sms) * (w + 264);
        };
        int64_t best = waves_cost(bn);
        for (int w : {160, 128}) {
            const int64_t c = waves_cost(w);
            if (c <= best) {
                best = c;
                bn = w;
            }
        }
    }
    pl->bn = bn;
    // Split-K when the tiles leave most SMs idle and the workspace holds the split area:
    // each tile's K range is cut into `splits` units (at least 512 K bytes each) so that about
    // one unit runs per SM; units add their int32 partial tiles into a zeroed accumulation tile.
    pl->splits = 1;
    // K stages of the kernel: 512 bytes for token tiles of at most 64, else 256 bytes.
    const int64_t kstage = bn <= 64 ? 512 : 256;
    const int64_t num_k = (K + kstage - 1) / kstage;
    const int64_t m_tiles = (M + bn - 1) / bn;
    const int64_t tiles_all = m_tiles * tiles;
    // Measured on B200: splitting pays for token tiles of up to 32, and of 64 with long K
    // loops; for wider tiles the atomic reduction of the partial tiles costs more than the
    // shorter main loop saves.
    const bool split_pays = !swiglu && (bn <= 32 || (bn == 64 && K >= 4096));
    const int64_t unit_stages = 512 / kstage;  // a split unit spans at least 512 K bytes
    if (split_pays && tiles_all * 4 <= sms && tiles_all <= kMaxSplitTiles &&
        num_k >= 2 * unit_stages && workspace_bytes >= ws_total_bytes(M, K) + ws_split_bytes(M)) {
        int64_t sp = sms / tiles_all;
        if (sp > num_k / unit_stages) sp = num_k / unit_stages;
        if (sp > 8) sp = 8;
        if (sp >= 2) pl->splits = static_cast<int>(sp);
    }
    const int64_t units = tiles_all * pl->splits;
    pl->grid = static_cast<int>(units < sms ? units : sms);
    return BITNET_OK;
}

// Runs a validated batch. x_bf16 or q_in (int8, contraction-only) is the input. swiglu: the
// batch is one interleaved gate/up matrix of N = 2I rows whose output is h (M, I) bf16.
// Tensor-core path only: xmax, the (M, K/16) block maxima of |x| that the quantiser reduces
// instead of x's rows; hmax, the (M, I/16) block maxima of |h| the SwiGLU epilogue writes.
bitnet_status run_batch(const uint16_t* x_bf16, const int8_t* q_in, int64_t M, int64_t K,
                        const Batch& b, int out_kind, void* workspace, size_t workspace_bytes,
                        bitnet_path path, cudaStream_t stream, bool swiglu = false,
                        bool act_per_tensor = false, const uint16_t* xmax = nullptr,
                        uint16_t* hmax = nullptr) {
    Plan pl;
    bitnet_status pst = plan_batch(x_bf16, q_in, M, K, b, out_kind, workspace, workspace_bytes,
                                   path, swiglu, act_per_tensor, &pl);
    if (pst != BITNET_OK) return pst;
    if (pl.kernel != BITNET_KERNEL_TC && (xmax || hmax)) return BITNET_ERR_UNSUPPORTED;
    if (pl.kernel == BITNET_KERNEL_GS)
        return from_cuda(launch_gemv_gs(pl.gp, /*b3=*/false, tc_num_sms(), stream, /*pdl=*/true));
    if (pl.kernel == BITNET_KERNEL_STREAM) {
        int32_t* err = device_error_word();
        if (!err) return BITNET_ERR_CUDA;
        return from_cuda(launch_gemv_stream(pl.gp, pl.n_stages, pl.depth, pl.stage_bytes,
                                            tc_num_sms(), err, stream, /*pdl=*/true));
    }
    if (pl.kernel == BITNET_KERNEL_MMA_GEMV) {
        int32_t* err = device_error_word();
        if (!err) return BITNET_ERR_CUDA;
        return from_cuda(launch_gemv_mma(pl.gp, pl.rt, pl.grid, pl.cpt, err, stream, /*pdl=*/true));
    }
    if (pl.kernel == BITNET_KERNEL_GEMV) return from_cuda(launch_gemv(pl.gp, stream, /*pdl=*/true));

    bitnet_status st = check_workspace(workspace, workspace_bytes, M, K);
    if (st != BITNET_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int8_t* q_ws = reinterpret_cast<int8_t*>(ws);
    float* s_x = reinterpret_cast<float*>(ws + ws_q_bytes(M, K));
    float* r_x = reinterpret_cast<float*>(ws + ws_q_bytes(M, K) + ws_scale_bytes(M));
    int32_t* qsum = reinterpret_cast<int32_t*>(ws + ws_q_bytes(M, K) + 2 * ws_scale_bytes(M));
    uint32_t* amax_parts =
        reinterpret_cast<uint32_t*>(ws + ws_q_bytes(M, K) + 3 * ws_scale_bytes(M));

    TcParams p;
    std::memset(&p, 0, sizeof(p));
    int tiles = 0;
    for (int i = 0; i < b.nproj; ++i) {
        const int64_t N = b.proj[i].N;
        if (!encode_tmap_2d_u8(&p.tmap_w[i], b.proj[i].packed, uint64_t(K / 4), uint64_t(N),
                               uint64_t(K / 4), 64, 128, /*swizzle_bytes=*/64))
            return BITNET_ERR_CUDA;
        p.proj[i].s_w = b.proj[i].s_w;
        p.proj[i].y = b.proj[i].y;
        p.proj[i].N = N;
        p.proj[i].per_row = b.proj[i].mode == BITNET_SCALE_PER_ROW;
        if (swiglu) {  // the factor table holds 1/s_x; each lane applies its row's scale
            p.proj[i].sw_pair = b.proj[i].mode == BITNET_SCALE_PER_TENSOR;
            p.proj[i].per_row = 1;
        }
        p.proj[i].tile_begin = tiles;
        tiles += static_cast<int>((N + 127) / 128);
    }
    const int bn = pl.bn;
    if (!encode_tmap_2d_u8(&p.tmap_q, q_ws, uint64_t(K), uint64_t(M), uint64_t(K), 128,
                           uint32_t(bn), /*swizzle_bytes=*/128))
        return BITNET_ERR_CUDA;
    // Outputs go out through TMA stores when the rows of y are 16-byte aligned; otherwise
    // the epilogue stores from registers.
    const uint64_t elem = out_kind == 0 ? 2 : 4;
    const int y_type = out_kind == 0   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                       : out_kind == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                       : CU_TENSOR_MAP_DATA_TYPE_INT32;
    if (swiglu) {  // h (M, I) bf16 through TMA stores of 16 outputs x tc_store_cols tokens
        const uint64_t I = uint64_t(b.proj[0].N) / 2;
        if (!encode_tmap_2d(&p.tmap_y[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b.proj[0].y, I,
                            uint64_t(M), I * 2, kSwigluBlock, uint32_t(tc_store_cols(bn)),
                            /*swizzle_bytes=*/0))
            return BITNET_ERR_CUDA;
        p.proj[0].tma_store = 1;
        p.swiglu = 1;
        p.hmax = hmax;
    }
    for (int i = 0; i < b.nproj && !swiglu; ++i) {
        const uint64_t N = uint64_t(b.proj[i].N);
        p.proj[i].tma_store = 0;
        if ((reinterpret_cast<uintptr_t>(b.proj[i].y) & 15) == 0 && (N * elem) % 16 == 0) {
            if (!encode_tmap_2d(&p.tmap_y[i], y_type, b.proj[i].y, N, uint64_t(M), N * elem, 32,
                                uint32_t(tc_store_cols(bn)), /*swizzle_bytes=*/0))
                return BITNET_ERR_CUDA;
            p.proj[i].tma_store = 1;
        }
    }
    p.r_x = r_x;
    p.qsum = qsum;
    p.err = device_error_word();
    if (!p.err) return BITNET_ERR_CUDA;
    p.K = K;
    p.M = static_cast<int32_t>(M);
    p.nproj = b.nproj;
    p.n_tiles_total = tiles;
    p.out_kind = out_kind;

    p.splits = pl.splits;
    void* zero = nullptr;
    int64_t zero_bytes = 0;
    if (pl.splits > 1) {
        const int64_t tiles_all = ((M + bn - 1) / bn) * tiles;
        uint8_t* split = ws + ws_total_bytes(M, K);
        p.split_cnt = reinterpret_cast<int32_t*>(split);
        p.split_acc = reinterpret_cast<int32_t*>(split + ws_split_cnt_bytes());
        zero = split;
        zero_bytes = int64_t(ws_split_cnt_bytes() + size_t(tiles_all) * size_t(128) * bn * 4);
    }

    const bool per_tensor = act_per_tensor && !q_in;
    if (per_tensor && launch_amax_parts(x_bf16, M, K, amax_parts, stream, /*pdl=*/true) !=
                          cudaSuccess)
        return BITNET_ERR_CUDA;
    cudaError_t e = launch_quant(x_bf16, q_in, M, K, q_ws, q_in ? nullptr : s_x,
                                 q_in ? nullptr : r_x, /*permuted=*/1, stream, /*pdl=*/true, zero,
                                 zero_bytes, qsum, per_tensor ? amax_parts : nullptr,
                                 per_tensor ? amax_parts_count(M, K) : 0, xmax);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    return from_cuda(launch_tc_gemm(p, bn, stream, /*pdl=*/true));
}

}  // namespace

int32_t* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_bitnet_watchdog) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int32_t*>(ptr);
    }
    return g_err_ptr[dev];
}

bool encode_tmap_2d(CUtensorMap* map, int dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                    int swizzle_bytes) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = g_encode(map, static_cast<CUtensorMapDataType>(dtype), 2, const_cast<void*>(base),
                                dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace bitnet

using namespace bitnet;

extern "C" {

bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, bitnet_scale_mode mode,
                                  uint8_t* packed, float* s_w, void* stream) {
    if (!W || !packed || !s_w) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(1, K);
    if (st != BITNET_OK) return st;
    if ((st = check_n(N)) != BITNET_OK) return st;
    if (mode != BITNET_SCALE_PER_TENSOR && mode != BITNET_SCALE_PER_ROW) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(s_w, 4)) return BITNET_ERR_ALIGN;
    return from_cuda(launch_pack_weights(W, N, K, mode == BITNET_SCALE_PER_ROW, packed, s_w,
                                         static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_pack_ternary(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                  void* stream) {
    if (!t || !packed) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(1, K);
    if (st != BITNET_OK) return st;
    if ((st = check_n(N)) != BITNET_OK) return st;
    if (!aligned(t, 16) || !aligned(packed, 16)) return BITNET_ERR_ALIGN;
    return from_cuda(launch_pack_ternary(t, N, K, packed, static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s_x,
                               void* stream) {
    if (!x || !q || !s_x) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s_x, 4)) return BITNET_ERR_ALIGN;
    return from_cuda(launch_quant(x, nullptr, M, K, q, s_x, nullptr, /*permuted=*/0,
                                  static_cast<cudaStream_t>(stream), /*pdl=*/false));
}

bitnet_status bitnet_quant_act_ex(const uint16_t* x, int64_t M, int64_t K, bitnet_act_mode act,
                                  int8_t* q, float* s_x, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    if (act != BITNET_ACT_PER_TOKEN && act != BITNET_ACT_PER_TENSOR) return BITNET_ERR_UNSUPPORTED;
    if (act == BITNET_ACT_PER_TOKEN) return bitnet_quant_act(x, M, K, q, s_x, stream);
    if (!x || !q || !s_x) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s_x, 4)) return BITNET_ERR_ALIGN;
    static_assert(BITNET_QUANT_WORKSPACE_BYTES >= kMaxAmaxParts * 4, "partial maxima fit");
    if (!workspace || workspace_bytes < BITNET_QUANT_WORKSPACE_BYTES) return BITNET_ERR_WORKSPACE;
    if (!aligned(workspace, 4)) return BITNET_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* parts = static_cast<uint32_t*>(workspace);
    if (launch_amax_parts(x, M, K, parts, s, /*pdl=*/false) != cudaSuccess) return BITNET_ERR_CUDA;
    return from_cuda(launch_quant(x, nullptr, M, K, q, s_x, nullptr, /*permuted=*/0, s,
                                  /*pdl=*/true, nullptr, 0, nullptr, parts,
                                  amax_parts_count(M, K)));
}

size_t bitnet_linear_workspace_size(int64_t M, int64_t K) {
    if (M < 1 || K < 1) return 0;
    return ws_total_bytes(M, K) + ws_split_bytes(M);
}

bitnet_status bitnet_linear_batch_ex(const uint16_t* x, int64_t M, int64_t K,
                                     const bitnet_proj* projs, int32_t nproj,
                                     bitnet_out_dtype out_dtype, void* workspace,
                                     size_t workspace_bytes, bitnet_path path, void* stream) {
    if (out_dtype != BITNET_OUT_BF16 && out_dtype != BITNET_OUT_F32) return BITNET_ERR_UNSUPPORTED;
    if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC &&
        path != BITNET_PATH_MMA)
        return BITNET_ERR_UNSUPPORTED;
    Batch b;
    bitnet_status st = validate_batch(x, M, K, projs, nproj, int(out_dtype), &b);
    if (st != BITNET_OK) return st;
    return run_batch(x, nullptr, M, K, b, int(out_dtype), workspace, workspace_bytes, path,
                     static_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_linear_batch_act(const uint16_t* x, int64_t M, int64_t K,
                                      const bitnet_proj* projs, int32_t nproj,
                                      bitnet_out_dtype out_dtype, bitnet_act_mode act,
                                      void* workspace, size_t workspace_bytes, bitnet_path path,
                                      void* stream) {
    if (act != BITNET_ACT_PER_TOKEN && act != BITNET_ACT_PER_TENSOR) return BITNET_ERR_UNSUPPORTED;
    if (out_dtype != BITNET_OUT_BF16 && out_dtype != BITNET_OUT_F32) return BITNET_ERR_UNSUPPORTED;
    if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC &&
        path != BITNET_PATH_MMA)
        return BITNET_ERR_UNSUPPORTED;
    Batch b;
    bitnet_status st = validate_batch(x, M, K, projs, nproj, int(out_dtype), &b);
    if (st != BITNET_OK) return st;
    return run_batch(x, nullptr, M, K, b, int(out_dtype), workspace, workspace_bytes, path,
                     static_cast<cudaStream_t>(stream), /*swiglu=*/false,
                     act == BITNET_ACT_PER_TENSOR);
}

bitnet_status bitnet_linear_batch(const uint16_t* x, int64_t M, int64_t K,
                                  const bitnet_proj* projs, int32_t nproj,
                                  bitnet_out_dtype out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    return bitnet_linear_batch_ex(x, M, K, projs, nproj, out_dtype, workspace, workspace_bytes,
                                  BITNET_PATH_AUTO, stream);
}

bitnet_status bitnet_linear_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                               const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                               bitnet_out_dtype out_dtype, void* workspace,
                               size_t workspace_bytes, bitnet_path path, void* stream) {
    bitnet_proj pr;
    pr.packed = packed;
    pr.s_w = s_w;
    pr.mode = int32_t(mode);
    pr.reserved = 0;
    pr.N = N;
    pr.y = y;
    return bitnet_linear_batch_ex(x, M, K, &pr, 1, out_dtype, workspace, workspace_bytes, path,
                                  stream);
}

bitnet_status bitnet_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                            const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                            bitnet_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                            void* stream) {
    return bitnet_linear_ex(x, M, K, packed, s_w, mode, N, y, out_dtype, workspace,
                            workspace_bytes, BITNET_PATH_AUTO, stream);
}

bitnet_status bitnet_linear_i32(const int8_t* q, int64_t M, int64_t K, const uint8_t* packed,
                                int64_t N, int32_t* acc, void* workspace, size_t workspace_bytes,
                                bitnet_path path, void* stream) {
    if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC &&
        path != BITNET_PATH_MMA)
        return BITNET_ERR_UNSUPPORTED;
    bitnet_proj pr;
    pr.packed = packed;
    pr.s_w = nullptr;
    pr.mode = BITNET_SCALE_PER_TENSOR;
    pr.reserved = 0;
    pr.N = N;
    pr.y = acc;
    Batch b;
    bitnet_status st = validate_batch(q, M, K, &pr, 1, /*out_kind=*/2, &b);
    if (st != BITNET_OK) return st;
    return run_batch(nullptr, q, M, K, b, 2, workspace, workspace_bytes, path,
                     static_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_interleave_gate_up(const uint8_t* packed_gate, const float* s_w_gate,
                                        const uint8_t* packed_up, const float* s_w_up,
                                        bitnet_scale_mode mode, int64_t I, int64_t K,
                                        uint8_t* packed_gu, float* s_w_gu, void* stream) {
    if (!packed_gate || !s_w_gate || !packed_up || !s_w_up || !packed_gu || !s_w_gu)
        return BITNET_ERR_NULL;
    bitnet_status st = check_mk(1, K);
    if (st != BITNET_OK) return st;
    if ((st = check_n(I)) != BITNET_OK) return st;
    if (I % kSwigluBlock != 0) return BITNET_ERR_SHAPE;
    if (mode != BITNET_SCALE_PER_TENSOR && mode != BITNET_SCALE_PER_ROW) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(packed_gate, 16) || !aligned(packed_up, 16) || !aligned(packed_gu, 16) ||
        !aligned(s_w_gate, 4) || !aligned(s_w_up, 4) || !aligned(s_w_gu, 4))
        return BITNET_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Blocks of 16 rows: gate block b -> rows 32b.., up block b -> rows 32b + 16.. (one 2D
    // copy per matrix, a "row" of the copy being one block).
    const size_t row = size_t(K / 4);
    const size_t blk = row * kSwigluBlock;
    const size_t nblk = size_t(I / kSwigluBlock);
    cudaError_t e = cudaMemcpy2DAsync(packed_gu, 2 * blk, packed_gate, blk, blk, nblk,
                                      cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(packed_gu + blk, 2 * blk, packed_up, blk, blk, nblk,
                              cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) {
        if (mode == BITNET_SCALE_PER_ROW) {
            const size_t sblk = sizeof(float) * kSwigluBlock;
            e = cudaMemcpy2DAsync(s_w_gu, 2 * sblk, s_w_gate, sblk, sblk, nblk,
                                  cudaMemcpyDeviceToDevice, s);
            if (e == cudaSuccess)
                e = cudaMemcpy2DAsync(s_w_gu + kSwigluBlock, 2 * sblk, s_w_up, sblk, sblk, nblk,
                                      cudaMemcpyDeviceToDevice, s);
        } else {
            e = cudaMemcpyAsync(s_w_gu, s_w_gate, sizeof(float), cudaMemcpyDeviceToDevice, s);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(s_w_gu + 1, s_w_up, sizeof(float), cudaMemcpyDeviceToDevice, s);
        }
    }
    return from_cuda(e);
}

bitnet_status bitnet_linear_swiglu(const uint16_t* x, int64_t M, int64_t K,
                                   const uint8_t* packed_gu, const float* s_w_gu,
                                   bitnet_scale_mode mode, int64_t I, uint16_t* h,
                                   void* workspace, size_t workspace_bytes, bitnet_path path,
                                   void* stream) {
    if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC &&
        path != BITNET_PATH_MMA)
        return BITNET_ERR_UNSUPPORTED;
    if (!h) return BITNET_ERR_NULL;
    bitnet_status st = check_n(I);
    if (st != BITNET_OK) return st;
    if (I % kSwigluBlock != 0 || 2 * I >= (int64_t(1) << 31)) return BITNET_ERR_SHAPE;
    bitnet_proj pr;
    pr.packed = packed_gu;
    pr.s_w = s_w_gu;
    pr.mode = int32_t(mode);
    pr.reserved = 0;
    pr.N = 2 * I;
    pr.y = h;
    Batch b;
    if ((st = validate_batch(x, M, K, &pr, 1, /*out_kind=*/0, &b)) != BITNET_OK) return st;
    return run_batch(x, nullptr, M, K, b, 0, workspace, workspace_bytes, path,
                     static_cast<cudaStream_t>(stream), /*swiglu=*/true);
}

bitnet_status bitnet_linear_swiglu_hmax(const uint16_t* x, int64_t M, int64_t K,
                                        const uint8_t* packed_gu, const float* s_w_gu,
                                        bitnet_scale_mode mode, int64_t I, uint16_t* h,
                                        uint16_t* hmax, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    if (!h || !hmax) return BITNET_ERR_NULL;
    bitnet_status st = check_n(I);
    if (st != BITNET_OK) return st;
    if (I % kSwigluBlock != 0 || 2 * I >= (int64_t(1) << 31)) return BITNET_ERR_SHAPE;
    if (!aligned(hmax, 2)) return BITNET_ERR_ALIGN;
    bitnet_proj pr;
    pr.packed = packed_gu;
    pr.s_w = s_w_gu;
    pr.mode = int32_t(mode);
    pr.reserved = 0;
    pr.N = 2 * I;
    pr.y = h;
    Batch b;
    if ((st = validate_batch(x, M, K, &pr, 1, /*out_kind=*/0, &b)) != BITNET_OK) return st;
    return run_batch(x, nullptr, M, K, b, 0, workspace, workspace_bytes, BITNET_PATH_TC,
                     static_cast<cudaStream_t>(stream), /*swiglu=*/true, false, nullptr, hmax);
}

bitnet_status bitnet_linear_hmax(const uint16_t* x, const uint16_t* xmax, int64_t M, int64_t K,
                                 const uint8_t* packed, const float* s_w, bitnet_scale_mode mode,
                                 int64_t N, void* y, bitnet_out_dtype out_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (out_dtype != BITNET_OUT_BF16 && out_dtype != BITNET_OUT_F32) return BITNET_ERR_UNSUPPORTED;
    if (!xmax) return BITNET_ERR_NULL;
    if (!aligned(xmax, 8)) return BITNET_ERR_ALIGN;
    bitnet_proj pr;
    pr.packed = packed;
    pr.s_w = s_w;
    pr.mode = int32_t(mode);
    pr.reserved = 0;
    pr.N = N;
    pr.y = y;
    Batch b;
    bitnet_status st = validate_batch(x, M, K, &pr, 1, int(out_dtype), &b);
    if (st != BITNET_OK) return st;
    return run_batch(x, nullptr, M, K, b, int(out_dtype), workspace, workspace_bytes,
                     BITNET_PATH_TC, static_cast<cudaStream_t>(stream), /*swiglu=*/false, false,
                     xmax, nullptr);
}

bitnet_status bitnet_quant_act_hmax(const uint16_t* x, const uint16_t* xmax, int64_t M,
                                    int64_t K, int8_t* q, float* s_x, void* stream) {
    if (!x || !xmax || !q || !s_x) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (!aligned(x, 16) || !aligned(xmax, 8) || !aligned(q, 16) || !aligned(s_x, 4))
        return BITNET_ERR_ALIGN;
    return from_cuda(launch_quant(x, nullptr, M, K, q, s_x, nullptr, /*permuted=*/0,
                                  static_cast<cudaStream_t>(stream), /*pdl=*/false, nullptr, 0,
                                  nullptr, nullptr, 0, xmax));
}

int64_t bitnet_b3_row_bytes(int64_t K) { return K < 1 ? 0 : b3_row_bytes(K); }

bitnet_status bitnet_pack_ternary_b3(const int8_t* t, int64_t N, int64_t K, uint8_t* packed,
                                     void* stream) {
    if (!t || !packed) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(1, K);
    if (st != BITNET_OK) return st;
    if ((st = check_n(N)) != BITNET_OK) return st;
    if (!aligned(t, 16) || !aligned(packed, 16)) return BITNET_ERR_ALIGN;
    return from_cuda(launch_pack_b3(t, N, K, packed, static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_linear_b3(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_b3,
                               const float* s_w, bitnet_scale_mode mode, int64_t N, void* y,
                               bitnet_out_dtype out_dtype, void* stream) {
    if (!x || !packed_b3 || !s_w || !y) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if ((st = check_n(N)) != BITNET_OK) return st;
    if (M != 1 || K > 16384) return BITNET_ERR_UNSUPPORTED;
    if (mode != BITNET_SCALE_PER_TENSOR && mode != BITNET_SCALE_PER_ROW) return BITNET_ERR_UNSUPPORTED;
    if (out_dtype != BITNET_OUT_BF16 && out_dtype != BITNET_OUT_F32) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(packed_b3, 16) || !aligned(y, 16) || !aligned(s_w, 4))
        return BITNET_ERR_ALIGN;
    GemvParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = x;
    p.K = K;
    p.M = 1;
    p.nproj = 1;
    p.out_kind = int(out_dtype);
    p.total_rows = N;
    p.proj[0].packed = packed_b3;
    p.proj[0].s_w = s_w;
    p.proj[0].y = y;
    p.proj[0].N = N;
    p.proj[0].per_row = mode == BITNET_SCALE_PER_ROW;
    return from_cuda(launch_gemv_gs(p, /*b3=*/true, tc_num_sms(), static_cast<cudaStream_t>(stream),
                                    true));
}

bitnet_status bitnet_act_amax(const uint16_t* x, int64_t M, int64_t K, float* amax, void* stream) {
    if (!x || !amax) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (!aligned(x, 16) || !aligned(amax, 4)) return BITNET_ERR_ALIGN;
    return from_cuda(launch_act_amax(x, M, K, amax, static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_quant_act_amax(const uint16_t* x, int64_t M, int64_t K, const float* amax,
                                    int8_t* q, float* s_x, void* stream) {
    if (!x || !amax || !q || !s_x) return BITNET_ERR_NULL;
    bitnet_status st = check_mk(M, K);
    if (st != BITNET_OK) return st;
    if (M * (K / 8) >= (int64_t(1) << 39)) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(amax, 4) || !aligned(s_x, 4))
        return BITNET_ERR_ALIGN;
    return from_cuda(launch_quant_amax(x, amax, M, K, q, s_x, static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_dequant(const int32_t* acc, int64_t M, int64_t N, const float* s_x,
                             const float* s_w, bitnet_scale_mode mode, void* y,
                             bitnet_out_dtype out_dtype, void* stream) {
    if (!acc || !s_x || !s_w || !y) return BITNET_ERR_NULL;
    if (M < 1 || M >= (int64_t(1) << 31)) return BITNET_ERR_SHAPE;
    bitnet_status st = check_n(N);
    if (st != BITNET_OK) return st;
    if (M * N >= (int64_t(1) << 39)) return BITNET_ERR_UNSUPPORTED;
    if (mode != BITNET_SCALE_PER_TENSOR && mode != BITNET_SCALE_PER_ROW) return BITNET_ERR_UNSUPPORTED;
    if (out_dtype != BITNET_OUT_BF16 && out_dtype != BITNET_OUT_F32) return BITNET_ERR_UNSUPPORTED;
    if (!aligned(acc, 4) || !aligned(s_x, 4) || !aligned(s_w, 4) ||
        !aligned(y, out_dtype == BITNET_OUT_BF16 ? 2 : 4))
        return BITNET_ERR_ALIGN;
    return from_cuda(launch_dequant(acc, M, N, s_x, s_w, mode == BITNET_SCALE_PER_ROW, y,
                                    int(out_dtype), static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_linear_plan(int64_t M, int64_t K, const int64_t* Ns, int32_t nproj,
                                 int32_t swiglu, size_t workspace_bytes, bitnet_path path,
                                 bitnet_plan* plan) {
    if (!Ns || !plan) return BITNET_ERR_NULL;
    if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC &&
        path != BITNET_PATH_MMA)
        return BITNET_ERR_UNSUPPORTED;
    if (swiglu && nproj != 1) return BITNET_ERR_SHAPE;
    // Stand-in addresses (never dereferenced): 256-byte aligned, as a real call's would be.
    static const uintptr_t kFake = uintptr_t(1) << 40;
    const void* fake = reinterpret_cast<const void*>(kFake);
    if (nproj < 1 || nproj > kMaxProj) return BITNET_ERR_SHAPE;
    bitnet_proj pr[kMaxProj];
    for (int i = 0; i < nproj; ++i) {
        pr[i].packed = static_cast<const uint8_t*>(fake);
        pr[i].s_w = static_cast<const float*>(fake);
        pr[i].mode = BITNET_SCALE_PER_TENSOR;
        pr[i].reserved = 0;
        pr[i].N = Ns[i];
        pr[i].y = const_cast<void*>(fake);
    }
    if (swiglu && (Ns[0] % (2 * kSwigluBlock) != 0)) return BITNET_ERR_SHAPE;
    Batch b;
    bitnet_status st = validate_batch(fake, M, K, pr, nproj, /*out_kind=*/0, &b);
    if (st != BITNET_OK) return st;
    Plan pl;
    st = plan_batch(static_cast<const uint16_t*>(fake), nullptr, M, K, b, 0,
                    workspace_bytes ? fake : nullptr, workspace_bytes, path, swiglu != 0, false,
                    &pl);
    if (st != BITNET_OK) return st;
    std::memset(plan, 0, sizeof(*plan));
    plan->kernel = pl.kernel;
    plan->grid = pl.grid;
    plan->tile_tokens = pl.kernel == BITNET_KERNEL_TC ? pl.bn : 0;
    plan->splits = pl.kernel == BITNET_KERNEL_TC ? pl.splits : 0;
    plan->tile_rows = pl.kernel == BITNET_KERNEL_MMA_GEMV ? 16 * pl.rt : 0;
    if (pl.kernel == BITNET_KERNEL_GEMV) {  // 16 warps of rw rows (SwiGLU: rw / 2 pairs) each
        const int rw = gemv_rows_per_warp(pl.gp, tc_num_sms());
        const int64_t units = swiglu ? 16 * (rw / 2) : 16 * rw;
        plan->tile_rows = 16 * rw;
        plan->grid = static_cast<int32_t>((pl.gp.total_rows + units - 1) / units);
    }
    return BITNET_OK;
}

bitnet_status bitnet_check_device_errors(int32_t* flags) {
    if (!flags) return BITNET_ERR_NULL;
    int32_t* dptr = device_error_word();
    if (!dptr) return BITNET_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return BITNET_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, dptr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BITNET_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpy(dptr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return BITNET_ERR_CUDA;
    *flags = v;
    return v ? BITNET_ERR_TIMEOUT : BITNET_OK;
}

const char* bitnet_status_string(bitnet_status status) {
    switch (status) {
        case BITNET_OK: return "ok";
        case BITNET_ERR_NULL: return "null pointer";
        case BITNET_ERR_SHAPE: return "bad shape";
        case BITNET_ERR_ALIGN: return "misaligned pointer";
        case BITNET_ERR_UNSUPPORTED: return "unsupported argument";
        case BITNET_ERR_CUDA: return "CUDA error";
        case BITNET_ERR_TIMEOUT: return "kernel wait timed out";
        case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int32_t bitnet_version(void) { return 100; }

}  // extern "C"
