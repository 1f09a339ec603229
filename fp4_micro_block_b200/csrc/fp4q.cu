// fp4q.cu -- the extern "C" boundary of the quantizer library: host-side
// argument validation, TMA descriptor encoding and kernel launches.  All
// arithmetic runs in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <type_traits>
#include <utility>

#include "../../include/fp4q.h"
#include "fp4q_arc.cuh"
#include "fp4q_dequant.cuh"
#include "fp4q_dqmma.cuh"
#include "fp4q_device.cuh"
#include "fp4q_gemm.cuh"
#include "fp4q_mma.cuh"
#include "fp4q_mma_wide.cuh"
#include "fp4q_quant.cuh"

#define FP4Q_API extern "C" __attribute__((visibility("default")))

namespace {

using namespace fp4q;

constexpr int kMaxGrid = 4096;  // partial maxima fit FP4Q_WORKSPACE_BYTES
static_assert(kMaxGrid * sizeof(float) <= FP4Q_WORKSPACE_BYTES, "workspace too small");

// ---------------------------------------------------------------- device info
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

fp4q_status sm_count(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERR_UNSUPPORTED;
    int n = g_sm_count[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FP4Q_ERR_CUDA;
        g_sm_count[dev].store(n, std::memory_order_relaxed);
    }
    *out = n;
    return FP4Q_OK;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::atomic<EncodeTiledFn> g_encode{nullptr};

fp4q_status encode_fn(EncodeTiledFn* out) {
    EncodeTiledFn fn = g_encode.load(std::memory_order_acquire);
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return FP4Q_ERR_CUDA;
        fn = reinterpret_cast<EncodeTiledFn>(p);
        g_encode.store(fn, std::memory_order_release);
    }
    *out = fn;
    return FP4Q_OK;
}

// bf16 [M, K] with row stride ldx elements; boxes of 64 columns x box_rows rows
// (8: the G2 warp-tile halves; 128: the tensor-core tile halves), 128-byte
// swizzle, zero fill outside the matrix.
fp4q_status make_x_map(CUtensorMap* map, const void* x, int64_t M, int64_t K, int64_t ldx,
                       uint32_t box_rows = 8) {
    EncodeTiledFn enc;
    fp4q_status st = encode_fn(&enc);
    if (st != FP4Q_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4Q_OK : FP4Q_ERR_CUDA;
}

#ifdef FP4Q_TEST_HOOKS
// Test build only: index of a tile that CTA 0 of the next register-path
// quantizer launch does not issue (-1: none); consumed by that launch.
std::atomic<int64_t> g_test_skip_tile{-1};
#endif

// uint8 [rows, row_bytes] (packed E2M1 codes), boxes of 128 bytes x box_rows
// rows with the 128-byte swizzle, zero fill outside the matrix.
fp4q_status make_codes_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t row_bytes,
                           uint32_t box_rows) {
    EncodeTiledFn enc;
    fp4q_status st = encode_fn(&enc);
    if (st != FP4Q_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4Q_OK : FP4Q_ERR_CUDA;
}

// Row-major [rows, cols] of 1-byte or 4-byte elements (row stride row_bytes, a
// multiple of 16), boxes of box_cols x box_rows, no swizzle, zero fill outside.
fp4q_status make_plain_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, int64_t rows, int64_t cols,
                           int64_t row_bytes, uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn enc;
    fp4q_status st = encode_fn(&enc);
    if (st != FP4Q_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4Q_OK : FP4Q_ERR_CUDA;
}

// Packed codes [rows, row_bytes] written by TMA stores of box_bytes x 128 rows
// (64-byte boxes with the 64-byte swizzle, 128-byte boxes with the 128-byte
// one); rows past `rows` are not written.
fp4q_status make_codes_store_map(CUtensorMap* map, void* codes, int64_t rows, int64_t row_bytes,
                                 uint32_t box_bytes) {
    EncodeTiledFn enc;
    fp4q_status st = encode_fn(&enc);
    if (st != FP4Q_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_bytes, 128u};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4Q_OK : FP4Q_ERR_CUDA;
}

// bf16 [rows, cols] output (row stride cols * 2 bytes, a multiple of 16) stored
// by the TMA in boxes of 32 columns x 128 rows with the 64-byte swizzle; rows
// past `rows` are not written.
fp4q_status make_bf16_store_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn enc;
    fp4q_status st = encode_fn(&enc);
    if (st != FP4Q_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {32u, 128u};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4Q_OK : FP4Q_ERR_CUDA;
}

// ---------------------------------------------------------------- validation
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

constexpr int64_t kMaxDim = (int64_t)1 << 31;

fp4q_status check_x(const void* x, int64_t M, int64_t K, int64_t ldx) {
    if (M < 0 || K <= 0 || ldx < K) return FP4Q_ERR_INVALID_ARG;
    if (M >= kMaxDim || K >= kMaxDim || ldx >= kMaxDim) return FP4Q_ERR_UNSUPPORTED;
    if (K < 64) return FP4Q_ERR_UNSUPPORTED;
    if (M > 0 && !x) return FP4Q_ERR_INVALID_ARG;
    if (ldx % 8 != 0 || !aligned(x, 16)) return FP4Q_ERR_ALIGNMENT;
    return FP4Q_OK;
}

fp4q_status check_out(const uint8_t* codes, const uint8_t* scales) {
    if (!codes || !scales) return FP4Q_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 4)) return FP4Q_ERR_ALIGNMENT;
    return FP4Q_OK;
}

bool valid_had(int n) {
    return n == 0 || n == 16 || n == 32 || n == 64 || n == 128 || n == 256 || n == 512;
}

// Launches kern on stream s with programmatic stream serialization, so the
// kernel's prologue may overlap the end of the previous kernel in the stream
// (each kernel waits in pdl_wait() before it touches global memory).
template <typename... KArgs, typename... Args>
fp4q_status launch(void (*kern)(KArgs...), int grid, int threads, int smem, cudaStream_t s, Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA;
}

fp4q_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA;
}

// Raises a kernel's dynamic shared-memory limit once per device (the attribute
// is per function and device; setting it again is harmless but costs host time).
template <typename Kern>
fp4q_status ensure_smem(Kern kern, int bytes, std::atomic<uint64_t>& done) {
    if (bytes <= 48 * 1024) return FP4Q_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return FP4Q_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return FP4Q_OK;
}

// ---------------------------------------------------------------- quantizer launch
// Launches quant_kernel<FMT, HAD, AMAX> persistently (one CTA per SM, at most
// one per tile); returns the grid through *grid_out.
template <int FMT, int HAD, bool AMAX>
fp4q_status launch_quant_t(const CUtensorMap& map, QuantParams p, int sms, cudaStream_t s,
                           int* grid_out) {
    using G = QGeo<FMT, HAD>;
    auto kern = quant_kernel<FMT, HAD, AMAX>;
    static std::atomic<uint64_t> done{0};
    fp4q_status st = ensure_smem(kern, G::smem, done);
    if (st != FP4Q_OK) return st;
    p.n_cs = (p.K + G::tc - 1) / G::tc;
    p.n_tiles = (p.M + kQBoxRows - 1) / kQBoxRows * p.n_cs;
    const int grid = (int)std::min<int64_t>({p.n_tiles, (int64_t)kQCtas * sms, (int64_t)kMaxGrid});
    st = launch(kern, grid, G::threads, G::smem, s, map, p);
    if (grid_out) *grid_out = grid;
    return st;
}

template <int FMT, bool AMAX>
fp4q_status launch_quant_h(int had, const CUtensorMap& map, const QuantParams& p, int sms,
                           cudaStream_t s, int* grid_out) {
    if constexpr (FMT == FMT_DUAL) {  // K % 128 == 0: every rotation takes the tensor cores
        if (had != 0) return FP4Q_ERR_INVALID_ARG;
        return launch_quant_t<FMT, 0, AMAX>(map, p, sms, s, grid_out);
    } else {
        switch (had) {
            case 0: return launch_quant_t<FMT, 0, AMAX>(map, p, sms, s, grid_out);
            case 16: return launch_quant_t<FMT, 16, AMAX>(map, p, sms, s, grid_out);
            case 32: return launch_quant_t<FMT, 32, AMAX>(map, p, sms, s, grid_out);
            case 64: return launch_quant_t<FMT, 64, AMAX>(map, p, sms, s, grid_out);
            default: return FP4Q_ERR_INVALID_ARG;  // 128 and up: tensor cores (K % 128 == 0)
        }
    }
}

float had_norm(int n) { return n > 0 ? (float)(1.0 / std::sqrt((double)n)) : 1.0f; }

// ---------------------------------------------------------------- tensor-core rotation launch
// Rotations on K a multiple of the 128-column tile go through the tcgen05
// kernels (sizes 16..128: one UMMA tile per block group; 256, 512: H_128 on
// the tensor cores and the cross-group butterfly in the epilogue); other
// shapes use the register-FWHT warp pipelines.
#ifndef FP4Q_REGISTER_FWHT_MAX
#define FP4Q_REGISTER_FWHT_MAX 0  // rotations up to this size take the register path on every K
#endif
bool use_mma(int had, int64_t K) { return had > FP4Q_REGISTER_FWHT_MAX && had >= 16 && K % kMmaTile == 0; }

template <int FMT, int HAD, bool AMAX>
fp4q_status launch_mma_t(const CUtensorMap& map, const MmaParams& p, int grid, cudaStream_t s) {
    static std::atomic<uint64_t> done{0};
    if constexpr (HAD <= kMmaTile) {
        auto kern = had_mma_kernel<FMT, HAD, AMAX>;
        fp4q_status st = ensure_smem(kern, MmaGeo<FMT>::smem, done);
        if (st != FP4Q_OK) return st;
        // the codes go out by TMA stores of 128-row x 64-byte boxes (the amax
        // pre-pass writes none: it gets the input's map as a placeholder)
        CUtensorMap codes_map = map;
        if constexpr (!AMAX)
            if ((st = make_codes_store_map(&codes_map, p.codes, p.M, p.K / 2, 64)) != FP4Q_OK) return st;
        return launch(kern, grid, MmaGeo<FMT>::threads, MmaGeo<FMT>::smem, s, map, codes_map, p);
    } else {
        auto kern = had_mma_wide_kernel<FMT, HAD, AMAX>;
        constexpr int smem = Wide<HAD>::smem;
        fp4q_status st = ensure_smem(kern, smem, done);
        if (st != FP4Q_OK) return st;
        // the codes are written by TMA stores of 128-row x 128-byte boxes (the
        // amax pre-pass writes none: it gets the input's map as a placeholder)
        CUtensorMap codes_map = map;
        if constexpr (!AMAX)
            if ((st = make_codes_store_map(&codes_map, p.codes, p.M, p.K / 2, 128)) != FP4Q_OK) return st;
        return launch(kern, grid, kWideThreads, smem, s, map, codes_map, p);
    }
}

template <int FMT, bool AMAX>
fp4q_status launch_mma_h(int had, const CUtensorMap& map, const MmaParams& p, int grid, cudaStream_t s) {
    switch (had) {
        case 16: return launch_mma_t<FMT, 16, AMAX>(map, p, grid, s);
        case 32: return launch_mma_t<FMT, 32, AMAX>(map, p, grid, s);
        case 64: return launch_mma_t<FMT, 64, AMAX>(map, p, grid, s);
        case 128: return launch_mma_t<FMT, 128, AMAX>(map, p, grid, s);
        case 256: return launch_mma_t<FMT, 256, AMAX>(map, p, grid, s);
        case 512: return launch_mma_t<FMT, 512, AMAX>(map, p, grid, s);
        default: return FP4Q_ERR_INVALID_ARG;
    }
}


// signs (host, may be NULL): the random-sign pattern of a rotation, bit j for
// input channel j of every min(had, 128) channels; tensor-core paths only.
fp4q_status quantize_common(const void* x, int64_t M, int64_t K, int64_t ldx, int had,
                            int fmt, uint8_t* codes, uint8_t* scales, float* scale_fp32,
                            fp4q_tscale_mode mode, fp4q_scale_layout layout, void* ws,
                            size_t ws_bytes, cudaStream_t stream, const uint32_t* signs = nullptr) {
    fp4q_status st = check_x(x, M, K, ldx);
    if (st != FP4Q_OK) return st;
    if (!valid_had(had)) return FP4Q_ERR_INVALID_ARG;
    if (signs && had == 0) return FP4Q_ERR_INVALID_ARG;
    if (signs && !use_mma(had, K)) return FP4Q_ERR_UNSUPPORTED;  // K % 128 != 0: register path
    if (layout != FP4Q_SCALES_LINEAR && layout != FP4Q_SCALES_SWIZZLED) return FP4Q_ERR_INVALID_ARG;
    const int B = fmt == FMT_MXFP4 ? 32 : 16;
    if (K % B != 0 || (had && K % had != 0)) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FMT_DUAL && K % 128 != 0) return FP4Q_ERR_INVALID_ARG;
    const bool dynamic = fmt == FMT_NVFP4 && mode == FP4Q_TSCALE_DYNAMIC;
    if (fmt == FMT_NVFP4 && mode != FP4Q_TSCALE_DYNAMIC && mode != FP4Q_TSCALE_STATIC)
        return FP4Q_ERR_INVALID_ARG;
    if (M == 0) return FP4Q_OK;
    if ((st = check_out(codes, scales)) != FP4Q_OK) return st;
    if (fmt != FMT_MXFP4) {
        if (!scale_fp32) return FP4Q_ERR_INVALID_ARG;
        if (!aligned(scale_fp32, 4)) return FP4Q_ERR_ALIGNMENT;
    }
    if (dynamic) {
        if (!ws) return FP4Q_ERR_INVALID_ARG;
        if (ws_bytes < FP4Q_WORKSPACE_BYTES) return FP4Q_ERR_INVALID_ARG;
        if (!aligned(ws, 4)) return FP4Q_ERR_ALIGNMENT;
    }

    int sms = 0;
    if ((st = sm_count(&sms)) != FP4Q_OK) return st;
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const bool mma = use_mma(had, K);
    if ((st = make_x_map(&map, x, M, K, ldx, mma ? kMmaTile : kQBoxRows)) != FP4Q_OK) return st;

    QuantParams p{};
    p.M = M;
    p.K = K;
    p.codes = codes;
    p.scales = scales;
    p.scale_fp32 = scale_fp32;
    p.partials = static_cast<float*>(ws);
    p.swizzled = layout == FP4Q_SCALES_SWIZZLED;
    p.dynamic = dynamic;
    p.had_norm = had_norm(had);
#ifdef FP4Q_TEST_HOOKS
    p.skip_tile = g_test_skip_tile.exchange(-1);
#endif

    if (p.swizzled) {  // padding rows/columns of the tiled layout read as zero
        const int64_t ncols = K / B;
        const int64_t bytes = fp4q_scales_bytes(M, ncols, FP4Q_SCALES_SWIZZLED);
        if (bytes != M * ncols && cudaMemsetAsync(scales, 0, (size_t)bytes, stream) != cudaSuccess)
            return FP4Q_ERR_CUDA;
    }
    if (mma) {
        MmaParams q{};
        q.M = M;
        q.K = K;
        q.n_ct = K / std::max(had, kMmaTile);
        q.n_tiles = (M + kMmaTile - 1) / kMmaTile * q.n_ct;
        q.codes = codes;
        q.scales = scales;
        q.scale_fp32 = scale_fp32;
        q.partials = static_cast<float*>(ws);
        q.swizzled = p.swizzled;
        q.dynamic = dynamic;
        if (signs)
            for (int w = 0; w < (std::min(had, kMmaTile) + 31) / 32; ++w) q.signs[w] = signs[w];
        const int grid = (int)std::min<int64_t>({q.n_tiles, (int64_t)sms, (int64_t)kMaxGrid});
        if (dynamic) {
            if ((st = launch_mma_h<FMT_NVFP4, true>(had, map, q, grid, stream)) != FP4Q_OK) return st;
            q.n_partials = grid;
        }
        switch (fmt) {
            case FMT_NVFP4: return launch_mma_h<FMT_NVFP4, false>(had, map, q, grid, stream);
            case FMT_MXFP4: return launch_mma_h<FMT_MXFP4, false>(had, map, q, grid, stream);
            case FMT_DUAL: return launch_mma_h<FMT_DUAL, false>(had, map, q, grid, stream);
            default: return FP4Q_ERR_INVALID_ARG;
        }
    }
    if (dynamic) {  // amax pre-pass: one partial maximum per CTA into the workspace
        int grid_a = 0;
        st = launch_quant_h<FMT_NVFP4, true>(had, map, p, sms, stream, &grid_a);
        if (st != FP4Q_OK) return st;
        p.n_partials = grid_a;
    }
    switch (fmt) {
        case FMT_NVFP4: return launch_quant_h<FMT_NVFP4, false>(had, map, p, sms, stream, nullptr);
        case FMT_MXFP4: return launch_quant_h<FMT_MXFP4, false>(had, map, p, sms, stream, nullptr);
        case FMT_DUAL: return launch_quant_h<FMT_DUAL, false>(had, map, p, sms, stream, nullptr);
        default: return FP4Q_ERR_INVALID_ARG;
    }
}

// ---------------------------------------------------------------- dequantizer launch
// The tensor-core dequantizer (NVFP4 and dual, n >= 16): K % 512 == 0, linear
// scales, scale arrays 16-byte aligned (the TMA boxes' bases and row strides).
bool dqm_applies(int fmt, int had, const DequantParams& p) {
    return fmt != FMT_MXFP4 && had >= 16 && p.K % 512 == 0 && !p.swizzled && aligned(p.scales, 16) &&
           (fmt != FMT_DUAL || aligned(p.scale_fp32, 16));
}

template <int FMT, int HAD>
fp4q_status launch_dqm_t(const DequantParams& d, int sms, cudaStream_t s) {
    CUtensorMap codes_map, scales_map, g_map, y_map;
    fp4q_status st;
    if ((st = make_bf16_store_map(&y_map, d.y, d.M, d.K)) != FP4Q_OK) return st;
    if ((st = make_codes_map(&codes_map, d.codes, d.M, d.K / 2, 128)) != FP4Q_OK ||
        (st = make_plain_map(&scales_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, d.scales, d.M, d.K / 16, d.K / 16, 32,
                             128)) != FP4Q_OK)
        return st;
    if constexpr (FMT == FMT_DUAL) {
        if ((st = make_plain_map(&g_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d.scale_fp32, d.M, d.K / 128,
                                 d.K / 128 * 4, 4, 128)) != FP4Q_OK)
            return st;
    } else {
        g_map = scales_map;  // not read
    }
    DqmParams p{};
    p.M = d.M;
    p.K = d.K;
    p.n_ct = d.K / 512;
    p.n_tiles = ((d.M + 127) / 128) * p.n_ct;
    p.scale_fp32 = d.scale_fp32;
    p.had_norm = d.had_norm;
    for (int w = 0; w < 4; ++w) p.signs[w] = d.signs[w];
    auto kern = dequant_mma_kernel<FMT, HAD>;
    static std::atomic<uint64_t> done{0};
    if ((st = ensure_smem(kern, kDqmSmem, done)) != FP4Q_OK) return st;
    const int grid = (int)std::min<int64_t>({p.n_tiles, (int64_t)sms, (int64_t)kMaxGrid});
    return launch(kern, grid, kDqmThreads, kDqmSmem, s, codes_map, scales_map, g_map, y_map, p);
}

template <int FMT>
fp4q_status launch_dqm(int had, const DequantParams& p, int sms, cudaStream_t s) {
    switch (had) {
        case 16: return launch_dqm_t<FMT, 16>(p, sms, s);
        case 32: return launch_dqm_t<FMT, 32>(p, sms, s);
        case 64: return launch_dqm_t<FMT, 64>(p, sms, s);
        case 128: return launch_dqm_t<FMT, 128>(p, sms, s);
        case 256: return launch_dqm_t<FMT, 256>(p, sms, s);
        case 512: return launch_dqm_t<FMT, 512>(p, sms, s);
        default: return FP4Q_ERR_INVALID_ARG;
    }
}

// Rotation sizes 64..512: the TMA-fed kernel when K % 512 == 0, the scales are
// linear and the scale arrays 16-byte aligned (the copies' bases and row
// strides must be), else the kernel that loads codes and scales itself.
template <int FMT, int HAD, bool SIGNED>
fp4q_status launch_dequant_t(const DequantParams& p, int sms, cudaStream_t s) {
    constexpr int kWarps = kThreads / 32;
    const int64_t units = ((p.M + 1) / 2) * p.n_col_tiles;  // (row pair, 512 columns)
    const int grid = (int)std::min<int64_t>({(units + kWarps - 1) / kWarps, (int64_t)kDequantCtasPerSm * sms,
                                            (int64_t)kMaxGrid});
    fp4q_status st;
    if (p.K % kTileCols == 0 && !p.swizzled && aligned(p.scales, 16) &&
        (FMT != FMT_DUAL || aligned(p.scale_fp32, 16))) {
        constexpr int B = FMT == FMT_MXFP4 ? 32 : 16;
        CUtensorMap codes_map, scales_map, g_map;
        if ((st = make_plain_map(&codes_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.codes, p.M, p.K / 2, p.K / 2,
                                 kTileCols / 2, 2)) != FP4Q_OK ||
            (st = make_plain_map(&scales_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.scales, p.M, p.K / B, p.K / B,
                                 kTileCols / B, 2)) != FP4Q_OK)
            return st;
        if constexpr (FMT == FMT_DUAL) {
            if ((st = make_plain_map(&g_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.scale_fp32, p.M, p.K / 128,
                                     p.K / 128 * 4, kTileCols / 128, 2)) != FP4Q_OK)
                return st;
        } else {
            g_map = scales_map;  // not read
        }
        auto kern = dequant_tma_kernel<FMT, HAD, SIGNED>;
        constexpr int smem = kWarps * kDqRingSmem;
        static std::atomic<uint64_t> done{0};
        if ((st = ensure_smem(kern, smem, done)) != FP4Q_OK) return st;
        return launch(kern, grid, kThreads, smem, s, p, codes_map, scales_map, g_map);
    }
    auto kern = dequant_warp_kernel<FMT, HAD, SIGNED>;
    constexpr int smem = kWarps * kDqWarpSmem;
    static std::atomic<uint64_t> done{0};
    if ((st = ensure_smem(kern, smem, done)) != FP4Q_OK) return st;
    return launch(kern, grid, kThreads, smem, s, p);
}

// Rotation sizes 0, 16, 32: the streaming kernel, 4 CTAs of 256 threads per SM.
template <int FMT, int HAD, bool SIGNED>
fp4q_status launch_dequant_stream(const DequantParams& p, int sms, cudaStream_t s) {
    const int64_t units = p.M * ((p.K + 31) / 32);
    const int grid = (int)std::min<int64_t>({(units + kThreads - 1) / kThreads, (int64_t)3 * sms,
                                            (int64_t)kMaxGrid});
    const int w32 = ((reinterpret_cast<uintptr_t>(p.y) & 31) == 0 && (p.K & 15) == 0) ? 1 : 0;
    return launch(dequant_stream_kernel<FMT, HAD, SIGNED>, grid, kThreads, 0, s, p, w32);
}

template <int FMT, bool SIGNED>
fp4q_status launch_dequant_h(int had, const DequantParams& p, int sms, cudaStream_t s) {
    switch (had) {
        case 0:
            if constexpr (SIGNED) return FP4Q_ERR_INVALID_ARG;
            else return launch_dequant_stream<FMT, 0, false>(p, sms, s);
        case 16: return launch_dequant_stream<FMT, 16, SIGNED>(p, sms, s);
        case 32: return launch_dequant_stream<FMT, 32, SIGNED>(p, sms, s);
        case 64: return launch_dequant_t<FMT, 64, SIGNED>(p, sms, s);
        case 128: return launch_dequant_t<FMT, 128, SIGNED>(p, sms, s);
        case 256: return launch_dequant_t<FMT, 256, SIGNED>(p, sms, s);
        case 512: return launch_dequant_t<FMT, 512, SIGNED>(p, sms, s);
        default: return FP4Q_ERR_INVALID_ARG;
    }
}

// ---------------------------------------------------------------- ARC launch
// One ARC kernel instantiation and its shared-memory size.
template <int FMT, bool AMAX_ONLY>
struct ArcKern {
    static constexpr void (*fn)(const ArcParams) = arc_kernel<FMT, AMAX_ONLY>;
    static constexpr int wpp = arc_warps_per_pair<FMT, AMAX_ONLY>();
    static constexpr int max_warps = arc_max_warps<FMT, AMAX_ONLY>();
    static int total(int64_t K, int64_t S, int warps) { return arc_layout<AMAX_ONLY>(K, S, warps / wpp).total; }
};

// ---------------------------------------------------------------- self-test kernel
__global__ void selftest_div_kernel(const float* x, const float* d, int64_t n, float* qf,
                                    float* qi) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float dv = d[i], xv = x[i];
        qi[i] = __fdiv_rn(xv, dv);
        qf[i] = div_fast_ok(dv, fabsf(xv)) ? div_split(-xv, dv, make_rcp(dv)) : __fdiv_rn(xv, dv);
    }
}

}  // namespace

// ---------------------------------------------------------------- allocation-free variant
// Scratch of fp4q_quantize_nvfp4_noalloc: the per-CTA partial maxima of the
// tensor-scale pre-pass, in static device memory instead of a caller-supplied
// workspace.  Every GPU that loads the library keeps these 16 KiB until the
// process exits.  In host code the symbol is only a stand-in; the kernels get
// the device address that cudaGetSymbolAddress returns for the current device.
constexpr int kNoAllocPartials = 4096;
static_assert(kNoAllocPartials >= kMaxGrid, "scratch must hold one partial per pre-pass CTA");
static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartials];

namespace {
std::atomic<float*> g_noalloc_ptr[kMaxDevices];

// Device address of the scratch on the current device.  Outside stream capture
// it is looked up on every call (so a context re-created after
// cudaDeviceReset gets its own address) and cached; while `stream` is
// capturing, the cached address of the last uncaptured call is used.
fp4q_status noalloc_scratch(cudaStream_t stream, float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return FP4Q_ERR_CUDA;
    float* ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (cap == cudaStreamCaptureStatusNone) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_noalloc_partials) != cudaSuccess || !a) return FP4Q_ERR_CUDA;
        ptr = static_cast<float*>(a);
        g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
    }
    if (!ptr) return FP4Q_ERR_CUDA;  // first call made under capture: no address yet
    *out = ptr;
    return FP4Q_OK;
}

// CTAs of the amax pre-pass that fp4q_quantize_nvfp4 launches in DYNAMIC mode
// (one partial maximum each): the register quantizer's grid for NVFP4 without
// rotation, min(tiles, CTAs per SM x SMs, kMaxGrid).
int64_t nvfp4_prepass_grid(int64_t M, int64_t K, int sms) {
    using G = QGeo<FMT_NVFP4, 0>;
    const int64_t tiles = (M + kQBoxRows - 1) / kQBoxRows * ((K + G::tc - 1) / G::tc);
    return std::min<int64_t>({tiles, (int64_t)kQCtas * sms, (int64_t)kMaxGrid});
}
}  // namespace

// ==================================================================== C ABI

FP4Q_API size_t fp4q_workspace_bytes(int64_t M, int64_t K) {
    (void)M;
    (void)K;
    return FP4Q_WORKSPACE_BYTES;
}

FP4Q_API int64_t fp4q_scales_bytes(int64_t M, int64_t ncols, fp4q_scale_layout layout) {
    if (M < 0 || ncols < 0) return -1;
    if (layout == FP4Q_SCALES_LINEAR) return M * ncols;
    if (layout == FP4Q_SCALES_SWIZZLED) return ((M + 127) / 128 * 128) * ((ncols + 3) / 4 * 4);
    return -1;
}

FP4Q_API fp4q_status fp4q_quantize_nvfp4(const void* x, int64_t M, int64_t K, int64_t ldx,
                                         uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                         fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                         void* workspace, size_t workspace_bytes,
                                         fp4q_stream_t stream) {
    return quantize_common(x, M, K, ldx, 0, FMT_NVFP4, codes, scales, tensor_scale, mode, layout,
                           workspace, workspace_bytes, (cudaStream_t)stream);
}

FP4Q_API fp4q_status fp4q_quantize_nvfp4_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx,
                                                 uint8_t* codes, uint8_t* scales,
                                                 float* tensor_scale, fp4q_scale_layout layout,
                                                 fp4q_stream_t stream) {
    fp4q_status st = check_x(x, M, K, ldx);
    if (st != FP4Q_OK) return st;
    if (K % 16 != 0) return FP4Q_ERR_INVALID_ARG;
    if (layout != FP4Q_SCALES_LINEAR && layout != FP4Q_SCALES_SWIZZLED) return FP4Q_ERR_INVALID_ARG;
    if (M == 0) return FP4Q_OK;
    int sms = 0;
    if ((st = sm_count(&sms)) != FP4Q_OK) return st;
    if (nvfp4_prepass_grid(M, K, sms) > kNoAllocPartials) return FP4Q_ERR_UNSUPPORTED;
    float* scratch = nullptr;
    if ((st = noalloc_scratch((cudaStream_t)stream, &scratch)) != FP4Q_OK) return st;
    return quantize_common(x, M, K, ldx, 0, FMT_NVFP4, codes, scales, tensor_scale,
                           FP4Q_TSCALE_DYNAMIC, layout, scratch,
                           (size_t)kNoAllocPartials * sizeof(float), (cudaStream_t)stream);
}

FP4Q_API fp4q_status fp4q_quantize_mxfp4(const void* x, int64_t M, int64_t K, int64_t ldx,
                                         uint8_t* codes, uint8_t* scales,
                                         fp4q_scale_layout layout, fp4q_stream_t stream) {
    return quantize_common(x, M, K, ldx, 0, FMT_MXFP4, codes, scales, nullptr,
                           FP4Q_TSCALE_STATIC, layout, nullptr, 0, (cudaStream_t)stream);
}

FP4Q_API fp4q_status fp4q_hadamard_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                                            int had_size, fp4q_format format, uint8_t* codes,
                                            uint8_t* scales, float* scale_fp32,
                                            fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                            void* workspace, size_t workspace_bytes,
                                            fp4q_stream_t stream) {
    int fmt;
    switch (format) {
        case FP4Q_NVFP4: fmt = FMT_NVFP4; break;
        case FP4Q_MXFP4: fmt = FMT_MXFP4; break;
        case FP4Q_NVFP4_DUAL: fmt = FMT_DUAL; break;
        default: return FP4Q_ERR_INVALID_ARG;
    }
    return quantize_common(x, M, K, ldx, had_size, fmt, codes, scales, scale_fp32, mode, layout,
                           workspace, workspace_bytes, (cudaStream_t)stream);
}

FP4Q_API fp4q_status fp4q_hadamard_quantize_signed(const void* x, int64_t M, int64_t K, int64_t ldx,
                                                   int had_size, const uint32_t* signs,
                                                   fp4q_format format, uint8_t* codes, uint8_t* scales,
                                                   float* scale_fp32, fp4q_tscale_mode mode,
                                                   fp4q_scale_layout layout, void* workspace,
                                                   size_t workspace_bytes, fp4q_stream_t stream) {
    if (!signs) return FP4Q_ERR_INVALID_ARG;
    int fmt;
    switch (format) {
        case FP4Q_NVFP4: fmt = FMT_NVFP4; break;
        case FP4Q_MXFP4: fmt = FMT_MXFP4; break;
        case FP4Q_NVFP4_DUAL: fmt = FMT_DUAL; break;
        default: return FP4Q_ERR_INVALID_ARG;
    }
    return quantize_common(x, M, K, ldx, had_size, fmt, codes, scales, scale_fp32, mode, layout,
                           workspace, workspace_bytes, (cudaStream_t)stream, signs);
}

FP4Q_API fp4q_status fp4q_arc_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                                       const void* gamma, float eps, const int32_t* perm,
                                       const int32_t* outliers, int64_t S, fp4q_format format,
                                       uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                       fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                       void* workspace, size_t workspace_bytes,
                                       fp4q_stream_t stream) {
    fp4q_status st = check_x(x, M, K, ldx);
    if (st != FP4Q_OK) return st;
    if (format != FP4Q_NVFP4 && format != FP4Q_MXFP4 && format != FP4Q_INT4) return FP4Q_ERR_INVALID_ARG;
    const bool mx = format == FP4Q_MXFP4, i4 = format == FP4Q_INT4;
    const int B = mx ? 32 : 16;
    if (K % B != 0 || S < 0 || S % B != 0 || S > K) return FP4Q_ERR_INVALID_ARG;
    if (K > 16384) return FP4Q_ERR_UNSUPPORTED;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return FP4Q_ERR_INVALID_ARG;
    if (!mx && mode != FP4Q_TSCALE_DYNAMIC && mode != FP4Q_TSCALE_STATIC) return FP4Q_ERR_INVALID_ARG;
    if (layout != FP4Q_SCALES_LINEAR && layout != FP4Q_SCALES_SWIZZLED) return FP4Q_ERR_INVALID_ARG;
    if (M == 0) return FP4Q_OK;
    if ((st = check_out(codes, scales)) != FP4Q_OK) return st;
    if (!gamma || !perm || (!mx && !tensor_scale) || (S > 0 && !outliers)) return FP4Q_ERR_INVALID_ARG;
    if (!aligned(gamma, 2) || !aligned(perm, 4) || (!mx && !aligned(tensor_scale, 4)) ||
        (S > 0 && !aligned(outliers, 4)))
        return FP4Q_ERR_ALIGNMENT;
    const bool dynamic = !mx && mode == FP4Q_TSCALE_DYNAMIC;
    if (dynamic && (!workspace || workspace_bytes < FP4Q_WORKSPACE_BYTES)) return FP4Q_ERR_INVALID_ARG;
    if (dynamic && !aligned(workspace, 4)) return FP4Q_ERR_ALIGNMENT;

    int sms = 0;
    if ((st = sm_count(&sms)) != FP4Q_OK) return st;
    ArcParams p{};
    p.M = M;
    p.K = K;
    p.S = S;
    p.perm = perm;
    p.outliers = outliers;
    p.gamma = static_cast<const uint16_t*>(gamma);
    p.x = static_cast<const uint8_t*>(x);
    p.ldx_bytes = ldx * 2;
    p.eps = eps;
    p.codes = codes;
    p.scales = scales;
    p.tensor_scale = tensor_scale;
    p.partials = static_cast<float*>(workspace);
    p.swizzled = layout == FP4Q_SCALES_SWIZZLED;
    p.dynamic = dynamic;
    // Warps per CTA (the kernel's warps per row pair times the pairs): as many pairs as the
    // shared memory holds, up to the kernel's launch bound.
    constexpr int kSmemMax = 227 * 1024;
    auto warps_for = [&](auto kern) -> int {
        using Kn = decltype(kern);
        for (int slots = Kn::max_warps / Kn::wpp; slots >= 1; --slots)
            if (Kn::total(K, S, slots * Kn::wpp) <= kSmemMax) return slots * Kn::wpp;
        return 0;
    };
    const int W = mx ? warps_for(ArcKern<FMT_MXFP4, false>{})
                     : i4 ? warps_for(ArcKern<FMT_INT4, false>{}) : warps_for(ArcKern<FMT_NVFP4, false>{});
    const int Wa = dynamic ? warps_for(ArcKern<FMT_NVFP4, true>{}) : 1;
    if (W == 0 || Wa == 0) return FP4Q_ERR_UNSUPPORTED;
    const int64_t pairs = (M + 1) / 2;
    if (p.swizzled) {
        const int64_t ncols = (K + S) / B;
        const int64_t bytes = fp4q_scales_bytes(M, ncols, FP4Q_SCALES_SWIZZLED);
        if (bytes != M * ncols && cudaMemsetAsync(scales, 0, (size_t)bytes, (cudaStream_t)stream) != cudaSuccess)
            return FP4Q_ERR_CUDA;
    }
    // The shared-memory size depends on K and S, so the attribute is set on every call.
    auto run = [&](auto kern, int warps) -> fp4q_status {
        const int slots = warps / decltype(kern)::wpp;
        const int grid = (int)std::min<int64_t>({(pairs + slots - 1) / slots, (int64_t)sms, (int64_t)kMaxGrid});
        p.warps = warps;
        const int smem = decltype(kern)::total(K, S, warps);
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return FP4Q_ERR_CUDA;
        return launch(kern.fn, grid, 32 * warps, smem, (cudaStream_t)stream, p);
    };
    if (dynamic) {
        const int grid_a = (int)std::min<int64_t>({(pairs + Wa - 1) / Wa, (int64_t)sms, (int64_t)kMaxGrid});
        if ((st = run(ArcKern<FMT_NVFP4, true>{}, Wa)) != FP4Q_OK) return st;
        p.n_partials = grid_a;
    }
    if (mx) return run(ArcKern<FMT_MXFP4, false>{}, W);
    if (i4) return run(ArcKern<FMT_INT4, false>{}, W);
    return run(ArcKern<FMT_NVFP4, false>{}, W);
}

namespace {
fp4q_status dequantize_common(fp4q_format format, const uint8_t* codes, const uint8_t* scales,
                              const float* scale_fp32, int64_t M, int64_t K, fp4q_scale_layout layout,
                              int inv_had_size, const uint32_t* signs, void* y, fp4q_stream_t stream) {
    if (M < 0 || K <= 0) return FP4Q_ERR_INVALID_ARG;
    if (M >= kMaxDim || K >= kMaxDim) return FP4Q_ERR_UNSUPPORTED;
    if (K < 64) return FP4Q_ERR_UNSUPPORTED;
    if (!valid_had(inv_had_size)) return FP4Q_ERR_INVALID_ARG;
    if (signs && inv_had_size == 0) return FP4Q_ERR_INVALID_ARG;
    if (layout != FP4Q_SCALES_LINEAR && layout != FP4Q_SCALES_SWIZZLED) return FP4Q_ERR_INVALID_ARG;
    int fmt;
    switch (format) {
        case FP4Q_NVFP4: fmt = FMT_NVFP4; break;
        case FP4Q_MXFP4: fmt = FMT_MXFP4; break;
        case FP4Q_NVFP4_DUAL: fmt = FMT_DUAL; break;
        case FP4Q_INT4: fmt = FMT_INT4; break;
        default: return FP4Q_ERR_INVALID_ARG;
    }
    const int B = fmt == FMT_MXFP4 ? 32 : 16;
    if (K % B != 0 || (inv_had_size && K % inv_had_size != 0)) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FMT_INT4 && inv_had_size != 0) return FP4Q_ERR_UNSUPPORTED;  // no rotated INT4 path
    if (fmt == FMT_DUAL && K % 128 != 0) return FP4Q_ERR_INVALID_ARG;
    if (M == 0) return FP4Q_OK;
    if (!codes || !scales || !y || (fmt != FMT_MXFP4 && !scale_fp32)) return FP4Q_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(y, 16) || (scale_fp32 && !aligned(scale_fp32, 4)))
        return FP4Q_ERR_ALIGNMENT;
    int sms = 0;
    fp4q_status st;
    if ((st = sm_count(&sms)) != FP4Q_OK) return st;
    DequantParams p{};
    p.M = M;
    p.K = K;
    p.n_col_tiles = (K + kTileCols - 1) / kTileCols;
    p.codes = codes;
    p.scales = scales;
    p.scale_fp32 = scale_fp32;
    p.y = static_cast<uint16_t*>(y);
    p.swizzled = layout == FP4Q_SCALES_SWIZZLED;
    p.had_norm = had_norm(inv_had_size);
    cudaStream_t s = (cudaStream_t)stream;
    if (signs)
        for (int w = 0; w < (std::min(inv_had_size, kMmaTile) + 31) / 32; ++w) p.signs[w] = signs[w];
    if (fmt == FMT_INT4) return launch_dequant_stream<FMT_INT4, 0, false>(p, sms, s);
    if (dqm_applies(fmt, inv_had_size, p))
        return fmt == FMT_DUAL ? launch_dqm<FMT_DUAL>(inv_had_size, p, sms, s)
                               : launch_dqm<FMT_NVFP4>(inv_had_size, p, sms, s);
    if (signs) {
        switch (fmt) {
            case FMT_NVFP4: return launch_dequant_h<FMT_NVFP4, true>(inv_had_size, p, sms, s);
            case FMT_MXFP4: return launch_dequant_h<FMT_MXFP4, true>(inv_had_size, p, sms, s);
            default: return launch_dequant_h<FMT_DUAL, true>(inv_had_size, p, sms, s);
        }
    }
    switch (fmt) {
        case FMT_NVFP4: return launch_dequant_h<FMT_NVFP4, false>(inv_had_size, p, sms, s);
        case FMT_MXFP4: return launch_dequant_h<FMT_MXFP4, false>(inv_had_size, p, sms, s);
        default: return launch_dequant_h<FMT_DUAL, false>(inv_had_size, p, sms, s);
    }
}
}  // namespace

FP4Q_API fp4q_status fp4q_dequantize(fp4q_format format, const uint8_t* codes,
                                     const uint8_t* scales, const float* scale_fp32, int64_t M,
                                     int64_t K, fp4q_scale_layout layout, int inv_had_size,
                                     void* y, fp4q_stream_t stream) {
    return dequantize_common(format, codes, scales, scale_fp32, M, K, layout, inv_had_size, nullptr, y,
                             stream);
}

FP4Q_API fp4q_status fp4q_dequantize_signed(fp4q_format format, const uint8_t* codes,
                                            const uint8_t* scales, const float* scale_fp32, int64_t M,
                                            int64_t K, fp4q_scale_layout layout, int inv_had_size,
                                            const uint32_t* signs, void* y, fp4q_stream_t stream) {
    if (!signs) return FP4Q_ERR_INVALID_ARG;
    return dequantize_common(format, codes, scales, scale_fp32, M, K, layout, inv_had_size, signs, y,
                             stream);
}

FP4Q_API fp4q_status fp4q_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                                     const float* a_scale, const uint8_t* b_codes,
                                     const uint8_t* b_scales, const float* b_scale, int64_t M,
                                     int64_t N, int64_t K, void* d, int d_bf16, fp4q_stream_t stream) {
    if (M < 0 || N <= 0 || K <= 0) return FP4Q_ERR_INVALID_ARG;
    if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim) return FP4Q_ERR_UNSUPPORTED;
    if (K % kGemmBK != 0 || N % kGemmBN != 0) return FP4Q_ERR_UNSUPPORTED;
    if (d_bf16 != 0 && d_bf16 != 1) return FP4Q_ERR_INVALID_ARG;
    if (M == 0) return FP4Q_OK;
    if (!a_codes || !a_scales || !a_scale || !b_codes || !b_scales || !b_scale || !d)
        return FP4Q_ERR_INVALID_ARG;
    if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) || !aligned(b_scales, 16) ||
        !aligned(a_scale, 4) || !aligned(b_scale, 4) || !aligned(d, 16))
        return FP4Q_ERR_ALIGNMENT;
    int sms = 0;
    fp4q_status st;
    if ((st = sm_count(&sms)) != FP4Q_OK) return st;
    CUtensorMap map_a, map_b;
    std::memset(&map_a, 0, sizeof(map_a));
    std::memset(&map_b, 0, sizeof(map_b));
    if ((st = make_codes_map(&map_a, a_codes, M, K / 2, kGemmBM)) != FP4Q_OK) return st;
    if ((st = make_codes_map(&map_b, b_codes, N, K / 2, kGemmBN)) != FP4Q_OK) return st;
    GemmParams p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.a_sf = a_scales;
    p.b_sf = b_scales;
    p.a_scale = a_scale;
    p.b_scale = b_scale;
    p.d = d;
    p.out_bf16 = d_bf16;
    p.n_mt = (M + kGemmBM - 1) / kGemmBM;
    p.n_tiles = p.n_mt * (N / kGemmBN);
    p.sf_nc = K / 64;
    static std::atomic<uint64_t> done{0};
    if ((st = ensure_smem(gemm_nvfp4_kernel, kGemmSmem, done)) != FP4Q_OK) return st;
    const int grid = (int)std::min<int64_t>({p.n_tiles, (int64_t)sms, (int64_t)kMaxGrid});
    return launch(gemm_nvfp4_kernel, grid, kGemmThreads, kGemmSmem, (cudaStream_t)stream, map_a, map_b, p);
}

FP4Q_API const char* fp4q_status_string(fp4q_status status) {
    switch (status) {
        case FP4Q_OK: return "FP4Q_OK";
        case FP4Q_ERR_INVALID_ARG: return "FP4Q_ERR_INVALID_ARG: invalid argument";
        case FP4Q_ERR_UNSUPPORTED: return "FP4Q_ERR_UNSUPPORTED: unsupported size or option";
        case FP4Q_ERR_ALIGNMENT: return "FP4Q_ERR_ALIGNMENT: misaligned pointer or stride";
        case FP4Q_ERR_CUDA: return "FP4Q_ERR_CUDA: CUDA call failed";
        case FP4Q_ERR_DEVICE: return "FP4Q_ERR_DEVICE: device-side wait timed out";
        default: return "FP4Q: unknown status";
    }
}

FP4Q_API int fp4q_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return -1;
    if (v && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
    return (int)v;
}

FP4Q_API fp4q_status fp4q_selftest_div(const float* x, const float* d, int64_t n, float* q_fast,
                                       float* q_ieee, fp4q_stream_t stream) {
    if (n < 0) return FP4Q_ERR_INVALID_ARG;
    if (n == 0) return FP4Q_OK;
    if (!x || !d || !q_fast || !q_ieee) return FP4Q_ERR_INVALID_ARG;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
    selftest_div_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(x, d, n, q_fast, q_ieee);
    return launch_status();
}

#ifdef FP4Q_TEST_HOOKS
// Test build only (not declared in include/fp4q.h): makes CTA 0 of the next
// register-path quantizer launch skip issuing its tile number j, so that the
// consumers' bounded wait for it runs out and the kernel takes its timeout path.
FP4Q_API void fp4q_test_skip_tile(int64_t j) { g_test_skip_tile.store(j); }
#endif
