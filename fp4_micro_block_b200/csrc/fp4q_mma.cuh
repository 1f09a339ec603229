// fp4q_mma.cuh -- block Hadamard rotation on the 5th-generation tensor cores
// (tcgen05), fused with NVFP4 / MXFP4 / dual-scale quantization.
//
// For rotation sizes n <= 128 the rotated tile is a dense product: a tile X of
// 128 rows x 128 columns times B = -2^-f * blockdiag(H_n, ..., H_n) (128 x 128,
// Sylvester order, f = floor(log2(n) / 2); with a random-sign pattern D the
// rows of B change sign, B = -2^-f * D * blockdiag(H_n)).  Every product of a bf16 input with
// +-2^-f is exact and the sums accumulate in fp32 in tensor memory, so the tile
// arrives in TMEM as the negated, (partly) normalised rotation; odd log2(n)
// leaves a factor RN(1/sqrt(2)) for the epilogue.  B's columns come in the
// acc_col order, which puts the two 16-column blocks of a 32-column chunk in
// alternate accumulator columns.  (MR-GPTQ applies the
// Hadamard as a matrix product on the activations; FP4Quant notes the FWHT as
// one of the costs of the format.)
//
// CTA roles (one persistent CTA per SM):
//   warps 0, 2 lane 0 of each streams alternate X tiles by TMA into a ring of
//              kMmaStages stages;
//   warp 1     allocates TMEM; lane 0 issues 8 UMMAs (K = 16 each) per tile
//              into one of G fp32 accumulators (128 columns each; G = 3,
//              the dual format 2: MmaGeo)
//              and commits them to the tile's barriers;
//   warps 3..  G warpgroups of epilogue: warpgroup g takes the CTA's
//              tiles j = g (mod G); thread = one row of the tile
//              (TMEM lane), reading 32 columns at a time with tcgen05.ld and
//              quantizing them in registers (two 16-blocks or one 32-block).
// Every wait is bounded: a wait that runs out sets g_device_error and the role
// stops; the CTA then drains its own copies and MMAs (bounded again) and frees
// its TMEM before it exits.
#pragma once

#include "fp4q_quant.cuh"

namespace fp4q {

// X ring depth: four 32 KiB stages (one n = 512 tile) measured faster than
// five (C5 quantize 79.2 -> 77.7 us, C3 n = 128 18.9 -> 18.1 us) and than
// three (82.4, 18.8 us).
#ifndef FP4Q_MMA_STAGES
#define FP4Q_MMA_STAGES 4
#endif
#ifndef FP4Q_EPI_GROUPS
#define FP4Q_EPI_GROUPS 3
#endif

constexpr int kMmaTile = 128;                         // tile rows = tile columns
constexpr int kMmaStages = FP4Q_MMA_STAGES;           // X ring depth
constexpr int kEpiGroups = FP4Q_EPI_GROUPS;           // epilogue warpgroups = accumulators
constexpr int kTileBytes = kMmaTile * kMmaTile * 2;   // 32 KiB of bf16
constexpr int kHalfBytes = kTileBytes / 2;            // one TMA box: 64 columns x 128 rows

// UMMA instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// M = 128, N = 128 (fields: D format [4,6), A format [7,10), B format [10,13),
// N >> 3 at [17,23), M >> 4 at [24,29)).
constexpr uint32_t kIdescBf16M128N128 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kMmaTile >> 3) << 17) | ((uint32_t)(kMmaTile >> 4) << 24);

// Shared-memory matrix descriptor of a K-major operand stored as rows of 128
// bytes with the 128-byte swizzle, 8-row groups 1024 bytes apart: start address
// >> 4 at [0,14), leading byte offset 16 >> 4 at [16,30) (unused by this
// swizzle), stride byte offset 1024 >> 4 at [32,46), descriptor version 1 at
// [46,48), layout "128-byte swizzle" (2) at [61,64).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// ---------------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t slot_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// The barrier receives one arrival when every tcgen05 operation this thread
// issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, M = N = 128, K = 16.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (shape 32x32b, x32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    // The wait takes the destination registers as operands, so no use of them
    // can be scheduled before the asynchronous load has completed.
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
          "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
          "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
          "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}



// ---------------------------------------------------------------- shared memory
// [B 32 KiB][X ring kMmaStages x 32 KiB][barriers][tmem slot][NVFP4 table][reduction]
constexpr int kMmaBOff = 0;
constexpr int kMmaRingOff = kTileBytes;
constexpr int kMmaBarOff = kMmaRingOff + kMmaStages * kTileBytes;

// Epilogue warpgroups (= TMEM accumulators), threads and shared-memory layout
// per format.  The dual format's two passes over a tile (group maximum, then
// the quantization) need more registers per thread: it runs two epilogue
// warpgroups, within the register file without spills, instead of three.
template <int FMT>
struct MmaGeo {
    static constexpr int groups = FMT == FMT_DUAL ? 2 : kEpiGroups;
    static constexpr int threads = 96 + 128 * groups;  // 2 producer warps, the MMA warp, epilogue
    static constexpr uint32_t tmem_cols = groups * kMmaTile <= 128 ? 128u : groups * kMmaTile <= 256 ? 256u : 512u;
    static constexpr int num_bars = 2 * kMmaStages + 2 * groups + 1;
    static constexpr int slot_off = kMmaBarOff + num_bars * 8;
    static constexpr int tab_off = (slot_off + 4 + 15) / 16 * 16;
    static constexpr int red_off = tab_off + 128 * 16;
    // codes staging for the TMA stores: per epilogue warpgroup two boxes of
    // 128 rows x 64 bytes (one tile's codes, 64-byte swizzle)
    static constexpr int box_bytes = kMmaTile * 64;
    static constexpr int stg_off = (red_off + (threads / 32) * 4 + 1023) / 1024 * 1024;
    static constexpr int smem = 1024 + stg_off + groups * 2 * box_bytes;
    static_assert(groups * kMmaTile <= 512, "accumulators exceed TMEM");
    static_assert(smem <= 227 * 1024, "shared memory");
};

// Output column held by accumulator column j.  Within each 32-column chunk,
// accumulator columns 2i and 2i+1 hold output columns i and 16 + i, so that a
// 32-column TMEM load lands the quantizer's pairs (one column of each 16-column
// block) in adjacent registers.
__host__ __device__ constexpr int acc_col(int j) { return (j & ~31) | ((j & 1) << 4) | ((j >> 1) & 15); }

// B = -2^-f * blockdiag(H_n) in the K-major 128-byte-swizzled layout of the
// tile: element (row nn, column k) of half h = k / 64 lives at byte
// h * 16 KiB + nn * 128 + ((k % 64) / 8 ^ nn % 8) * 16 + (k % 8) * 2; row nn
// holds the Hadamard entries of output column acc_col(nn).
// Sign bit of tile column k (0..127) for a sign pattern of period min(n, 128).
__device__ __forceinline__ uint32_t sign_bit(const uint32_t (&signs)[4], int k) {
    return (signs[(k >> 5) & 3] >> (k & 31)) & 1u;
}

// With signs, B = -2^-f * D * blockdiag(H_n) (D = diag of the +-1 pattern):
// entry (k, oc) changes sign where channel k of the period is negated.
template <int HAD>
__device__ __forceinline__ void build_hadamard_b(uint8_t* b, const uint32_t (&signs)[4]) {
    constexpr int lg = HAD == 16 ? 4 : HAD == 32 ? 5 : HAD == 64 ? 6 : 7;
    const uint32_t mag = 0x3f80u - (uint32_t)(lg / 2) * 0x80u;  // bf16 bits of 2^-f
    for (int chunk = threadIdx.x; chunk < kTileBytes / 16; chunk += blockDim.x) {
        const int h = chunk / 1024, nn = (chunk / 8) % 128, cp = chunk % 8;  // physical chunk cp
        const int c = cp ^ (nn & 7);                                          // logical 16-byte chunk
        const int oc = acc_col(nn);  // B row nn (accumulator column nn) is output column oc
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            uint32_t pair = 0;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int k = h * 64 + c * 8 + e + t;
                uint32_t bits = 0;
                if (k / HAD == oc / HAD) {
                    const int par = __popc((uint32_t)((k % HAD) & (oc % HAD))) & 1;
                    bits = mag | (par ? 0u : 0x8000u);  // -(+-1) * 2^-f
                    bits ^= sign_bit(signs, k % HAD) << 15;
                }
                pair |= bits << (16 * t);
            }
            w[e / 2] = pair;
        }
        *reinterpret_cast<uint4*>(b + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

struct MmaParams {
    int64_t M, K;
    int64_t n_ct, n_tiles;       // column tiles per row band, tiles
    uint8_t* codes;
    uint8_t* scales;
    float* scale_fp32;
    float* partials;
    int n_partials;
    int swizzled;
    int dynamic;
    uint32_t signs[4];           // random-sign rotation: bit j negates input channel j of every
                                 // min(n, 128) channels (all zero: the plain rotation)
};

// Quantize the 32 values of one chunk (negated pairs n): codes into w, returns
// the scale bytes of the chunk (NVFP4 / dual: two, MXFP4: one).
template <int FMT>
__device__ __forceinline__ uint32_t quant_chunk(const float2* n, const ScaleCtx& ctx, const float4* tab,
                                                float fold, uint32_t (&w)[4]) {
    if constexpr (FMT == FMT_MXFP4) {
        return mxfp4_unit(n, fold, w);
    } else {
        const float2 am = amax_pair(n);
        return nvfp4_unit<FMT == FMT_NVFP4, false>(n, am, ctx, tab, fold, w);
    }
}

// Stores the codes of two adjacent 16-byte chunks (wa: chunk c, wb: chunk c + 1)
// of the rows held by a lane pair (2i, 2i + 1; lane = row): the two lanes swap
// halves so that each store instruction writes whole 32-byte sectors (16 rows
// x 32 bytes) instead of 16-byte halves of 32 rows.  mine = this lane's row at
// chunk c; stride = bytes between rows; live_even / live_odd: the pair's rows
// exist.  Every lane of the warp must call it.
__device__ __forceinline__ void store_chunk_pair(uint8_t* mine, int64_t stride, bool live_even, bool live_odd,
                                                 uint32_t lane, const uint32_t (&wa)[4], const uint32_t (&wb)[4]) {
    const bool odd = lane & 1u;
    uint32_t d1[4], d2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t got = __shfl_xor_sync(0xffffffffu, odd ? wa[k] : wb[k], 1);
        d1[k] = odd ? got : wa[k];  // row 2i: chunk c (even lane), c + 1 (odd lane)
        d2[k] = odd ? wb[k] : got;  // row 2i + 1
    }
    uint8_t* p1 = mine - (odd ? stride : 0) + (odd ? 16 : 0);
    if (live_even) *reinterpret_cast<uint4*>(p1) = make_uint4(d1[0], d1[1], d1[2], d1[3]);
    if (live_odd) *reinterpret_cast<uint4*>(p1 + stride) = make_uint4(d2[0], d2[1], d2[2], d2[3]);
}

template <int FMT, int HAD, bool AMAX_ONLY>
__global__ void __launch_bounds__(MmaGeo<FMT>::threads, 1)
    had_mma_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap codes_map,
                   const MmaParams p) {
    using Geo = MmaGeo<FMT>;
    constexpr int kGroups = Geo::groups;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<1024>(smem_raw);
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kMmaBarOff);
    const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kMmaStages;
    const uint32_t accf0 = empty0 + 8 * kMmaStages, acce0 = accf0 + 8 * kGroups;
    const uint32_t done_bar = acce0 + 8 * kGroups;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Geo::slot_off);
    float4* tab = reinterpret_cast<float4*>(smem + Geo::tab_off);
    float* red = reinterpret_cast<float*>(smem + Geo::red_off);
    constexpr bool kOddLog = HAD == 32 || HAD == 128;  // RN(1/sqrt(2)) left for the epilogue

    if (tid == 0) {
        prefetch_tmap(&tmap_x);
        if constexpr (!AMAX_ONLY) prefetch_tmap(&codes_map);
        for (int s = 0; s < kMmaStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(accf0 + 8 * g, 1);
            mbar_init(acce0 + 8 * g, 4);  // one arrival per epilogue warp
        }
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Geo::tmem_cols);
        tmem_relinquish();
    }
    build_hadamard_b<HAD>(smem + kMmaBOff, p.signs);
    fence_proxy_async_smem();  // B is read by the tensor cores (async proxy)
    pdl_wait();
    pdl_trigger();
    float s_t = 0.0f;
    if constexpr (FMT == FMT_NVFP4 && !AMAX_ONLY) {
        if (p.dynamic) {
            s_t = tensor_scale_from_partials(p.partials, p.n_partials, red);
            if (blockIdx.x == 0 && tid == 0) *p.scale_fp32 = s_t;
        } else {
            s_t = *p.scale_fp32;
        }
        build_table(tab, s_t);
    }
    if constexpr (FMT == FMT_DUAL && !AMAX_ONLY) build_table(tab, 1.0f);  // per-group s: RN(1/E4M3(e))
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t n_my = p.n_tiles > (int64_t)blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    float my_amax = 0.0f;

    if (warp == 0 || warp == 2) {
        // ------------------------------------------------ TMA producers
        // Two warps issue alternate tiles: the copies of one issuing thread are
        // handled one after the other, and two streams of 16 KiB boxes keep an
        // SM's share of HBM bandwidth busy where one does not.
        if (lane == 0) {
            const int64_t pj = warp >> 1;
            int64_t j = pj;
            for (; j < n_my; j += 2) {
                const int s = (int)(j % kMmaStages);
                if (j >= kMmaStages &&
                    !mbar_wait(empty0 + 8 * s, (uint32_t)((j / kMmaStages - 1) & 1))) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                const int64_t t = blockIdx.x + j * gridDim.x;
                const int32_t x0 = (int32_t)((t % p.n_ct) * kMmaTile), y0 = (int32_t)((t / p.n_ct) * kMmaTile);
                const uint32_t dst = smem_u32(smem + kMmaRingOff + s * kTileBytes);
                mbar_arrive_expect_tx(full0 + 8 * s, kTileBytes);
                tma_load_2d(dst, &tmap_x, x0, y0, full0 + 8 * s);
                tma_load_2d(dst + kHalfBytes, &tmap_x, x0 + 64, y0, full0 + 8 * s);
            }
            // Every issued copy must have landed before the CTA may exit: the
            // MMA warp waited for all of them unless something ran out.
            for (int64_t k = pj; k < j; k += 2)
                if (k + kMmaStages >= j)
                    (void)mbar_wait(full0 + 8 * (int)(k % kMmaStages), (uint32_t)((k / kMmaStages) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t b_addr = smem_u32(smem + kMmaBOff);
            for (int64_t j = 0; j < n_my; ++j) {
                const int s = (int)(j % kMmaStages), a = (int)(j % kGroups);
                bool ok = mbar_wait(full0 + 8 * s, (uint32_t)((j / kMmaStages) & 1));
                if (ok && j >= kGroups)
                    ok = mbar_wait(acce0 + 8 * a, (uint32_t)((j / kGroups - 1) & 1));
                if (!ok) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + kMmaRingOff + s * kTileBytes);
                const uint32_t d = tmem_base + (uint32_t)(a * kMmaTile);
#pragma unroll
                for (int k = 0; k < kMmaTile / 16; ++k) {
                    const uint32_t off = (uint32_t)((k / 4) * kHalfBytes + (k % 4) * 32);
                    umma_bf16(d, sw128_desc(a_addr + off), sw128_desc(b_addr + off), kIdescBf16M128N128,
                              k > 0 ? 1u : 0u);
                }
                tc_commit(empty0 + 8 * s);
                tc_commit(accf0 + 8 * a);
            }
            // all MMAs of this CTA complete before TMEM is freed
            tc_commit(done_bar);
            if (!mbar_wait(done_bar, 0)) atomicOr(&g_device_error, kErrWaitTimeout);
        }
    } else {
        // ------------------------------------------------ epilogue
        const uint32_t ew = warp - 3, g = ew / 4, quarter = warp & 3;
        const uint32_t lane_base = (quarter * 32u) << 16;
        ScaleCtx ctx = make_ctx(s_t);
        // odd log2 n: the remaining RN(1/sqrt 2) is applied per block by the quantizer
        const float fold = kOddLog ? __uint_as_float(0x3f3504f3u) : 1.0f;
        // The warpgroup's four warps vote at every accumulator wait (named
        // barrier 1 + g), so an exit is joint; each tile's codes go through one
        // of the warpgroup's two staging boxes and a TMA store by its first thread.
        const bool issuer = (ew & 3u) == 0 && lane == 0;
        const uint32_t bar_id = 1u + g;
        const uint32_t stg_g = smem_u32(smem + Geo::stg_off) + g * 2u * Geo::box_bytes;
        const uint32_t rt_ = quarter * 32u + lane, sw = (rt_ >> 1) & 3u;  // row of the tile, its swizzle
#pragma unroll 1
        for (int64_t j = g; j < n_my; j += kGroups) {
            // the store issued from this box two tiles ago has read it
            if constexpr (!AMAX_ONLY) {
                if (issuer) bulk_wait_read1();
            }
            const bool ok = mbar_wait(accf0 + 8 * g, (uint32_t)((j / kGroups) & 1));
            if (!bar_and((int)bar_id, 128, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            tc_fence_after();
            const int64_t t = blockIdx.x + j * gridDim.x;
            const int64_t ct = t % p.n_ct, rt = t / p.n_ct;
            const int64_t row = rt * kMmaTile + quarter * 32 + lane;
            const bool live = row < p.M;
            const uint32_t tacc = tmem_base + lane_base + g * kMmaTile;

            auto load_chunk = [&](int c, float2* n) {
                float v[32];
                tmem_ld32(tacc + 32u * c, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) n[i] = make_float2(v[2 * i], v[2 * i + 1]);
            };
            auto release = [&]() {  // every lane's loads of this accumulator are done
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce0 + 8 * g);
            };

            if constexpr (AMAX_ONLY) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(tacc + 32u * c, v);
                    if (c == 3) release();
                    float m0 = fmaxf(fabsf(v[0]), fabsf(v[1]));
#pragma unroll
                    for (int i = 2; i < 32; i += 2) m0 = max3(m0, fabsf(v[i]), fabsf(v[i + 1]));
                    m0 *= fold;  // RN is monotone: the max of the scaled values
                    const float2 am = make_float2(m0, m0);
                    if (live) my_amax = fmaxf(my_amax, fmaxf(am.x, am.y));
                    pin(my_amax);
                }
            } else {
                if constexpr (FMT == FMT_DUAL) {  // group scale: amax over the 128 columns
                    float gm = 0.0f;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        float2 n[16];
                        load_chunk(c, n);
                        const float2 am = amax_pair(n);
                        gm = fmaxf(gm, fmaxf(am.x, am.y));
                        pin(gm);
                    }
                    gm *= fold;
                    const float Gs = (gm >= 0x1p-90f) ? div_split(-gm, 2688.0f, rcp2688()) : __fdiv_rn(gm, 2688.0f);
                    ctx = make_ctx(Gs);
                    if (live) p.scale_fp32[row * (p.K / 128) + ct] = Gs;
                }
                const uint32_t box = stg_g + (uint32_t)((j / kGroups) & 1) * Geo::box_bytes + rt_ * 64u;
                uint32_t sc0 = 0u, sc1 = 0u;  // scale bytes of blocks 0-3 / 4-7 (MXFP4: sc0)
#pragma unroll 1
                for (int c = 0; c < 4; c += 2) {
                    uint32_t wa[4], wb[4];
                    float2 n[16];
                    load_chunk(c, n);
                    const uint32_t ea = quant_chunk<FMT>(n, ctx, tab, fold, wa);
                    load_chunk(c + 1, n);
                    if (c + 1 == 3) release();
                    const uint32_t eb = quant_chunk<FMT>(n, ctx, tab, fold, wb);
                    // 16-byte chunks c and c + 1 of the row's 64 bytes, swizzled
                    sts_v4(box + (((uint32_t)c ^ sw) << 4), wa[0], wa[1], wa[2], wa[3]);
                    sts_v4(box + (((uint32_t)(c + 1) ^ sw) << 4), wb[0], wb[1], wb[2], wb[3]);
                    if constexpr (FMT == FMT_MXFP4) {
                        sc0 |= (ea | (eb << 8)) << (8 * c);
                    } else {
                        if (c == 0) sc0 = ea | (eb << 16);
                        else sc1 = ea | (eb << 16);
                    }
                }
                if (live) {
                    if constexpr (FMT == FMT_MXFP4) {
                        const int64_t nsc = p.K / 32;
                        uint8_t* sp = p.swizzled ? p.scales + swizzle_offset(row, ct * 4, (nsc + 3) / 4)
                                                 : p.scales + row * nsc + ct * 4;
                        *reinterpret_cast<uint32_t*>(sp) = sc0;
                    } else {
                        const int64_t nsc = p.K / 16;
                        if (p.swizzled) {
                            const int64_t nC = (nsc + 3) / 4;
                            *reinterpret_cast<uint32_t*>(p.scales + swizzle_offset(row, ct * 8, nC)) = sc0;
                            *reinterpret_cast<uint32_t*>(p.scales + swizzle_offset(row, ct * 8 + 4, nC)) = sc1;
                        } else {
                            uint32_t* sp = reinterpret_cast<uint32_t*>(p.scales + row * nsc + ct * 8);
                            sp[0] = sc0;
                            sp[1] = sc1;
                        }
                    }
                }
                // the tile's codes are in the box: its first thread stores them
                // (rows past M are clipped by the map)
                fence_proxy_async_smem();
                bar_sync((int)bar_id, 128);
                if (issuer) {
                    tma_store_2d(&codes_map, (int32_t)(ct * (kMmaTile / 2)), (int32_t)(rt * kMmaTile),
                                 stg_g + (uint32_t)((j / kGroups) & 1) * Geo::box_bytes);
                    bulk_commit();
                }
            }
        }
        if constexpr (!AMAX_ONLY) {
            if (issuer) bulk_wait0();  // every store has completed before the CTA exits
        }
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_amax = fmaxf(my_amax, __shfl_xor_sync(0xffffffffu, my_amax, o));
        if (lane == 0) red[warp] = my_amax;
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (AMAX_ONLY) {
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < Geo::threads / 32; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Geo::tmem_cols);
    }
}

}  // namespace fp4q
