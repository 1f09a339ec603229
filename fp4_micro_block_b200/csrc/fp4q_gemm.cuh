// fp4q_gemm.cuh -- the consumer of the quantized activations: a block-scaled
// NVFP4 GEMM on the 5th-generation tensor cores (tcgen05, kind::mxf4nvf4 with
// 16-element E4M3 block scales).
//
//   D[m, n] = s_a * s_b * sum_k (E2M1(A[m,k]) * E4M3(SA[m, k/16])) *
//                               (E2M1(B[n,k]) * E4M3(SB[n, k/16]))
//
// A [M, K] is an activation tensor as the quantizers write it (packed codes
// [M, K/2], low nibble = even column; scales in the 128x4 tiled layout; one FP32
// tensor scale), B [N, K] a weight tensor in the same form.  The ARCQuant
// operand [primary K | residual S] is consumed unchanged with K + S in place of
// K and the weights [W | W_S] (ARCQuant summary, Methodologie items 3-4: one
// GEMM over the augmented reduction dimension; MR-GPTQ abstract: kernels that
// consume the quantized activations on B200).
//
// The tiled scale layout is the one the tensor cores read: each 512-byte tile
// (128 rows x 4 scale columns, row r%32 at 16 r bytes, row group (r%128)/32 at
// 4 bytes, column at 1 byte) is one tcgen05.cp of shape 32x128b, broadcast to
// the four 32-lane quarters of tensor memory, where lane l of column c + q then
// holds the four scales of row 32 q + l % 32: the block-scaled MMA reads them
// from there.  A wrong byte order in the layout gives a wrong product.
//
// CTA roles (persistent, one CTA per SM; 6 warps):
//   warp 0 lane 0  streams, per 256-column K step, the A tile (128 rows x 128
//                  bytes) and B tile (256 rows x 128 bytes) by TMA (128-byte
//                  swizzle) and their scale tiles (2 + 4 KiB) by bulk copies
//                  into a ring of kGemmStages stages;
//   warp 1         allocates TMEM; lane 0 copies the scale tiles of a K step
//                  into TMEM (tcgen05.cp) and issues its 4 MMAs (M = 128,
//                  N = 256, K = 64) into the fp32 accumulator;
//   warps 2..5     epilogue: thread = one accumulator row (TMEM lane), 32
//                  columns per tcgen05.ld, times s_a * s_b, stored as fp32 or
//                  bf16.
// Every wait is bounded; a wait that runs out sets g_device_error and the role
// stops; the CTA drains its copies and MMAs and frees TMEM before it exits.
#pragma once

#include "fp4q_mma.cuh"

namespace fp4q {

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 256;  // K in elements (128 bytes)
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = kGemmBM * kGemmBK / 2;         // 16 KiB
constexpr int kGemmBBytes = kGemmBN * kGemmBK / 2;         // 32 KiB
constexpr int kGemmSfaBytes = kGemmBM * kGemmBK / 16;      // 2 KiB: four 512-byte scale tiles
constexpr int kGemmSfbBytes = kGemmBN * kGemmBK / 16;      // 4 KiB
constexpr int kGemmStageBytes = kGemmABytes + kGemmBBytes + kGemmSfaBytes + kGemmSfbBytes;
constexpr int kGemmBarOff = kGemmStages * kGemmStageBytes;
constexpr int kGemmNumBars = 2 * kGemmStages + 3;
constexpr int kGemmSlotOff = kGemmBarOff + kGemmNumBars * 8;
constexpr int kGemmSmem = 1024 + kGemmSlotOff + 16;
constexpr int kGemmThreads = 192;
constexpr uint32_t kGemmTmemCols = 512;  // accumulator 256 + scales 16 (A) + 32 (B)
constexpr uint32_t kGemmSfaCol = 256, kGemmSfbCol = 272;
static_assert(kGemmStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle");
static_assert(kGemmSmem <= 227 * 1024, "shared memory");

// Instruction descriptor of kind::mxf4nvf4 with block scales: A and B E2M1
// (format 1 at [7,10) and [10,13)), both K-major, N >> 3 at [17,23), scale
// format E4M3 (0 at bit 23), M >> 4 at [24,29), scale-factor byte ids 0
// ([4,6) and [29,31)), K = 64 (bit 31 clear).
constexpr uint32_t kIdescNvfp4M128N256 =
    (1u << 7) | (1u << 10) | ((uint32_t)(kGemmBN >> 3) << 17) | ((uint32_t)(kGemmBM >> 4) << 24);

// Shared-memory descriptor of one 512-byte scale tile read by tcgen05.cp as 32
// rows of 16 bytes: no swizzle (layout 0 at [61,64)), 8-row core matrices 128
// bytes apart (stride byte offset at [32,46)), descriptor version 1 at [46,48).
__device__ __forceinline__ uint64_t sf_tile_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(512u >> 4) << 16) |
           ((uint64_t)(128u >> 4) << 32) | ((uint64_t)1u << 46);
}

// 32 rows x 128 bits from shared memory to TMEM columns [taddr, taddr + 4),
// broadcast to the four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A * B^T with E2M1 operands and E4M3 block scales (16 elements).
__device__ __forceinline__ void umma_nvfp4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(
            tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
}

struct GemmParams {
    int64_t M, N, K;
    const uint8_t* a_sf;  // tiled scale layout, rows padded to 128
    const uint8_t* b_sf;
    const float* a_scale;  // FP32 tensor scales (1 float each)
    const float* b_scale;
    void* d;               // [M, N] fp32 or bf16
    int out_bf16;
    int64_t n_mt, n_tiles;  // row tiles of A; tiles (row tile fastest)
    int64_t sf_nc;          // 512-byte scale tiles per 128 rows: K / 64
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<1024>(smem_raw);
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t full0 = smem_u32(smem + kGemmBarOff), empty0 = full0 + 8 * kGemmStages;
    const uint32_t accf = empty0 + 8 * kGemmStages, acce = accf + 8, done_bar = acce + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kGemmSlotOff);

    if (tid == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 4);  // one arrival per epilogue warp
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kGemmTmemCols);
        tmem_relinquish();
    }
    pdl_wait();
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t KT = p.K / kGemmBK;
    const int64_t n_my = p.n_tiles > (int64_t)blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const int64_t total = n_my * KT;
            int64_t g = 0;
            for (; g < total; ++g) {
                const int s = (int)(g % kGemmStages);
                if (g >= kGemmStages && !mbar_wait(empty0 + 8 * s, (uint32_t)((g / kGemmStages - 1) & 1))) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                const int64_t t = blockIdx.x + (g / KT) * gridDim.x, kt = g % KT;
                const int64_t mt = t % p.n_mt, nt = t / p.n_mt;
                uint8_t* st = smem + s * kGemmStageBytes;
                const uint32_t bar = full0 + 8 * s;
                mbar_arrive_expect_tx(bar, kGemmStageBytes);
                tma_load_2d(smem_u32(st), &tmap_a, (int32_t)(kt * (kGemmBK / 2)), (int32_t)(mt * kGemmBM), bar);
                tma_load_2d(smem_u32(st + kGemmABytes), &tmap_b, (int32_t)(kt * (kGemmBK / 2)),
                            (int32_t)(nt * kGemmBN), bar);
                // scale tiles of K step kt: columns 16 kt .. 16 kt + 15 = tiles 4 kt .. 4 kt + 3
                bulk_load_1d(smem_u32(st + kGemmABytes + kGemmBBytes),
                             p.a_sf + (mt * p.sf_nc + 4 * kt) * 512, kGemmSfaBytes, bar);
                bulk_load_1d(smem_u32(st + kGemmABytes + kGemmBBytes + kGemmSfaBytes),
                             p.b_sf + ((2 * nt) * p.sf_nc + 4 * kt) * 512, kGemmSfaBytes, bar);
                bulk_load_1d(smem_u32(st + kGemmABytes + kGemmBBytes + kGemmSfaBytes + kGemmSfaBytes),
                             p.b_sf + ((2 * nt + 1) * p.sf_nc + 4 * kt) * 512, kGemmSfaBytes, bar);
            }
            // every issued copy lands before the CTA may exit
            for (int64_t k = (g > kGemmStages ? g - kGemmStages : 0); k < g; ++k)
                (void)mbar_wait(full0 + 8 * (int)(k % kGemmStages), (uint32_t)((k / kGemmStages) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------ scale copies + MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int64_t i = 0; i < n_my && ok; ++i) {
                if (i > 0 && !mbar_wait(acce, (uint32_t)((i - 1) & 1))) {  // epilogue done with the accumulator
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int64_t kt = 0; kt < KT; ++kt) {
                    const int64_t g = i * KT + kt;
                    const int s = (int)(g % kGemmStages);
                    if (!mbar_wait(full0 + 8 * s, (uint32_t)((g / kGemmStages) & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kGemmStageBytes);
                    const uint32_t sfa = st + kGemmABytes + kGemmBBytes, sfb = sfa + kGemmSfaBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {  // scales of the 4 MMAs (K = 64 each)
                        tmem_cp_32x128b_x4(tmem_base + kGemmSfaCol + 4 * j, sf_tile_desc(sfa + 512 * j));
                        tmem_cp_32x128b_x4(tmem_base + kGemmSfbCol + 8 * j, sf_tile_desc(sfb + 512 * j));
                        tmem_cp_32x128b_x4(tmem_base + kGemmSfbCol + 8 * j + 4,
                                           sf_tile_desc(sfb + kGemmSfaBytes + 512 * j));
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_nvfp4(tmem_base, sw128_desc(st + 32 * j), sw128_desc(st + kGemmABytes + 32 * j),
                                   kIdescNvfp4M128N256, tmem_base + kGemmSfaCol + 4 * j,
                                   tmem_base + kGemmSfbCol + 8 * j, (kt > 0 || j > 0) ? 1u : 0u);
                    tc_commit(empty0 + 8 * s);
                }
                if (!ok) break;
                tc_commit(accf);
            }
            if (!ok) atomicOr(&g_device_error, kErrWaitTimeout);
            // all MMAs of this CTA complete before TMEM is freed
            tc_commit(done_bar);
            if (!mbar_wait(done_bar, 0)) atomicOr(&g_device_error, kErrWaitTimeout);
        }
    } else {
        // ------------------------------------------------ epilogue
        const uint32_t quarter = warp & 3;
        const uint32_t lane_base = (quarter * 32u) << 16;
        const float sab = *p.a_scale * *p.b_scale;
#pragma unroll 1
        for (int64_t i = 0; i < n_my; ++i) {
            const bool ok = mbar_wait(accf, (uint32_t)(i & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            tc_fence_after();
            const int64_t t = blockIdx.x + i * gridDim.x;
            const int64_t mt = t % p.n_mt, nt = t / p.n_mt;
            const int64_t row = mt * kGemmBM + quarter * 32 + lane;
            const bool live = row < p.M;
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 32; ++c) {
                float v[32];
                tmem_ld32(tmem_base + lane_base + 32u * c, v);
                if (!live) continue;
                const int64_t col = nt * kGemmBN + 32 * c;
                if (p.out_bf16) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.d) + row * p.N + col);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(bf16x2_pack(v[8 * q] * sab, v[8 * q + 1] * sab),
                                            bf16x2_pack(v[8 * q + 2] * sab, v[8 * q + 3] * sab),
                                            bf16x2_pack(v[8 * q + 4] * sab, v[8 * q + 5] * sab),
                                            bf16x2_pack(v[8 * q + 6] * sab, v[8 * q + 7] * sab));
                } else {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.d) + row * p.N + col);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(v[4 * q] * sab, v[4 * q + 1] * sab, v[4 * q + 2] * sab,
                                             v[4 * q + 3] * sab);
                }
            }
            // this warp's accumulator reads are done: the next tile may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kGemmTmemCols);
    }
}

}  // namespace fp4q
