// fp4q_dqmma.cuh -- dequantization with the inverse block Hadamard on the
// tensor cores, fed with the packed codes and block scales as they are stored
// (NVFP4 and the dual-scale format; n = 16..512, K % 512 == 0, linear scales).
//
// The block-scaled MMA (kind::mxf4nvf4, 16-element E4M3 scales) multiplies the
// E2M1 codes, each scaled by its block's E4M3 value, with a second E2M1 operand
// at scale 1: with that operand B = D_s * blockdiag(H), entries +-1 (D_s the
// random-sign pattern, identity without one), one 128-column group of a row
// comes out as
//     z[c] = sum_k E2M1(code_k) * E4M3(scale_(k/16)) * B[c][k],
// the rotation of the group's dequantized values without the FP32 scale: the
// products are exact and the tensor cores sum each 64-element K step exactly
// or to one fp32 ulp, then add the two steps in fp32 (measured on B200), so z
// carries about the error of one fp32 rounding.  The epilogue multiplies z by
// the FP32 scale of the row's group (dual) or the tensor scale (NVFP4) and by
// the normalisation 1/sqrt(n), applies the butterfly across the 128-column
// groups of a block (n = 256: H_2, n = 512: H_4 -- Sylvester's H_n factors as
// H_(n/128) (x) H_128, and the FP32 scales, constant over a group, commute with
// H_128), and stores bf16.  (FP4Quant abstract: the receiving side of FP4
// compressed activations; the oracle computes H_n times the dequantized block.)
//
// Tile = 128 rows x 512 columns (four groups); the accumulator of a tile is
// produced in four slices of 32 output columns of every group (M = 128,
// N = 32 per group), three slices in flight in TMEM, so the tensor cores work
// on the next slices while the epilogue drains one.
//
// CTA roles (persistent, one CTA per SM, 3 + 8 warps):
//   warp 0 lane 0  TMA: per tile the codes (two 128-byte-swizzled boxes of
//                  128 rows x 256 codes), the linear scale bytes (128 x 32) and
//                  the group scales (128 x 4, dual) into a ring of stages;
//   warp 1         TMEM allocation; lane 0 copies a tile's scale tiles into
//                  TMEM (tcgen05.cp) and issues its MMAs slice by slice;
//   warp 2         rewrites a tile's linear scale bytes into the 128 x 4 tiled
//                  layout that tcgen05.cp reads (eight 512-byte tiles, one per
//                  64-column K step);
//   warps 3..10    epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (one row
//                  each) and 16 of the 32 columns of every slice (half wg of
//                  warpgroup wg = (w - 3) / 4).
// Every wait is bounded: a wait that runs out sets g_device_error, the role
// stops, and the CTA drains its copies and MMAs before it frees TMEM and exits.
#pragma once

#include "fp4q_gemm.cuh"

namespace fp4q {

constexpr int kDqmStages = 3;                       // TMA ring depth (tiles)
constexpr int kDqmSlots = 3;                        // accumulator slices in TMEM
constexpr int kDqmCodeBytes = 128 * 256;            // 128 rows x 512 codes
constexpr int kDqmScaleBytes = 128 * 32;            // 128 rows x 32 linear scale bytes
constexpr int kDqmGBytes = 128 * 16;                // 128 rows x 4 group scales
constexpr int kDqmStageBytes = kDqmCodeBytes + kDqmScaleBytes + kDqmGBytes;  // 38 KiB
constexpr int kDqmSfBytes = 8 * 512;                // eight tiled scale tiles per tile
constexpr int kDqmBOff = kDqmStages * kDqmStageBytes;  // B: 128 rows x 128 bytes, 16 KiB
constexpr int kDqmSfOff = kDqmBOff + 128 * 128;        // 2 repacked scale buffers
constexpr int kDqmOneOff = kDqmSfOff + 2 * kDqmSfBytes;  // 512 bytes of E4M3 1.0 (scales of B)
constexpr int kDqmBarOff = kDqmOneOff + 512;
constexpr int kDqmNumBars = 2 * kDqmStages + 2 * 2 + 2 * kDqmSlots + 1;
constexpr int kDqmSlotOff = kDqmBarOff + kDqmNumBars * 8;
// bf16 output staging for the TMA stores: two buffers of one slice each, four
// boxes (one per group) of 128 rows x 32 columns with the 64-byte swizzle
constexpr int kDqmBoxBytes = 128 * 64;
constexpr int kDqmStgBytes = 4 * kDqmBoxBytes;
constexpr int kDqmStgOff = (kDqmSlotOff + 16 + 1023) / 1024 * 1024;
constexpr int kDqmSmem = 1024 + kDqmStgOff + 2 * kDqmStgBytes;
// Two epilogue warpgroups, both reading every slice (one half of its columns
// each).  The slice barriers are waited on by phase parity, which is exact only
// while every waiter takes every phase of a slot in turn: a warpgroup that
// skipped the uses of a slot by other warpgroups (slots are reused by slices of
// alternating parity) could see a phase two ahead as complete.
constexpr int kDqmEpiWg = 2;
constexpr int kDqmThreads = 96 + 128 * kDqmEpiWg;      // 3 role warps + the epilogue
constexpr uint32_t kDqmTmemCols = 512;
constexpr uint32_t kDqmSfaCol = 384, kDqmSfbCol = 416;  // after the three 128-column slices
static_assert(kDqmStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle");
static_assert(kDqmSmem <= 227 * 1024, "shared memory");

// kind::mxf4nvf4, E2M1 A and B (K-major), E4M3 block scales, M = 128, N = 32.
constexpr uint32_t kIdescNvfp4M128N32 = (1u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);

struct DqmParams {
    int64_t M, K;
    int64_t n_ct, n_tiles;  // 512-column tiles per row; tiles (column tile fastest)
    const float* scale_fp32;  // NVFP4: the tensor scale (the dual format's come by TMA)
    float had_norm;
    uint32_t signs[4];
};

// B = D_s * blockdiag(H_n) (n <= 128) or D_s * H_128 (n >= 128) as E2M1 codes
// (+1 = 0x2, -1 = 0xA, 0 off the diagonal blocks), in the K-major 128-byte
// swizzled layout: row c (an output column of the group) holds B[c][k] for
// k < 128 in its first 64 bytes and again in its last 64, so that the K steps
// of both groups of a 256-code box read the same B.  The sign pattern (period
// min(n, 128)) negates output column c.
template <int HAD>
__device__ __forceinline__ void build_dqm_b(uint8_t* b, const uint32_t (&signs)[4]) {
    constexpr int nb = HAD < 128 ? HAD : 128;
    for (int chunk = threadIdx.x; chunk < 128 * 8; chunk += blockDim.x) {
        const int c = chunk / 8, pc = chunk % 8;  // row, physical 16-byte chunk
        const int lc = pc ^ (c & 7);              // logical chunk: codes 32 lc .. 32 lc + 31
        const uint32_t neg = sign_bit(signs, c % nb);
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k = (32 * lc + 8 * q + e) % 128;
                uint32_t code = 0;
                if (k / nb == c / nb) {
                    const uint32_t par = (__popc((uint32_t)((k % nb) & (c % nb))) & 1u) ^ neg;
                    code = par ? 0xAu : 0x2u;
                }
                word |= code << (4 * e);
            }
            w[q] = word;
        }
        *reinterpret_cast<uint4*>(b + (c / 8) * 1024 + (c % 8) * 128 + pc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// 16 consecutive fp32 columns of this thread's TMEM lane; the values are valid
// after tmem_wait_ld16x4().
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}
// Keeps the four loads' registers ordered after one wait.
__device__ __forceinline__ void tmem_wait_ld16x4(uint32_t (&r)[4][16]) {
    tmem_wait_ld16(r[0]);
    asm volatile("" : "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[1][4]), "+r"(r[1][5]),
                 "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[1][8]), "+r"(r[1][9]), "+r"(r[1][10]), "+r"(r[1][11]),
                 "+r"(r[1][12]), "+r"(r[1][13]), "+r"(r[1][14]), "+r"(r[1][15]) :: "memory");
    asm volatile("" : "+r"(r[2][0]), "+r"(r[2][1]), "+r"(r[2][2]), "+r"(r[2][3]), "+r"(r[2][4]), "+r"(r[2][5]),
                 "+r"(r[2][6]), "+r"(r[2][7]), "+r"(r[2][8]), "+r"(r[2][9]), "+r"(r[2][10]), "+r"(r[2][11]),
                 "+r"(r[2][12]), "+r"(r[2][13]), "+r"(r[2][14]), "+r"(r[2][15]) :: "memory");
    asm volatile("" : "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3]), "+r"(r[3][4]), "+r"(r[3][5]),
                 "+r"(r[3][6]), "+r"(r[3][7]), "+r"(r[3][8]), "+r"(r[3][9]), "+r"(r[3][10]), "+r"(r[3][11]),
                 "+r"(r[3][12]), "+r"(r[3][13]), "+r"(r[3][14]), "+r"(r[3][15]) :: "memory");
}

template <int FMT, int HAD>
__global__ void __launch_bounds__(kDqmThreads, 1)
    dequant_mma_kernel(const __grid_constant__ CUtensorMap codes_map, const __grid_constant__ CUtensorMap scales_map,
                       const __grid_constant__ CUtensorMap g_map, const __grid_constant__ CUtensorMap y_map,
                       const DqmParams p) {
    static_assert(FMT == FMT_NVFP4 || FMT == FMT_DUAL, "16-element E4M3 block scales");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<1024>(smem_raw);
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t full0 = smem_u32(smem + kDqmBarOff), empty0 = full0 + 8 * kDqmStages;
    const uint32_t sfr0 = empty0 + 8 * kDqmStages, sfe0 = sfr0 + 16;  // [2] repacked / copied out
    const uint32_t accf0 = sfe0 + 16, acce0 = accf0 + 8 * kDqmSlots, done_bar = acce0 + 8 * kDqmSlots;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kDqmSlotOff);
    constexpr uint32_t kTx = kDqmCodeBytes + kDqmScaleBytes + (FMT == FMT_DUAL ? kDqmGBytes : 0);

    if (tid == 0) {
        prefetch_tmap(&codes_map);
        prefetch_tmap(&scales_map);
        if constexpr (FMT == FMT_DUAL) prefetch_tmap(&g_map);
        prefetch_tmap(&y_map);
        for (int s = 0; s < kDqmStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 2 + 4 * kDqmEpiWg);  // the MMAs' commit, the repack warp, the epilogue warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfr0 + 8 * b, 1);
            mbar_init(sfe0 + 8 * b, 1);
        }
        for (int s = 0; s < kDqmSlots; ++s) {
            mbar_init(accf0 + 8 * s, 1);
            mbar_init(acce0 + 8 * s, 8);
        }
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kDqmTmemCols);
        tmem_relinquish();
    }
    build_dqm_b<HAD>(smem + kDqmBOff, p.signs);
    for (int i = tid; i < 512 / 16; i += blockDim.x)  // E4M3 1.0 = 0x38 in every byte
        reinterpret_cast<uint4*>(smem + kDqmOneOff)[i] = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
    fence_proxy_async_smem();
    pdl_wait();
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t n_my = p.n_tiles > (int64_t)blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int64_t i = 0;
            for (; i < n_my; ++i) {
                const int s = (int)(i % kDqmStages);
                if (i >= kDqmStages && !mbar_wait(empty0 + 8 * s, (uint32_t)((i / kDqmStages - 1) & 1))) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                const int64_t t = blockIdx.x + i * gridDim.x;
                const int32_t ct = (int32_t)(t % p.n_ct), y0 = (int32_t)((t / p.n_ct) * 128);
                uint8_t* st = smem + s * kDqmStageBytes;
                const uint32_t bar = full0 + 8 * s;
                mbar_arrive_expect_tx(bar, kTx);
                tma_load_2d(smem_u32(st), &codes_map, ct * 256, y0, bar);
                tma_load_2d(smem_u32(st + kDqmCodeBytes / 2), &codes_map, ct * 256 + 128, y0, bar);
                tma_load_2d(smem_u32(st + kDqmCodeBytes), &scales_map, ct * 32, y0, bar);
                if constexpr (FMT == FMT_DUAL)
                    tma_load_2d(smem_u32(st + kDqmCodeBytes + kDqmScaleBytes), &g_map, ct * 4, y0, bar);
            }
            // every issued copy lands before the CTA may exit
            for (int64_t k = (i > kDqmStages ? i - kDqmStages : 0); k < i; ++k)
                (void)mbar_wait(full0 + 8 * (int)(k % kDqmStages), (uint32_t)((k / kDqmStages) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------ scale copies + MMA issuer
        if (lane == 0) {
            tmem_cp_32x128b_x4(tmem_base + kDqmSfbCol, sf_tile_desc(smem_u32(smem + kDqmOneOff)));
            const uint32_t b_addr = smem_u32(smem + kDqmBOff);
            bool ok = true;
            for (int64_t i = 0; ok && i < n_my; ++i) {
                const int s = (int)(i % kDqmStages), sb = (int)(i & 1);
                ok = mbar_wait(full0 + 8 * s, (uint32_t)((i / kDqmStages) & 1)) &&
                     mbar_wait(sfr0 + 8 * sb, (uint32_t)((i >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                const uint32_t sf = smem_u32(smem + kDqmSfOff + sb * kDqmSfBytes);
#pragma unroll
                for (int k = 0; k < 8; ++k)  // K step k = 64 codes: group k / 2
                    tmem_cp_32x128b_x4(tmem_base + kDqmSfaCol + 4 * k, sf_tile_desc(sf + 512 * k));
                tc_commit(sfe0 + 8 * sb);  // the repacked buffer may be rewritten
                const uint32_t a_addr = smem_u32(smem + s * kDqmStageBytes);
                for (int q = 0; q < 4; ++q) {  // slices of 32 output columns
                    const int64_t j = 4 * i + q;
                    const int slot = (int)(j % kDqmSlots);
                    if (j >= kDqmSlots && !mbar_wait(acce0 + 8 * slot, (uint32_t)((j / kDqmSlots - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t koff = 32u * (uint32_t)(2 * (g & 1) + kk);  // bytes in the 128-byte row
                            umma_nvfp4(tmem_base + (uint32_t)(128 * slot + 32 * g),
                                       sw128_desc(a_addr + (uint32_t)(g >> 1) * (kDqmCodeBytes / 2) + koff),
                                       sw128_desc(b_addr + (uint32_t)(32 * q) * 128u + koff), kIdescNvfp4M128N32,
                                       tmem_base + kDqmSfaCol + 4 * (2 * g + kk), tmem_base + kDqmSfbCol,
                                       kk > 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(accf0 + 8 * slot);
                }
                if (ok) tc_commit(empty0 + 8 * s);
            }
            if (!ok) atomicOr(&g_device_error, kErrWaitTimeout);
            // all tensor-core work of this CTA completes before TMEM is freed
            tc_commit(done_bar);
            if (!mbar_wait(done_bar, 0)) atomicOr(&g_device_error, kErrWaitTimeout);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ scale repack: linear -> tiled
        // tile k (columns 4k .. 4k + 3 of the tile's 32 scale columns) holds at
        // 16 (r % 32) + 4 (r / 32) the four bytes of row r; lane l moves rows
        // l, l + 32, l + 64, l + 96 with one 16-byte store per tile.
        for (int64_t i = 0; i < n_my; ++i) {
            const int s = (int)(i % kDqmStages), sb = (int)(i & 1);
            bool ok = mbar_wait(full0 + 8 * s, (uint32_t)((i / kDqmStages) & 1));
            if (ok && i >= 2) ok = mbar_wait(sfe0 + 8 * sb, (uint32_t)(((i >> 1) - 1) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            const uint8_t* lin = smem + s * kDqmStageBytes + kDqmCodeBytes;
            uint8_t* sf = smem + kDqmSfOff + sb * kDqmSfBytes;
            uint4 w[4][2];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                w[q][0] = *reinterpret_cast<const uint4*>(lin + (32 * q + lane) * 32);
                w[q][1] = *reinterpret_cast<const uint4*>(lin + (32 * q + lane) * 32 + 16);
            }
            auto word = [&](int q, int k) -> uint32_t {
                const uint4& v = w[q][k >> 2];
                const int e = k & 3;
                return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
            };
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(sf + 512 * k + 16 * lane) = make_uint4(word(0, k), word(1, k), word(2, k), word(3, k));
            fence_proxy_async_smem();  // visible to tcgen05.cp
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sfr0 + 8 * sb);
                mbar_arrive(empty0 + 8 * s);  // this tile's scale bytes are read
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        // The eight epilogue warps vote at every wait on a named barrier (id 1),
        // so that an exit is always a joint decision, and meet once per slice
        // after writing it into a staging buffer; one thread then stores the
        // slice's four boxes with the TMA (bulk group per slice, two buffers).
        constexpr int G = HAD >= 256 ? HAD / 128 : 1;  // groups per Hadamard block
        constexpr int kEpiThreads = 128 * kDqmEpiWg;
        const uint32_t wg = (warp - 3) >> 2, quarter = warp & 3, half = wg & 1;
        const uint32_t lane_base = (quarter * 32u) << 16;
        const float st_scale = FMT == FMT_NVFP4 ? *p.scale_fp32 : 0.0f;
        const bool issuer = warp == 3 && lane == 0;
        // this thread's row of the tile and its two 16-byte chunks (columns
        // 16 half .. + 15 of the box's 32) after the 64-byte swizzle
        const uint32_t rt = quarter * 32u + lane, sw = (rt >> 1) & 3u;
        const uint32_t off0 = rt * 64u + (((2u * half) ^ sw) << 4), off1 = rt * 64u + (((2u * half + 1u) ^ sw) << 4);
        const uint32_t stg0 = smem_u32(smem + kDqmStgOff);
#pragma unroll 1
        for (int64_t i = 0; i < n_my; ++i) {
            const int s = (int)(i % kDqmStages);
            const bool ok = mbar_wait(full0 + 8 * s, (uint32_t)((i / kDqmStages) & 1));
            if (!bar_and(1, kEpiThreads, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            const int64_t t = blockIdx.x + i * gridDim.x;
            const int64_t ct = t % p.n_ct;
            const int32_t y0 = (int32_t)((t / p.n_ct) * 128);
            float gm[4];
            if constexpr (FMT == FMT_DUAL) {
                const float4 g4 = *reinterpret_cast<const float4*>(smem + s * kDqmStageBytes + kDqmCodeBytes +
                                                                   kDqmScaleBytes + 16 * (quarter * 32 + lane));
                gm[0] = g4.x * p.had_norm;
                gm[1] = g4.y * p.had_norm;
                gm[2] = g4.z * p.had_norm;
                gm[3] = g4.w * p.had_norm;
            } else {
#pragma unroll
                for (int g = 0; g < 4; ++g) gm[g] = st_scale * p.had_norm;
            }
            __syncwarp();  // every lane has its group scales: the stage may be refilled
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
            bool aok = true;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                const int64_t j = 4 * i + q;
                const int slot = (int)(j % kDqmSlots);
                const uint32_t box0 = stg0 + (uint32_t)(j & 1) * kDqmStgBytes;
                // the store issued from this buffer two slices ago has read it
                // before the issuer joins the vote below
                if (issuer) bulk_wait_read1();
                const bool a = mbar_wait(accf0 + 8 * slot, (uint32_t)((j / kDqmSlots) & 1));
                if (!bar_and(1, kEpiThreads, a)) {
                    aok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[4][16];
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    tmem_ld16(tmem_base + lane_base + (uint32_t)(128 * slot + 32 * g) + 16u * half, r[g]);
                tmem_wait_ld16x4(r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce0 + 8 * slot);  // the slice's TMEM may be overwritten
                float v[4][16];
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        const float2 x = __fmul2_rn(make_float2(__uint_as_float(r[g][e]), __uint_as_float(r[g][e + 1])),
                                                    make_float2(gm[g], gm[g]));
                        v[g][e] = x.x;
                        v[g][e + 1] = x.y;
                    }
                if constexpr (G >= 2) {  // butterflies across the groups of a block
                    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
                    for (int st = 1; st < G; st <<= 1)
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            if ((g & st) == 0)
#pragma unroll
                                for (int e = 0; e < 16; e += 2) {
                                    const float2 x0 = make_float2(v[g][e], v[g][e + 1]);
                                    const float2 x1 = make_float2(v[g + st][e], v[g + st][e + 1]);
                                    const float2 sm = __fadd2_rn(x0, x1), df = __ffma2_rn(x1, m1, x0);
                                    v[g][e] = sm.x;
                                    v[g][e + 1] = sm.y;
                                    v[g + st][e] = df.x;
                                    v[g + st][e + 1] = df.y;
                                }
                }
                // bf16 into the staging boxes: 16 columns of the row per group
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = bf16x2_pack(v[g][2 * e], v[g][2 * e + 1]);
                    const uint32_t bx = box0 + (uint32_t)g * kDqmBoxBytes;
                    sts_v4(bx + off0, o[0], o[1], o[2], o[3]);
                    sts_v4(bx + off1, o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async_smem();  // visible to the TMA store
                bar_sync(1, kEpiThreads);
                if (issuer) {  // rows past M are not written (the map ends at row M)
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        tma_store_2d(&y_map, (int32_t)(ct * 512 + 128 * g + 32 * q), y0,
                                     box0 + (uint32_t)g * kDqmBoxBytes);
                    bulk_commit();
                }
            }
            if (!aok) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
        }
        if (issuer) bulk_wait0();  // every store has completed before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kDqmTmemCols);
    }
}

}  // namespace fp4q
