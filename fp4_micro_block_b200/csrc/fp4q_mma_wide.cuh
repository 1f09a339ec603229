// fp4q_mma_wide.cuh -- tensor-core block Hadamard of size n = 256 or 512 fused
// with NVFP4 / MXFP4 / dual-scale quantization.
//
// Sylvester's matrix factors as H_n = H_G (x) H_128 (G = n / 128): with the
// column index i = 128 a + b of an n-block,
//     y[128 a + b] = sum_a' H_G[a][a'] * z[128 a' + b],   z = H_128 applied to
//     each 128-column group of the block.
// The tensor cores compute every z group as a 128 x 128 x 128 UMMA (the B
// operand is -2^-4 H_128, so TMEM receives negated, partly normalised values);
// the epilogue applies the G-point butterfly across the groups in registers.
// (FP4Quant builds its 512-point FWHT the same way, as a small transform
// inside a level of size 32 plus a level across it; here the inner level is a
// dense product on the tensor cores.)
//
// A tile is 128 rows x n columns: G accumulators of 128 TMEM columns, all 512
// columns for n = 512 (two tiles in flight for n = 256).  All four epilogue
// warpgroups work on the same tile, warpgroup w on the columns
// b in [32 w, 32 w + 32) of every group:
//   pass 1  reads z in steps of 8 columns of every group, applies H_G, takes
//           the per-group maxima and writes y back into TMEM in place (the
//           remaining RN(1/sqrt 2) of n = 512 is folded into the quantizer);
//   (sync)  the epilogue warps meet at a named barrier (their pass-2 columns
//           were written by other warpgroups), and the dual format's group
//           maxima of the four warpgroups meet in shared memory;
//   pass 2  two warpgroups per output group, each quantizing two adjacent
//           32-column chunks (64 consecutive columns of a lane's row); for
//           n = 512 in two rounds, groups 0-1 then 2-3.  A group's TMEM columns
//           go back to the MMA warp as soon as its two warpgroups have read
//           them, so the next tile's UMMAs overlap the rest of pass 2 (n = 512:
//           groups 0 and 1 during the second round).  The codes of a round
//           (128 rows x 128 bytes) are written into a shared-memory box with the
//           128-byte swizzle and stored by one thread with the TMA; the scale
//           bytes go out directly.
// The sixteen epilogue warps vote on the accumulator wait of every tile
// (bar.red.and), so an early exit is joint and no warp is left at the named
// barriers that follow.
#pragma once

#include "fp4q_mma.cuh"

namespace fp4q {

constexpr int kWideEpiWarps = 16;                    // four warpgroups
constexpr int kWideThreads = 96 + 32 * kWideEpiWarps;  // 2 producer warps, the MMA warp, epilogue
constexpr int kWideRedBytes = 2 * 4 * 4 * kMmaTile * 4;  // [parity][warpgroup][group][row] fp32
constexpr int kWideBoxBytes = kMmaTile * 128;            // codes of 256 columns x 128 rows

template <int HAD>
struct Wide {
    static constexpr int G = HAD / kMmaTile;           // 128-column groups per block
    static constexpr int NBUF = 4 / G;                 // tiles in TMEM
    static constexpr int bars = 2 * kMmaStages + NBUF + NBUF * G + 1;
    static constexpr int ring_off = kTileBytes;
    static constexpr int red_off = ring_off + kMmaStages * kTileBytes;
    static constexpr int bar_off = red_off + kWideRedBytes;
    static constexpr int slot_off = bar_off + bars * 8;
    static constexpr int tab_off = (slot_off + 4 + 15) / 16 * 16;
    static constexpr int misc_off = tab_off + 128 * 16;
    // codes staging for the TMA stores: one 128-row x 128-byte box per pass-2
    // round (128-byte swizzle), two buffers
    static constexpr int stg_off = (misc_off + (kWideThreads / 32) * 4 + 1023) / 1024 * 1024;
    static constexpr int smem = 1024 + stg_off + 2 * kWideBoxBytes;
    static_assert(smem <= 227 * 1024, "shared memory");
};

// Issues the load of 8 fp32 columns; the values are valid only after
// tmem_wait_ld8x(), which takes them as operands so that no use is scheduled
// before the wait.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
                   "=f"(v[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld8x2(float (&a)[8], float (&b)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7]),
                   "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]), "+f"(b[7])
                 :
                 : "memory");
}
template <int G>
__device__ __forceinline__ void tmem_wait_ld8x(float (&z)[G][8]) {
    if constexpr (G == 2) {
        tmem_wait_ld8x2(z[0], z[1]);
    } else {
        asm volatile("tcgen05.wait::ld.sync.aligned;"
                     : "+f"(z[0][0]), "+f"(z[0][1]), "+f"(z[0][2]), "+f"(z[0][3]), "+f"(z[0][4]), "+f"(z[0][5]),
                       "+f"(z[0][6]), "+f"(z[0][7]), "+f"(z[1][0]), "+f"(z[1][1]), "+f"(z[1][2]), "+f"(z[1][3]),
                       "+f"(z[1][4]), "+f"(z[1][5]), "+f"(z[1][6]), "+f"(z[1][7]), "+f"(z[2][0]), "+f"(z[2][1]),
                       "+f"(z[2][2]), "+f"(z[2][3]), "+f"(z[2][4]), "+f"(z[2][5]), "+f"(z[2][6]), "+f"(z[2][7]),
                       "+f"(z[3][0]), "+f"(z[3][1]), "+f"(z[3][2]), "+f"(z[3][3]), "+f"(z[3][4]), "+f"(z[3][5]),
                       "+f"(z[3][6]), "+f"(z[3][7])
                     :
                     : "memory");
    }
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}
// The G consecutive group scales of a row and tile: one 16- or 8-byte store
// when the address allows it.
template <int G>
__device__ __forceinline__ void store_group_scales(float* dst, const float (&g)[G]) {
    const uintptr_t al = reinterpret_cast<uintptr_t>(dst);
    if constexpr (G == 4) {
        if ((al & 15) == 0) {
            *reinterpret_cast<float4*>(dst) = make_float4(g[0], g[1], g[2], g[3]);
            return;
        }
    }
    if ((al & 7) == 0) {
#pragma unroll
        for (int a = 0; a < G; a += 2) *reinterpret_cast<float2*>(dst + a) = make_float2(g[a], g[a + 1]);
        return;
    }
#pragma unroll
    for (int a = 0; a < G; ++a) dst[a] = g[a];
}

// The dual format's group scale of a group maximum gm: gm / 2688, correctly
// rounded (the IEEE division for gm < 2^-90, out of line).
__device__ __noinline__ float group_scale_tiny(float gm) { return __fdiv_rn(gm, 2688.0f); }
__device__ __forceinline__ float group_scale(float gm) {
    return gm >= 0x1p-90f ? div_split(-gm, 2688.0f, rcp2688()) : group_scale_tiny(gm);
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// B = -2^-4 * D * H_128 (K-major, 128-byte swizzle) for n = 256 and 512, its
// rows (accumulator columns) in the acc_col order of the 128-column kernel; D
// is the random-sign pattern of period 128 (identity when all signs are zero),
// so that H_n D_n = H_(n/128) (x) (H_128 D_128) with D_n = I (x) D_128.
__device__ __forceinline__ void build_h128_b(uint8_t* b, const uint32_t (&signs)[4]) {
    const uint32_t mag = 0x3f80u - 4u * 0x80u;  // bf16 bits of 2^-4
    for (int chunk = threadIdx.x; chunk < kTileBytes / 16; chunk += blockDim.x) {
        const int h = chunk / 1024, nn = (chunk / 8) % 128, cp = chunk % 8;
        const int c = cp ^ (nn & 7), oc = acc_col(nn);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            uint32_t pair = 0;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int k = h * 64 + c * 8 + e + t;
                const int par = __popc((uint32_t)(k & oc)) & 1;
                pair |= ((mag | (par ? 0u : 0x8000u)) ^ (sign_bit(signs, k) << 15)) << (16 * t);
            }
            w[e / 2] = pair;
        }
        *reinterpret_cast<uint4*>(b + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int FMT, int HAD, bool AMAX_ONLY>
__global__ void __launch_bounds__(kWideThreads, 1)
    had_mma_wide_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap codes_map,
                        const MmaParams p) {
    using W = Wide<HAD>;
    constexpr int G = W::G, NBUF = W::NBUF;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<1024>(smem_raw);
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t full0 = smem_u32(smem + W::bar_off), empty0 = full0 + 8 * kMmaStages;
    const uint32_t accf0 = empty0 + 8 * kMmaStages, relg0 = accf0 + 8 * NBUF;
    const uint32_t done_bar = relg0 + 8 * NBUF * G;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + W::slot_off);
    float4* tab = reinterpret_cast<float4*>(smem + W::tab_off);
    float* red = reinterpret_cast<float*>(smem + W::misc_off);
    float* red2 = reinterpret_cast<float*>(smem + W::red_off);
    constexpr bool kOddLog = HAD == 512;

    if (tid == 0) {
        prefetch_tmap(&tmap_x);
        if constexpr (!AMAX_ONLY) prefetch_tmap(&codes_map);
        for (int s = 0; s < kMmaStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < NBUF; ++b) mbar_init(accf0 + 8 * b, 1);
        for (int k = 0; k < NBUF * G; ++k) mbar_init(relg0 + 8 * k, 8);  // two warpgroups read a group
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512u);
        tmem_relinquish();
    }
    build_h128_b(smem, p.signs);
    fence_proxy_async_smem();
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
        // ------------------------------------------------ TMA producers: G sub-tiles per tile,
        // alternate sub-tiles from two warps (see had_mma_kernel)
        if (lane == 0) {
            const int64_t n_sub = n_my * G, pu = warp >> 1;
            int64_t u = pu;
            for (; u < n_sub; u += 2) {
                const int s = (int)(u % kMmaStages);
                if (u >= kMmaStages && !mbar_wait(empty0 + 8 * s, (uint32_t)((u / kMmaStages - 1) & 1))) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                const int64_t t = blockIdx.x + (u / G) * gridDim.x;
                const int32_t x0 = (int32_t)((t % p.n_ct) * HAD + (u % G) * kMmaTile);
                const int32_t y0 = (int32_t)((t / p.n_ct) * kMmaTile);
                const uint32_t dst = smem_u32(smem + W::ring_off + s * kTileBytes);
                mbar_arrive_expect_tx(full0 + 8 * s, kTileBytes);
                tma_load_2d(dst, &tmap_x, x0, y0, full0 + 8 * s);
                tma_load_2d(dst + kHalfBytes, &tmap_x, x0 + 64, y0, full0 + 8 * s);
            }
            for (int64_t k = pu; k < u; k += 2)
                if (k + kMmaStages >= u)
                    (void)mbar_wait(full0 + 8 * (int)(k % kMmaStages), (uint32_t)((k / kMmaStages) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t b_addr = smem_u32(smem);
            bool ok = true;
            for (int64_t j = 0; ok && j < n_my; ++j) {
                const int b = (int)(j % NBUF);
                for (int a = 0; a < G; ++a) {
                    const int64_t u = j * G + a;
                    const int s = (int)(u % kMmaStages);
                    ok = mbar_wait(full0 + 8 * s, (uint32_t)((u / kMmaStages) & 1));
                    if (ok && j >= NBUF)
                        ok = mbar_wait(relg0 + 8 * (b * G + a), (uint32_t)((j / NBUF - 1) & 1));
                    if (!ok) {
                        atomicOr(&g_device_error, kErrWaitTimeout);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + W::ring_off + s * kTileBytes);
                    const uint32_t d = tmem_base + (uint32_t)((b * G + a) * kMmaTile);
#pragma unroll
                    for (int k = 0; k < kMmaTile / 16; ++k) {
                        const uint32_t off = (uint32_t)((k / 4) * kHalfBytes + (k % 4) * 32);
                        umma_bf16(d, sw128_desc(a_addr + off), sw128_desc(b_addr + off), kIdescBf16M128N128,
                                  k > 0 ? 1u : 0u);
                    }
                    tc_commit(empty0 + 8 * s);
                }
                if (ok) tc_commit(accf0 + 8 * b);
            }
            tc_commit(done_bar);
            if (!mbar_wait(done_bar, 0)) atomicOr(&g_device_error, kErrWaitTimeout);
        }
    } else {
        // ------------------------------------------------ epilogue
        const uint32_t ew = warp - 3, wg = ew >> 2, quarter = warp & 3;
        const uint32_t rowt = quarter * 32 + lane;
        const uint32_t lane_base = (quarter * 32u) << 16;
        // n = 512: the remaining RN(1/sqrt 2) is applied per block by the quantizer
        const float fold = kOddLog ? __uint_as_float(0x3f3504f3u) : 1.0f;
        const ScaleCtx ctx_t = make_ctx(s_t);
        const bool issuer = ew == 0 && lane == 0;
        const uint32_t stg0 = smem_u32(smem + W::stg_off);
#pragma unroll 1
        for (int64_t j = 0; j < n_my; ++j) {
            const int b = (int)(j % NBUF);
            const bool ok = mbar_wait(accf0 + 8 * b, (uint32_t)((j / NBUF) & 1));
            // a joint decision of the sixteen epilogue warps (named barrier 1),
            // so that none is left at the barriers below
            if (!bar_and(1, 32 * kWideEpiWarps, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            tc_fence_after();
            const int64_t t = blockIdx.x + j * gridDim.x;
            const int64_t ct = t % p.n_ct, rt = t / p.n_ct;
            const int64_t row = rt * kMmaTile + rowt;
            const bool live = row < p.M;
            const uint32_t tbuf = tmem_base + lane_base + (uint32_t)(b * G * kMmaTile);

            // ---- pass 1: y = H_G z, group maxima, y back into TMEM
            float m[G];
#pragma unroll
            for (int a = 0; a < G; ++a) m[a] = 0.0f;
#pragma unroll 1
            for (int k = 0; k < 4; ++k) {
                const uint32_t pos = 32u * wg + 8u * k;
                float z[G][8];
#pragma unroll
                for (int a = 0; a < G; ++a) tmem_ld8(tbuf + a * kMmaTile + pos, z[a]);
                tmem_wait_ld8x<G>(z);
                // butterflies on pairs of columns: the packed f32x2 adds halve the
                // issue slots (the FMA pipe has room to spare in this kernel)
                const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    float2 v[G];
#pragma unroll
                    for (int a = 0; a < G; ++a) v[a] = make_float2(z[a][i], z[a][i + 1]);
                    if constexpr (G == 2) {
                        const float2 s0 = __fadd2_rn(v[0], v[1]), d0 = __ffma2_rn(v[1], m1, v[0]);
                        v[0] = s0;
                        v[1] = d0;
                    } else {
                        const float2 s01 = __fadd2_rn(v[0], v[1]), d01 = __ffma2_rn(v[1], m1, v[0]);
                        const float2 s23 = __fadd2_rn(v[2], v[3]), d23 = __ffma2_rn(v[3], m1, v[2]);
                        v[0] = __fadd2_rn(s01, s23);
                        v[1] = __fadd2_rn(d01, d23);
                        v[2] = __ffma2_rn(s23, m1, s01);
                        v[3] = __ffma2_rn(d23, m1, d01);
                    }
#pragma unroll
                    for (int a = 0; a < G; ++a) {
                        z[a][i] = v[a].x;
                        z[a][i + 1] = v[a].y;
                    }
                }
#pragma unroll
                for (int a = 0; a < G; ++a) {
                    float mm = m[a];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) mm = max3(mm, fabsf(z[a][i]), fabsf(z[a][i + 1]));
                    m[a] = mm;
                    if constexpr (!AMAX_ONLY) tmem_st8(tbuf + a * kMmaTile + pos, z[a]);
                }
            }
            if constexpr (AMAX_ONLY) {
                if (live) {
#pragma unroll
                    for (int a = 0; a < G; ++a) my_amax = fmaxf(my_amax, m[a] * fold);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(relg0 + 8 * (b * G + (int)(wg % G)));
                    if constexpr (G == 4) mbar_arrive(relg0 + 8 * (b * G + (int)((wg + 2) % G)));
                }
                continue;
            } else {
                // Pass 2 reads columns that other warpgroups wrote in pass 1: every
                // epilogue warp meets the others here (bounded mbarrier wait), with
                // the tcgen05 fences that order their TMEM stores before our loads.
                // The dual format also exchanges its group maxima here.
                tmem_wait_st();
                float gs[G / 2];
                float* rp = red2 + (j & 1) * (4 * 4 * kMmaTile);
                if constexpr (FMT == FMT_DUAL) {
#pragma unroll
                    for (int a = 0; a < G; ++a) rp[(wg * 4 + a) * kMmaTile + rowt] = m[a];
                }
                tc_fence_before();
                // both codes staging buffers are free once the previous tile's
                // stores have read them: the issuer waits before it joins
                if (issuer) bulk_wait_read0();
                bar_sync(1, 32 * kWideEpiWarps);
                tc_fence_after();
                if constexpr (FMT == FMT_DUAL) {  // group maxima over the four warpgroups
                    auto gscale = [&](int a) {
                        const float* rg = rp + a * kMmaTile + rowt;
                        const float gm = fmaxf(fmaxf(rg[0], rg[4 * kMmaTile]), fmaxf(rg[8 * kMmaTile], rg[12 * kMmaTile]));
                        return group_scale(gm * fold);
                    };
                    if (wg == 0) {
                        // the first warpgroup writes the row's G group scales of the
                        // tile with one store (a 4-byte store per group from two
                        // warpgroups per round cost 2.5 us on the C5 quantizer)
                        float ga[G];
#pragma unroll
                        for (int a = 0; a < G; ++a) ga[a] = gscale(a);
                        if (live) store_group_scales<G>(p.scale_fp32 + row * (p.K / 128) + ct * G, ga);
#pragma unroll
                        for (int h = 0; h < G / 2; ++h) gs[h] = ga[G == 4 ? 2 * h : 0];
                    } else {
#pragma unroll
                        for (int h = 0; h < G / 2; ++h)  // the groups this warpgroup quantizes (pass 2)
                            gs[h] = gscale(G == 4 ? 2 * h + (int)(wg / 2) : (int)(wg % 2));
                    }
                }
                // ---- pass 2: two warpgroups per output group, each quantizing two
                // adjacent chunks of 32 columns, so that a lane writes 64
                // consecutive columns (whole 32-byte sectors) of its row.  n = 256:
                // warpgroup wg takes chunks [2 (wg / 2), +2) of group wg % 2.
                // n = 512: two rounds, groups {0, 1} then {2, 3}, warpgroup wg
                // taking chunks [2 (wg % 2), +2) of group 2 h + wg / 2; a group's
                // TMEM columns go back to the MMA warp as soon as its two
                // warpgroups have read them, so the next tile's UMMAs for groups
                // 0 and 1 overlap the second round.
#pragma unroll 1
                for (int h = 0; h < G / 2; ++h) {
                    const int a = G == 4 ? 2 * h + (int)(wg / 2) : (int)(wg % 2);
                    const int c = G == 4 ? 2 * (int)(wg % 2) : 2 * (int)(wg / 2);
                    float g = 0.0f;
                    if constexpr (FMT == FMT_DUAL) {
                        g = gs[0];
                        if constexpr (G == 4) g = h ? gs[G / 2 - 1] : g;  // no indexed (local) array
                    }
                    const ScaleCtx ctx = FMT == FMT_DUAL ? make_ctx(g) : ctx_t;
                    const int64_t col = ct * HAD + a * kMmaTile + 32 * c;  // first column of the pair
                    uint32_t wa[4], wb[4];
                    float2 n[16];
                    float v[32];
                    tmem_ld32(tbuf + a * kMmaTile + 32u * c, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) n[i] = make_float2(v[2 * i], v[2 * i + 1]);
                    const uint32_t ea = quant_chunk<FMT>(n, ctx, tab, fold, wa);
                    tmem_ld32(tbuf + a * kMmaTile + 32u * (c + 1), v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(relg0 + 8 * (b * G + a));
#pragma unroll
                    for (int i = 0; i < 16; ++i) n[i] = make_float2(v[2 * i], v[2 * i + 1]);
                    const uint32_t eb = quant_chunk<FMT>(n, ctx, tab, fold, wb);
                    // this row's 32 bytes of the round's box: 16-byte chunks
                    // 4 (a - 2h) + c and + 1, at their 128-byte-swizzle places
                    {
                        const uint32_t k0 = 4u * (uint32_t)(a - 2 * h) + (uint32_t)c, rs = rowt & 7u;
                        const uint32_t bx = stg0 + (uint32_t)h * kWideBoxBytes + rowt * 128u;
                        sts_v4(bx + ((k0 ^ rs) << 4), wa[0], wa[1], wa[2], wa[3]);
                        sts_v4(bx + (((k0 + 1u) ^ rs) << 4), wb[0], wb[1], wb[2], wb[3]);
                    }
                    if (live) {
                        if constexpr (FMT == FMT_MXFP4) {  // two E8M0 bytes, 2-byte aligned
                            const int64_t nsc = p.K / 32, cb = col / 32;
                            uint8_t* sp = p.swizzled ? p.scales + swizzle_offset(row, cb, (nsc + 3) / 4)
                                                     : p.scales + row * nsc + cb;
                            *reinterpret_cast<uint16_t*>(sp) = (uint16_t)(ea | (eb << 8));
                        } else {  // four E4M3 bytes, 4-byte aligned
                            const int64_t nsc = p.K / 16, cb = col / 16;
                            uint8_t* sp = p.swizzled ? p.scales + swizzle_offset(row, cb, (nsc + 3) / 4)
                                                     : p.scales + row * nsc + cb;
                            *reinterpret_cast<uint32_t*>(sp) = ea | (eb << 16);
                        }
                    }
                    // the round's box is written: one thread stores it (rows past
                    // M are clipped by the map)
                    fence_proxy_async_smem();
                    bar_sync(1, 32 * kWideEpiWarps);
                    if (issuer) {
                        tma_store_2d(&codes_map, (int32_t)(ct * (HAD / 2) + 128 * h), (int32_t)(rt * kMmaTile),
                                     stg0 + (uint32_t)h * kWideBoxBytes);
                        bulk_commit();
                    }
                }
            }
        }
        if (issuer) bulk_wait0();  // every store has completed before the CTA exits
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
            float mx = 0.0f;
            for (int w = 0; w < kWideThreads / 32; ++w) mx = fmaxf(mx, red[w]);
            p.partials[blockIdx.x] = mx;
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512u);
    }
}

}  // namespace fp4q
