// fp4q_quant.cuh -- register-path quantizer for sm_100a: no rotation, or a
// block Hadamard of size 16 / 32 / 64 on rows whose length is not a multiple
// of 128 (the tensor-core kernels take every other rotation), then NVFP4 /
// MXFP4 / dual-scale quantization, or the amax pre-pass of the dynamic tensor
// scale.
//
// Work decomposition: one persistent CTA per SM streams tiles of 64 rows x
// TC columns (TC = 64: one 8 KiB TMA box with the 128-byte swizzle; dual
// scale: TC = 128, two boxes, so that a row's 128-column scale group is in one
// tile) through a ring of stages fed by two producer warps that issue
// alternate tiles (the copies of one issuing thread are handled one after the
// other, and one stream per CTA does not keep an SM's share of HBM bandwidth
// busy).  Pairs of consumer warps take alternate tiles; inside a tile lane =
// row, and each lane quantizes the TC/32 units (32 columns) of its row.
// In the swizzled box the 16-byte chunk c of row r sits at chunk c ^ (r % 8),
// so the eight lanes of a shared-memory phase (eight consecutive rows) read
// eight different bank groups.
//
// Block Hadamard (Sylvester order, unnormalised here; RN(1/sqrt n) is applied
// per block by the unit quantizers): n = 16, 32 inside a unit; n = 64 as H_32
// on each of a lane's two units and H_2 across them (H_64 = H_2 (x) H_32).
#pragma once

#include "fp4q_unit.cuh"

namespace fp4q {

constexpr int kThreads = 256;          // CTA size of the dequantizer kernels
#ifndef FP4Q_QBOX_ROWS
#define FP4Q_QBOX_ROWS 64
#endif
#ifndef FP4Q_QPRODUCERS
#define FP4Q_QPRODUCERS 2
#endif
constexpr int kQBoxRows = FP4Q_QBOX_ROWS;   // TMA box: 64 columns x kQBoxRows rows
constexpr int kQBoxBytes = kQBoxRows * 128;
constexpr int kQWarpsPerTile = kQBoxRows / 32;
constexpr int kQProducers = FP4Q_QPRODUCERS;
#ifndef FP4Q_QCTAS
#define FP4Q_QCTAS 1
#endif
constexpr int kQCtas = FP4Q_QCTAS;             // CTAs per SM
constexpr int kQRingBytes = 192 * 1024 / kQCtas;

enum : int { FMT_NVFP4 = 0, FMT_MXFP4 = 1, FMT_DUAL = 2, FMT_INT4 = 3 };

struct QuantParams {
    int64_t M, K;
    int64_t n_cs, n_tiles;      // column strips (TC wide) per row band, tiles
    uint8_t* codes;             // [M, K/2]
    uint8_t* scales;            // [M, K/B] or swizzled
    float* scale_fp32;          // NVFP4: tensor scale; DUAL: [M, K/128]
    float* partials;            // amax pass: per-CTA maxima out; dynamic quant: in
    int n_partials;             // number of valid partials (dynamic quant)
    int swizzled;               // scale layout
    int dynamic;                // NVFP4: 1 = tensor scale from partials, 0 = read *scale_fp32
    float had_norm;             // RN(1/sqrt(n)), 1 without rotation
#ifdef FP4Q_TEST_HOOKS
    int64_t skip_tile;          // test build: CTA 0 never issues its tile of this index
#endif
};

template <int FMT, int HAD>
struct QGeo {
    static constexpr int tc = FMT == FMT_DUAL ? 128 : 64;      // tile columns
    static constexpr int boxes = tc / 64;
    static constexpr int stage_bytes = boxes * kQBoxBytes;
    static constexpr int stages = kQRingBytes / stage_bytes;    // 24 or 12 (one CTA per SM)
    static constexpr int units = tc / 32;                       // units per lane per tile
    // consumer warpgroups: three where a lane holds 64 values at once (n = 64)
    // or reduces a dual-scale group, so that 128 registers per thread fit
    static constexpr int cwarps = ((HAD == 64 || FMT == FMT_DUAL) ? 12 : 16) / kQCtas;
    static_assert(cwarps % kQWarpsPerTile == 0, "consumer warps form whole tile groups");
    static constexpr int groups = cwarps / kQWarpsPerTile;
    // Tile j lands in stage j % stages and goes to consumer group j % groups.
    // The stages' full barriers are waited on by phase parity, which is exact
    // only while one group takes every use of a stage: a group that skipped
    // another group's use of its stage could see a phase two ahead as complete.
    static_assert(stages % groups == 0, "each stage is consumed by one consumer group");
    static constexpr int threads = 32 * (kQProducers + cwarps);
    static constexpr int bar_off = kQRingBytes;
    static constexpr int red_off = bar_off + 2 * stages * 8;
    static constexpr int tab_off = (red_off + (threads / 32) * 4 + 15) / 16 * 16;
    static constexpr int smem = 1024 + tab_off + 128 * 16;
    static_assert(smem <= 227 * 1024, "shared memory");
};

// Tensor scale of the dynamic mode: amax over the per-CTA partials / top (the
// largest grid value times 448: 2688 for NVFP4, 3136 for INT4).
__device__ __forceinline__ float tensor_scale_from_partials(const float* partials, int n,
                                                            float* red, float top = 2688.0f) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0.0f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    __syncthreads();
    return __fdiv_rn(m, top);
}

// Orders the computation of x before any later volatile asm.
__device__ __forceinline__ void pin(float x) { asm volatile("" ::"f"(x)); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Negated values of 8 consecutive bf16: o[j] = -x[j].
__device__ __forceinline__ void nunpack8(uint4 q, float* o) {
    o[0] = nbf16lo(q.x); o[1] = nbf16hi(q.x); o[2] = nbf16lo(q.y); o[3] = nbf16hi(q.y);
    o[4] = nbf16lo(q.z); o[5] = nbf16hi(q.z); o[6] = nbf16lo(q.w); o[7] = nbf16hi(q.w);
}

// Unit u (32 columns) of this lane's row in the staged tile, negated, as unit
// pairs n[i] = (-v[i], -v[16+i]).  row_base = the row's 128 bytes in box 0.
__device__ __forceinline__ void read_unit(const uint8_t* row_base, uint32_t row, int u, float2* n) {
    const uint8_t* box = row_base + (u >> 1) * kQBoxBytes;
    float t[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t chunk = (uint32_t)(4 * (u & 1) + c);
        nunpack8(*reinterpret_cast<const uint4*>(box + (((chunk ^ row) & 7u) << 4)), t + 8 * c);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) n[i] = make_float2(t[i], t[16 + i]);
}

template <int FMT, int HAD, bool AMAX_ONLY>
__global__ void __launch_bounds__(QGeo<FMT, HAD>::threads, kQCtas)
    quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const QuantParams p) {
    using G = QGeo<FMT, HAD>;
    static_assert(FMT != FMT_DUAL || HAD == 0, "dual scale needs K % 128 == 0: rotations go to the tensor cores");
    static_assert(HAD == 0 || HAD == 16 || HAD == 32 || HAD == 64, "register-path rotation sizes");
    constexpr int S = G::stages, U = G::units, NG = G::groups;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<1024>(smem_raw);
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t full0 = smem_u32(smem + G::bar_off), empty0 = full0 + 8 * S;
    float* red = reinterpret_cast<float*>(smem + G::red_off);
    float4* tab = reinterpret_cast<float4*>(smem + G::tab_off);
    // Only the unrotated path needs the correctly rounded quotient of the
    // bit-exact acceptance; a rotation's RN(1/sqrt n) is folded per block.
    constexpr bool kExact = HAD == 0;

    if (tid == 0) {
        prefetch_tmap(&tmap_x);
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kQWarpsPerTile);  // the warps of the consuming group
        }
        fence_barrier_init();
    }
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
    __syncthreads();

    const int64_t n_my = p.n_tiles > (int64_t)blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    float my_amax = 0.0f;

    if (warp < kQProducers) {
        // ------------------------------------------------ TMA producers (alternate tiles)
        if (lane == 0) {
            int64_t j = warp;
            for (; j < n_my; j += kQProducers) {
                const int s = (int)(j % S);
                if (j >= S && !mbar_wait(empty0 + 8 * s, (uint32_t)((j / S - 1) & 1))) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    break;
                }
                const int64_t t = blockIdx.x + j * gridDim.x;
#ifdef FP4Q_TEST_HOOKS
                // a tile that never arrives: its consumers' wait runs out
                if (blockIdx.x == 0 && j == p.skip_tile) continue;
#endif
                const int32_t x0 = (int32_t)((t % p.n_cs) * G::tc), y0 = (int32_t)((t / p.n_cs) * kQBoxRows);
                const uint32_t dst = smem_u32(smem + s * G::stage_bytes);
                mbar_arrive_expect_tx(full0 + 8 * s, G::stage_bytes);
#pragma unroll
                for (int b = 0; b < G::boxes; ++b)
                    tma_load_2d(dst + b * kQBoxBytes, &tmap_x, x0 + 64 * b, y0, full0 + 8 * s);
            }
            // every issued copy lands before the CTA may exit
            for (int64_t k = warp; k < j; k += kQProducers)
                if (k + S >= j) (void)mbar_wait(full0 + 8 * (int)(k % S), (uint32_t)((k / S) & 1));
        }
    } else {
        // ------------------------------------------------ consumers
        const uint32_t cw = warp - kQProducers, q = cw / kQWarpsPerTile;
        const uint32_t row = (cw % kQWarpsPerTile) * 32 + lane;
        const int64_t kc = p.K / 2;
        const float fold = p.had_norm;
        const ScaleCtx ctx_t = make_ctx(s_t);
#pragma unroll 1
        for (int64_t j = q; j < n_my; j += NG) {
            const int s = (int)(j % S);
            const bool ok = mbar_wait(full0 + 8 * s, (uint32_t)((j / S) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicOr(&g_device_error, kErrWaitTimeout);
                break;
            }
            const uint8_t* rb = smem + s * G::stage_bytes + row * 128;
            // Hands the stage back to the producers.  It is called only after
            // instructions that consume every value this lane loaded from the
            // stage (the last unit's stores, or its maximum): a warp issues in
            // order and such an instruction waits for its shared-memory loads,
            // so no load of the stage can still be pending when the producer
            // reuses it (a release right after the loads let the next tile's
            // copy overwrite data that had not been read yet).
            auto release = [&]() {
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * s);
            };
            const int64_t t = blockIdx.x + j * gridDim.x;
            const int64_t grow = (t / p.n_cs) * kQBoxRows + row;
            const int64_t col0 = (t % p.n_cs) * G::tc;
            const bool live = grow < p.M;

            // codes and scale byte(s) of one unit held in n (no stores)
            auto compute = [&](const float2* n, const ScaleCtx& ctx, uint32_t(&w)[4]) -> uint32_t {
                if constexpr (FMT == FMT_MXFP4) return mxfp4_unit(n, fold, w);
                else return nvfp4_unit<FMT == FMT_NVFP4, kExact>(n, amax_pair(n), ctx, tab, fold, w);
            };
            // stores unit u of this lane's row (any K: ragged last strip, half units)
            auto store_unit = [&](int u, const uint32_t(&w)[4], uint32_t e) {
                const int64_t col = col0 + 32 * u;
                if (!live || col >= p.K) return;
                const bool full = col + 32 <= p.K;  // else half a unit (NVFP4 with K = 16 mod 32)
                uint8_t* cp = p.codes + grow * kc + col / 2;
                if constexpr (FMT == FMT_MXFP4) {
                    *reinterpret_cast<uint4*>(cp) = make_uint4(w[0], w[1], w[2], w[3]);
                    const int64_t nsc = p.K / 32, c0 = col / 32;
                    if (p.swizzled) p.scales[swizzle_offset(grow, c0, (nsc + 3) / 4)] = (uint8_t)e;
                    else p.scales[grow * nsc + c0] = (uint8_t)e;
                } else {
                    if ((p.K & 31) == 0) {  // rows of codes are 16-byte aligned
                        *reinterpret_cast<uint4*>(cp) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else {  // K = 16 (mod 32): rows are only 8-byte aligned
                        *reinterpret_cast<uint2*>(cp) = make_uint2(w[0], w[1]);
                        if (full) *reinterpret_cast<uint2*>(cp + 8) = make_uint2(w[2], w[3]);
                    }
                    const int64_t nsc = p.K / 16, c0 = col / 16;
                    if (p.swizzled) {
                        const int64_t nC = (nsc + 3) / 4;
                        p.scales[swizzle_offset(grow, c0, nC)] = (uint8_t)(e & 0xffu);
                        if (full) p.scales[swizzle_offset(grow, c0 + 1, nC)] = (uint8_t)(e >> 8);
                    } else if (full && ((grow * nsc + c0) & 1) == 0) {
                        *reinterpret_cast<uint16_t*>(p.scales + grow * nsc + c0) = (uint16_t)e;
                    } else {
                        p.scales[grow * nsc + c0] = (uint8_t)(e & 0xffu);
                        if (full) p.scales[grow * nsc + c0 + 1] = (uint8_t)(e >> 8);
                    }
                }
            };
            // stores units u, u + 1 (64 columns): with K a multiple of 64 the lanes of
            // a pair (rows 2i, 2i + 1) swap halves so that every store instruction
            // writes whole 32-byte sectors (16 rows x 32 bytes) instead of 16-byte
            // halves of 32 rows.
            auto store_pair = [&](int u, const uint32_t(&wa)[4], uint32_t ea, const uint32_t(&wb)[4],
                                  uint32_t eb) {
                if ((p.K & 63) != 0) {
                    store_unit(u, wa, ea);
                    store_unit(u + 1, wb, eb);
                    return;
                }
                const bool odd = lane & 1u;
                uint32_t d1[4], d2[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t got = __shfl_xor_sync(0xffffffffu, odd ? wa[k] : wb[k], 1);
                    d1[k] = odd ? got : wa[k];  // row 2i: unit u (even lane), u + 1 (odd lane)
                    d2[k] = odd ? wb[k] : got;  // row 2i + 1
                }
                const int64_t r1 = grow - (odd ? 1 : 0), r2 = r1 + 1;
                const int64_t col = col0 + 32 * (u + (odd ? 1 : 0));
                if (r1 < p.M) *reinterpret_cast<uint4*>(p.codes + r1 * kc + col / 2) = make_uint4(d1[0], d1[1], d1[2], d1[3]);
                if (r2 < p.M) *reinterpret_cast<uint4*>(p.codes + r2 * kc + col / 2) = make_uint4(d2[0], d2[1], d2[2], d2[3]);
                if (!live) return;
                if constexpr (FMT == FMT_MXFP4) {  // two E8M0 bytes, 2-byte aligned
                    const int64_t nsc = p.K / 32, c0 = (col0 + 32 * u) / 32;
                    uint8_t* sp = p.swizzled ? p.scales + swizzle_offset(grow, c0, (nsc + 3) / 4)
                                             : p.scales + grow * nsc + c0;
                    *reinterpret_cast<uint16_t*>(sp) = (uint16_t)(ea | (eb << 8));
                } else {  // four E4M3 bytes, 4-byte aligned
                    const int64_t nsc = p.K / 16, c0 = (col0 + 32 * u) / 16;
                    uint8_t* sp = p.swizzled ? p.scales + swizzle_offset(grow, c0, (nsc + 3) / 4)
                                             : p.scales + grow * nsc + c0;
                    *reinterpret_cast<uint32_t*>(sp) = ea | (eb << 16);
                }
            };
            // unit u in registers, rotated (n = 16, 32)
            auto fetch = [&](int u, float2* n) {
                read_unit(rb, row, u, n);
                if constexpr (HAD == 16) fwht16x2(n);
                if constexpr (HAD == 32) fwht32(n);
            };
            auto unit_amax = [&](int u, const float2* n) {  // of the live columns, unscaled
                const int64_t col = col0 + 32 * u;
                if (!live || col >= p.K) return 0.0f;
                const float2 am = amax_pair(n);
                return col + 32 <= p.K ? fmaxf(am.x, am.y) : am.x;
            };

            if constexpr (HAD == 64) {
                // H_64 = H_2 (x) H_32: H_32 on each unit, then the butterfly across them
#pragma unroll
                for (int u = 0; u < U; u += 2) {
                    float2 a[16], b[16];
                    read_unit(rb, row, u, a);
                    read_unit(rb, row, u + 1, b);
                    fwht32(a);
                    fwht32(b);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 x0 = a[i], x1 = b[i];
                        a[i] = add2(x0, x1);
                        b[i] = sub2(x0, x1);
                    }
                    if constexpr (AMAX_ONLY) {
                        my_amax = fmaxf(my_amax, fmaxf(unit_amax(u, a), unit_amax(u + 1, b)) * fold);
                        pin(my_amax);
                    } else {
                        uint32_t wa[4], wb[4];
                        const uint32_t ea = compute(a, ctx_t, wa);
                        const uint32_t eb = compute(b, ctx_t, wb);
                        store_pair(u, wa, ea, wb, eb);
                    }
                }
                release();
            } else if constexpr (AMAX_ONLY) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float2 n[16];
                    fetch(u, n);
                    my_amax = fmaxf(my_amax, unit_amax(u, n) * fold);
                }
                pin(my_amax);
                release();
            } else if constexpr (FMT == FMT_DUAL) {
                // pass 1: the row's 128-column group maximum; pass 2: quantize
                float gm = 0.0f;
#pragma unroll 1
                for (int u = 0; u < U; ++u) {
                    float2 n[16];
                    fetch(u, n);
                    const float2 am = amax_pair(n);
                    gm = fmaxf(gm, fmaxf(am.x, am.y));
                }
                gm *= fold;
                const float Gs = (gm >= 0x1p-90f) ? div_split(-gm, 2688.0f, rcp2688()) : __fdiv_rn(gm, 2688.0f);
                const ScaleCtx ctx = make_ctx(Gs);
                if (live) p.scale_fp32[grow * (p.K / 128) + col0 / 128] = Gs;
#pragma unroll 1
                for (int u = 0; u < U; u += 2) {
                    uint32_t wa[4], wb[4];
                    float2 n[16];
                    fetch(u, n);
                    const uint32_t ea = compute(n, ctx, wa);
                    fetch(u + 1, n);
                    const uint32_t eb = compute(n, ctx, wb);
                    store_pair(u, wa, ea, wb, eb);
                }
                release();
            } else {
#pragma unroll
                for (int u = 0; u < U; u += 2) {
                    uint32_t wa[4], wb[4];
                    float2 n[16];
                    fetch(u, n);
                    const uint32_t ea = compute(n, ctx_t, wa);
                    fetch(u + 1, n);
                    const uint32_t eb = compute(n, ctx_t, wb);
                    store_pair(u, wa, ea, wb, eb);
                }
                release();
            }
        }
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_amax = fmaxf(my_amax, __shfl_xor_sync(0xffffffffu, my_amax, o));
        if (lane == 0) red[warp] = my_amax;
        __syncthreads();
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < G::threads / 32; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

}  // namespace fp4q
