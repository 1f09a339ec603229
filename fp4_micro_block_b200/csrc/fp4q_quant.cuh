// fp4q_quant.cuh -- persistent quantizer kernels for sm_100a: optional block
// Hadamard rotation (sizes 16..512), then NVFP4 / MXFP4 / dual-scale
// quantization, or the amax pre-pass of the dynamic tensor scale.
//
// Work decomposition: warp pipelines.
//   Every warp streams its own "warp tiles" (1024 bf16 elements, 2 KiB)
//   through a private ring of kStages shared-memory stages with one mbarrier
//   each; lane 0 issues the copies for the tile kStages ahead as soon as the
//   warp has read a stage.  Warps never wait for each other, so a CTA needs no
//   block-wide barrier in its main loop, and the many warps of an SM keep
//   ~100-200 KiB of loads in flight.  Each lane owns one "unit" of 32
//   consecutive columns of one row.
//
// Warp-tile geometries (each keeps every shared-memory access below free of
// bank conflicts):
//   G2 (rotation n <= 128): 8 rows x 128 columns, two 2-D TMA boxes of
//      64 columns x 8 rows with the 128-byte swizzle.  lane -> row = lane & 7,
//      unit = lane >> 3, so the 8 lanes of a shared-memory phase are 8 rows.
//   G3 (rotation n = 256, 512): 1024/n rows x n columns, one 1-D bulk copy
//      per row into rows padded by 64 bytes.  lane -> row = lane / (n/32),
//      unit = lane % (n/32).
//
// Block Hadamard of size n = n2 * 32 (Sylvester order, H_n = H_n2 (x) H_32):
//   the n2 lanes owning one n-block read it "column-major" (for every k2 < n2
//   their 32/n2 columns k1), apply H_n2 across k2 in registers, exchange through
//   a swizzled per-warp fp32 scratch (n = 64: shuffles with the partner lane) so
//   that each lane holds its 32 contiguous values, and apply H_32 in registers.
//   n = 16, 32 need no exchange.  The result is scaled by RN(1/sqrt(n)).
#pragma once

#include "fp4q_unit.cuh"

namespace fp4q {

#ifndef FP4Q_STAGES
#define FP4Q_STAGES 4
#endif

constexpr int kWarps = 8;                     // consumer warps of a quantizer CTA
constexpr int kQuantThreads = kWarps * 32;
constexpr int kThreads = 256;                 // CTA size of the other kernels
constexpr int kStages = FP4Q_STAGES;     // per-warp ring depth
constexpr int kWtElems = 1024;           // elements of a warp tile
constexpr int kStageBytesG2 = 2048;      // two 1 KiB TMA boxes
constexpr int kStageBytesG3 = 2304;      // rows of n*2 bytes + 64 bytes of padding
constexpr int kScratchBytes = 4096;      // per-warp fp32 exchange (rotations >= 128)
constexpr int kRowPad = 64;

enum : int { FMT_NVFP4 = 0, FMT_MXFP4 = 1, FMT_DUAL = 2 };

struct QuantParams {
    int64_t M, K;
    int64_t n_rb, n_cb, n_wt;   // warp-tile grid: row blocks x column blocks
    const uint8_t* x;           // bf16 rows (bulk-copy geometry)
    int64_t ldx_bytes;
    uint8_t* codes;             // [M, K/2]
    uint8_t* scales;            // [M, K/B] or swizzled
    float* scale_fp32;          // NVFP4: tensor scale; DUAL: [M, K/128]
    float* partials;            // amax pass: per-CTA maxima out; dynamic quant: in
    int n_partials;             // number of valid partials (dynamic quant)
    int swizzled;               // scale layout
    int dynamic;                // NVFP4: 1 = tensor scale from partials, 0 = read *scale_fp32
    float had_norm;             // RN(1/sqrt(n))
};

template <int HAD>
struct Geo {
    static constexpr bool bulk = HAD >= 256;
    static constexpr int cols = bulk ? HAD : 128;             // warp-tile width
    static constexpr int rows = kWtElems / cols;              // 8, 4 or 2
    static constexpr int stage_bytes = bulk ? kStageBytesG3 : kStageBytesG2;
    static constexpr int row_bytes = bulk ? HAD * 2 + kRowPad : 0;
    static constexpr int lanes_per_row = cols / 32;           // 4, 8 or 16
    static constexpr int scratch = HAD >= 128 ? kScratchBytes : 0;
    // every warp's ring starts 1024-byte aligned (TMA swizzle-128 boxes); the
    // mbarriers of all warps sit after the rings
    static constexpr int warp_stride = kStages * stage_bytes + scratch;
    static_assert(bulk || warp_stride % 1024 == 0, "G2 rings must stay 1024-byte aligned");
    static_assert(warp_stride % 128 == 0, "warp regions must stay 128-byte aligned");
    static constexpr int min_ctas = HAD >= 128 ? 2 : 3;  // per SM (shared memory)
    static constexpr int n2 = HAD >= 64 ? HAD / 32 : 1;       // lanes per Hadamard block
    static constexpr int k1w = 32 / n2;                       // columns per k2 a lane reads
};

// Shared memory: the warps' rings, their mbarriers [kWarps][kStages], the
// reduction slots and the NVFP4 table.
template <int HAD>
constexpr int quant_smem_bytes() {
    return 1024 + kWarps * Geo<HAD>::warp_stride + kWarps * kStages * 8 + (kWarps + 2) * 4 + 16 +
           128 * 16 + 64;
}

// Stage byte offset of (row, column) in the G2 geometry: two boxes of
// 64 columns x 8 rows (1 KiB each), 128-byte swizzle.
__device__ __forceinline__ uint32_t g2_off(uint32_t row, uint32_t c) {
    return (c >> 6) * 1024u + swz128(row, (c & 63u) * 2u);
}

// Negated values of 8 consecutive bf16 into two float2 pairs-of-pairs order:
// out[j] = -x[j] for j < 8.
__device__ __forceinline__ void nunpack8(uint4 q, float* o) {
    o[0] = nbf16lo(q.x); o[1] = nbf16hi(q.x); o[2] = nbf16lo(q.y); o[3] = nbf16hi(q.y);
    o[4] = nbf16lo(q.z); o[5] = nbf16hi(q.z); o[6] = nbf16lo(q.w); o[7] = nbf16hi(q.w);
}

// 32 contiguous values t[0..31] -> unit pairs n[i] = (t[i], t[16+i]).
__device__ __forceinline__ void to_pairs(const float* t, float2* n) {
#pragma unroll
    for (int i = 0; i < 16; ++i) n[i] = make_float2(t[i], t[16 + i]);
}

// This lane's 32 rotated (unnormalised) values, negated, as unit pairs (unit
// `u` of row `row` of the staged tile).  For rotations >= 64 the call exchanges data with
// other lanes of the warp: every lane must call it.
template <int HAD>
__device__ __forceinline__ void load_unit(const uint8_t* stage, uint8_t* scratch, uint32_t lane,
                                          uint32_t row, uint32_t u, float2* n) {
    using G = Geo<HAD>;
    if constexpr (HAD <= 32) {
        float t[32];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            nunpack8(*reinterpret_cast<const uint4*>(stage + g2_off(row, 32 * u + 8 * c)), t + 8 * c);
        to_pairs(t, n);
        if constexpr (HAD == 16) fwht16x2(n);
        if constexpr (HAD == 32) fwht32(n);
    } else if constexpr (HAD == 64) {
        // units (2p, 2p+1) of a row = lanes l and l ^ 8; tau = position in the pair
        const uint32_t tau = u & 1u, c0 = 64u * (u >> 1);
        float a[2][16];
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
            nunpack8(*reinterpret_cast<const uint4*>(stage + g2_off(row, c0 + 32 * k2 + 16 * tau)), a[k2]);
            nunpack8(*reinterpret_cast<const uint4*>(stage + g2_off(row, c0 + 32 * k2 + 16 * tau + 8)),
                     a[k2] + 8);
        }
#pragma unroll
        for (int i = 0; i < 16; i += 2) {  // H_2 across k2
            const float2 x0 = make_float2(a[0][i], a[0][i + 1]), x1 = make_float2(a[1][i], a[1][i + 1]);
            const float2 s = add2(x0, x1), d = sub2(x0, x1);
            a[0][i] = s.x; a[0][i + 1] = s.y;
            a[1][i] = d.x; a[1][i + 1] = d.y;
        }
        // row k2 = tau: my 16 columns of it plus the partner's 16
        float t[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float send = tau ? a[0][i] : a[1][i];
            const float got = __shfl_xor_sync(0xffffffffu, send, 8);
            const float mine = tau ? a[1][i] : a[0][i];
            t[i] = tau ? got : mine;
            t[16 + i] = tau ? mine : got;
        }
        to_pairs(t, n);
        fwht32(n);
    } else {
        constexpr int n2 = G::n2, k1w = G::k1w, kp = k1w / 2;
        // A[k2][j] = -x[row, block + 32*k2 + k1w*tau + 2j + (0, 1)]
        float2 A[n2][kp];
        uint32_t tau, team;
        if constexpr (HAD == 128) {
            tau = u;  // lanes row, row+8, row+16, row+24
            team = row;
#pragma unroll
            for (int k2 = 0; k2 < n2; ++k2) {
                float o[8];
                nunpack8(*reinterpret_cast<const uint4*>(stage + g2_off(row, 32 * k2 + 8 * tau)), o);
#pragma unroll
                for (int j = 0; j < 4; ++j) A[k2][j] = make_float2(o[2 * j], o[2 * j + 1]);
            }
        } else {
            tau = lane % n2;
            team = lane / n2;
            const uint8_t* rp = stage + team * G::row_bytes;
#pragma unroll
            for (int k2 = 0; k2 < n2; ++k2) {
                const uint8_t* q = rp + (32 * k2 + k1w * tau) * 2;
                if constexpr (k1w == 2) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(q);
                    A[k2][0] = make_float2(nbf16lo(w), nbf16hi(w));
                } else {
                    const uint2 w = *reinterpret_cast<const uint2*>(q);
                    A[k2][0] = make_float2(nbf16lo(w.x), nbf16hi(w.x));
                    A[k2][1] = make_float2(nbf16lo(w.y), nbf16hi(w.y));
                }
            }
        }
#pragma unroll
        for (int s = 1; s < n2; s <<= 1) {  // H_n2 across k2
#pragma unroll
            for (int k2 = 0; k2 < n2; ++k2) {
                if ((k2 & s) == 0) {
#pragma unroll
                    for (int j = 0; j < kp; ++j) {
                        const float2 x0 = A[k2][j], x1 = A[k2 + s][j];
                        A[k2][j] = add2(x0, x1);
                        A[k2 + s][j] = sub2(x0, x1);
                    }
                }
            }
        }
        // Exchange through the warp's scratch: team rows R = team*n2 + k2 of 32
        // floats (128 B); the 16-byte chunk index is XORed with f(R) = team (n =
        // 128) or k2 & 7 (n >= 256), which keeps both the writes and the reads
        // free of bank conflicts.
        const uint32_t k1 = k1w * tau;
#pragma unroll
        for (int k2 = 0; k2 < n2; ++k2) {
            const uint32_t f = (HAD == 128) ? (team & 7u) : (uint32_t)(k2 & 7);
            uint8_t* rowp = scratch + (team * n2 + k2) * 128;
            if constexpr (k1w == 2) {
                *reinterpret_cast<float2*>(rowp + ((((k1 >> 2) ^ f) & 7u) << 4) + (k1 & 3u) * 4u) = A[k2][0];
            } else {
#pragma unroll
                for (int h = 0; h < k1w / 4; ++h)
                    *reinterpret_cast<float4*>(rowp + (((((k1 >> 2) + h) ^ f) & 7u) << 4)) =
                        make_float4(A[k2][2 * h].x, A[k2][2 * h].y, A[k2][2 * h + 1].x, A[k2][2 * h + 1].y);
            }
        }
        __syncwarp();
        {
            const uint32_t f = (HAD == 128) ? (team & 7u) : (tau & 7u);
            const uint8_t* rowp = scratch + (team * n2 + tau) * 128;
            float t[32];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const float4 q = *reinterpret_cast<const float4*>(rowp + (((ch ^ f) & 7u) << 4));
                t[4 * ch] = q.x;
                t[4 * ch + 1] = q.y;
                t[4 * ch + 2] = q.z;
                t[4 * ch + 3] = q.w;
            }
            to_pairs(t, n);
        }
        fwht32(n);
    }
}

// Tensor scale of the dynamic NVFP4 mode: amax over the per-CTA partials / 2688.
__device__ __forceinline__ float tensor_scale_from_partials(const float* partials, int n,
                                                            float* red) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0.0f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    __syncthreads();
    return __fdiv_rn(m, 2688.0f);
}

template <int FMT, int HAD, bool AMAX_ONLY>
__global__ void __launch_bounds__(kQuantThreads, Geo<HAD>::min_ctas)
    quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const QuantParams p) {
    using G = Geo<HAD>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31, warp = tid >> 5;
    uint64_t* full_bars = reinterpret_cast<uint64_t*>(smem + kWarps * G::warp_stride);
    float* red = reinterpret_cast<float*>(full_bars + kWarps * kStages);
    float4* tab = reinterpret_cast<float4*>((reinterpret_cast<uintptr_t>(red + kWarps + 2) + 15) &
                                            ~uintptr_t(15));
    // The rotation's normalisation RN(1/sqrt n) is applied per block by the
    // quantizer (nvfp4_unit / mxfp4_unit); only the unrotated path needs the
    // correctly rounded quotient of the bit-exact acceptance.
    constexpr bool kFold = HAD > 0;
    constexpr bool kExact = HAD == 0;

    if (tid == 0) {
        if constexpr (!G::bulk) prefetch_tmap(&tmap_x);
        for (int k = 0; k < kWarps * kStages; ++k) mbar_init(smem_u32(&full_bars[k]), 1);
        fence_barrier_init();
    }
    pdl_wait();
    pdl_trigger();
    // NVFP4: tensor scale, and the per-CTA table of decoded block scales.
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

    const int64_t nw = (int64_t)gridDim.x * kWarps;
    const int64_t step_rb = nw / p.n_cb, step_cb = nw % p.n_cb;
    auto advance = [&](int64_t& rb, int64_t& cb) {  // tile t -> t + nw without division
        cb += step_cb;
        rb += step_rb;
        if (cb >= p.n_cb) {
            cb -= p.n_cb;
            ++rb;
        }
    };
    float my_amax = 0.0f;

    if (warp < kWarps) {
        // Each warp streams its own tiles t = gw, gw + nw, ... : lane 0 refills a
        // stage as soon as the warp has read it, kStages tiles ahead.
        uint8_t* stages = smem + warp * G::warp_stride;
        uint8_t* scratch = stages + kStages * G::stage_bytes;
        uint64_t* bars = full_bars + warp * kStages;
        const uint32_t row = G::bulk ? lane / G::lanes_per_row : (lane & 7u);
        const uint32_t u = G::bulk ? lane % G::lanes_per_row : (lane >> 3);
        const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;
        const int64_t n_my = p.n_wt > gw ? (p.n_wt - 1 - gw) / nw + 1 : 0;
        int64_t rb = gw / p.n_cb, cb = gw % p.n_cb;  // tile being consumed
        int64_t irb = rb, icb = cb;                  // next tile to issue (lane 0)
        const int64_t kc = p.K / 2;
        ScaleCtx ctx = make_ctx(s_t);
        const float fold = kFold ? p.had_norm : 1.0f;

        auto issue = [&](int64_t i) {  // lane 0: tile (irb, icb) into stage i % kStages
            const uint32_t st = (uint32_t)(i % kStages);
            const uint32_t bar = smem_u32(&bars[st]);
            const uint32_t dst = smem_u32(stages + st * G::stage_bytes);
            if constexpr (G::bulk) {
                const int64_t r0 = irb * G::rows;
                const int nr = (int)min64(G::rows, p.M - r0);
                mbar_arrive_expect_tx(bar, (uint32_t)(nr * HAD * 2));
                const uint8_t* src = p.x + r0 * p.ldx_bytes + icb * HAD * 2;
                for (int r = 0; r < nr; ++r)
                    bulk_load_1d(dst + r * G::row_bytes, src + r * p.ldx_bytes, HAD * 2, bar);
            } else {
                const int32_t x0 = (int32_t)(icb * 128), y = (int32_t)(irb * 8);
                const int nb = (p.K - x0 > 64) ? 2 : 1;
                mbar_arrive_expect_tx(bar, (uint32_t)(nb * 1024));
                tma_load_2d(dst, &tmap_x, x0, y, bar);
                if (nb == 2) tma_load_2d(dst + 1024, &tmap_x, x0 + 64, y, bar);
            }
            advance(irb, icb);
        };
        if (lane == 0)
            for (int64_t i = 0; i < min64(kStages, n_my); ++i) issue(i);

        for (int64_t i = 0; i < n_my; ++i, advance(rb, cb)) {
            const uint32_t st = (uint32_t)(i % kStages);
            const bool ok = mbar_wait(smem_u32(&bars[st]), (uint32_t)((i / kStages) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                // A tile never arrived: record it, let this warp's copies land, stop.
                if (lane == 0) {
                    atomicOr(&g_device_error, kErrWaitTimeout);
                    for (int64_t k = i; k < min64(n_my, i + kStages); ++k)
                        (void)mbar_wait(smem_u32(&bars[k % kStages]), (uint32_t)((k / kStages) & 1));
                }
                break;
            }
            float2 n[16];
            load_unit<HAD>(stages + st * G::stage_bytes, scratch, lane, row, u, n);
            __syncwarp();  // every lane has read the stage (and the scratch): refill it
            if (lane == 0 && i + kStages < n_my) issue(i + kStages);

            const int64_t grow = rb * G::rows + row;
            const int64_t col = cb * G::cols + 32 * (int64_t)u;
            const bool live = grow < p.M && col < p.K;
            const bool full = col + 32 <= p.K;  // else half a unit (NVFP4 with K = 16 mod 32)

            if constexpr (AMAX_ONLY) {
                if (live) {
                    const float2 am = mul2(amax_pair(n), dup2(fold));
                    my_amax = fmaxf(my_amax, full ? fmaxf(am.x, am.y) : am.x);
                }
            } else if constexpr (FMT == FMT_MXFP4) {
                if (live) {
                    uint32_t w[4];
                    const uint32_t b = mxfp4_unit(n, fold, w);
                    *reinterpret_cast<uint4*>(p.codes + grow * kc + col / 2) = make_uint4(w[0], w[1], w[2], w[3]);
                    const int64_t nsc = p.K / 32, c0 = col / 32;
                    if (p.swizzled) p.scales[swizzle_offset(grow, c0, (nsc + 3) / 4)] = (uint8_t)b;
                    else p.scales[grow * nsc + c0] = (uint8_t)b;
                }
            } else {
                const float2 am = amax_pair(n);
                if constexpr (FMT == FMT_DUAL) {  // group scale over 4 units of one row
                    float g = fmaxf(am.x, am.y) * fold;
                    if constexpr (G::bulk) {  // the units of a group are 4 consecutive lanes
                        g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 1));
                        g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 2));
                    } else {  // lanes row, row+8, row+16, row+24
                        g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 8));
                        g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 16));
                    }
                    const float Gs = (g >= 0x1p-90f) ? div_split(-g, 2688.0f, rcp2688()) : __fdiv_rn(g, 2688.0f);
                    ctx = make_ctx(Gs);
                }
                if (live) {
                    uint32_t w[4];
                    const uint32_t e2 = nvfp4_unit<FMT == FMT_NVFP4, kExact>(n, am, ctx, tab, fold, w);
                    uint8_t* cp = p.codes + grow * kc + col / 2;
                    const int64_t nsc = p.K / 16, c0 = col / 16;
                    if ((p.K & 31) == 0) {  // rows of codes are 16-byte aligned
                        *reinterpret_cast<uint4*>(cp) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else {  // K = 16 (mod 32): rows are only 8-byte aligned
                        *reinterpret_cast<uint2*>(cp) = make_uint2(w[0], w[1]);
                        if (full) *reinterpret_cast<uint2*>(cp + 8) = make_uint2(w[2], w[3]);
                    }
                    if (p.swizzled) {
                        const int64_t nC = (nsc + 3) / 4;
                        p.scales[swizzle_offset(grow, c0, nC)] = (uint8_t)(e2 & 0xffu);
                        if (full) p.scales[swizzle_offset(grow, c0 + 1, nC)] = (uint8_t)(e2 >> 8);
                    } else if (full && ((grow * nsc + c0) & 1) == 0) {
                        *reinterpret_cast<uint16_t*>(p.scales + grow * nsc + c0) = (uint16_t)e2;
                    } else {
                        p.scales[grow * nsc + c0] = (uint8_t)(e2 & 0xffu);
                        if (full) p.scales[grow * nsc + c0 + 1] = (uint8_t)(e2 >> 8);
                    }
                    if constexpr (FMT == FMT_DUAL) {
                        if ((col & 127) == 0) p.scale_fp32[grow * (p.K / 128) + col / 128] = ctx.s;
                    }
                }
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
            for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

}  // namespace fp4q
