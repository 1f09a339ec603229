// fp4q_dequant.cuh -- dequantization kernels for sm_100a: packed E2M1 codes +
// block scales back to bf16, optionally followed by the inverse block Hadamard
// (the normalised Sylvester matrix is its own inverse).  This is the receiving
// side of FP4-compressed activations (FP4Quant abstract).
//
// A unit is 32 consecutive columns of one row (two NVFP4 blocks, one MXFP4
// block).  Codes and scales are read straight from global memory (0.5-0.6 byte
// per element); the bf16 output is written with 16- or 32-byte stores.
//   n <= 32: dequant_stream_kernel, one unit per thread at a time, several
//            units' loads in flight, the rotation in registers;
//   n >= 64: dequant_warp_kernel, a warp per (row pair, 512 columns): H_32 in
//            registers, an exchange through the warp's own shared memory, then
//            H_(n/32) across the 32-column sub-rows of each block.
#pragma once

#include "fp4q_quant.cuh"

namespace fp4q {

constexpr int kTileCols = 512;  // columns of a dequantizer unit for n >= 64

// In-register butterflies over v[0..N) (unnormalised Walsh-Hadamard).  With
// PACKED the strides >= 2 run on the packed f32x2 add, pairing (v[i], v[i+1])
// with (v[i+s], v[i+s+1]) (half the issue slots; the streaming dequantizer has
// no registers to spare for it); stride 1 stays scalar, which keeps every
// pair (v[i], v[i+1]) in its register pair between the stages.
template <int N, bool PACKED = false>
__device__ __forceinline__ void fwht_reg(float* v) {
    if constexpr (!PACKED) {
#pragma unroll
        for (int s = 1; s < N; s <<= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                if ((i & s) == 0) {
                    float a = v[i], b = v[i + s];
                    v[i] = a + b;
                    v[i + s] = a - b;
                }
            }
        }
        return;
    }
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < N; i += 2) {  // stride 1 in scalar adds: the pairs stay in place
        const float a = v[i], b = v[i + 1];
        v[i] = a + b;
        v[i + 1] = a - b;
    }
#pragma unroll
    for (int st = 2; st < N; st <<= 1) {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            if ((i & st) == 0) {
                const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + st], v[i + st + 1]);
                const float2 s = __fadd2_rn(a, b), d = __ffma2_rn(b, m1, a);
                v[i] = s.x;
                v[i + 1] = s.y;
                v[i + st] = d.x;
                v[i + st + 1] = d.y;
            }
        }
    }
}

template <int HAD>
struct HadShape {
    static constexpr int n2 = HAD >= 64 ? HAD / 32 : 1;  // threads per Hadamard block
    static constexpr int k1w = 32 / n2;                  // columns per k2 row a thread owns
};

struct DequantParams {
    int64_t M, K;
    int64_t n_col_tiles;  // 512-column tiles per row
    const uint8_t* codes;
    const uint8_t* scales;
    const float* scale_fp32;
    uint16_t* y;
    int swizzled;
    float had_norm;
    uint32_t signs[4];  // random-sign rotation: bit j negates output channel j of every min(n, 128)
};

// x^ = D H y for a random-sign rotation: flips the sign of v where bit (sh + i)
// of the pattern word w is set, i = 0..N-1 (all within one 32-bit word).
template <int N>
__device__ __forceinline__ void apply_signs(float* v, uint32_t w) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ ((w << (31 - i)) & 0x80000000u));
}

// Raw bytes of one 32-column unit: packed codes, its scale byte(s) and the fp32
// scale, loaded ahead of their use (software pipelining).
struct RawUnit {
    uint32_t w[4];
    uint32_t e0, e1;  // scale bytes of the unit's two 16-blocks (MXFP4: e0 only)
    float s;
};

template <int FMT>
__device__ __forceinline__ void load_raw(const DequantParams& p, int64_t row, int64_t col, int nval,
                                         RawUnit& u) {
    const uint8_t* cp = p.codes + row * (p.K / 2) + col / 2;
    if ((p.K & 31) == 0) {
        uint4 q = __ldg(reinterpret_cast<const uint4*>(cp));
        u.w[0] = q.x; u.w[1] = q.y; u.w[2] = q.z; u.w[3] = q.w;
    } else {
        uint2 q = __ldg(reinterpret_cast<const uint2*>(cp));
        u.w[0] = q.x; u.w[1] = q.y;
        if (nval > 16) {
            uint2 q2 = __ldg(reinterpret_cast<const uint2*>(cp + 8));
            u.w[2] = q2.x; u.w[3] = q2.y;
        } else {
            u.w[2] = 0u; u.w[3] = 0u;
        }
    }
    if constexpr (FMT == FMT_MXFP4) {
        const int64_t nsc = p.K / 32, c0 = col / 32;
        u.e0 = p.swizzled ? __ldg(p.scales + swizzle_offset(row, c0, (nsc + 3) / 4))
                          : __ldg(p.scales + row * nsc + c0);
        u.e1 = 0u;
        u.s = 0.0f;
    } else {
        const int64_t nsc = p.K / 16, c0 = col / 16;
        u.e1 = 0u;
        if (p.swizzled) {
            const int64_t nC = (nsc + 3) / 4;
            u.e0 = __ldg(p.scales + swizzle_offset(row, c0, nC));
            if (nval > 16) u.e1 = __ldg(p.scales + swizzle_offset(row, c0 + 1, nC));
        } else {
            u.e0 = __ldg(p.scales + row * nsc + c0);
            if (nval > 16) u.e1 = __ldg(p.scales + row * nsc + c0 + 1);
        }
        u.s = (FMT == FMT_DUAL) ? __ldg(p.scale_fp32 + row * (p.K / 128) + col / 128)
                                : __ldg(p.scale_fp32);
    }
}

template <int FMT>
__device__ __forceinline__ void decode_raw(const RawUnit& u, float* v) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t byte = (u.w[i >> 2] >> (8 * (i & 3))) & 0xffu;
        float2 c = FMT == FMT_INT4 ? int4x2_decode(byte) : e2m1x2_decode(byte);
        v[2 * i] = c.x;
        v[2 * i + 1] = c.y;
    }
    if constexpr (FMT == FMT_MXFP4) {
        const uint32_t b = u.e0;
        const float sc = b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);  // 2^(b-127)
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= sc;
    } else {
        const float ev0 = e4m3_decode(u.e0), ev1 = e4m3_decode(u.e1);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (v[i] * ev0) * u.s;
#pragma unroll
        for (int i = 16; i < 32; ++i) v[i] = (v[i] * ev1) * u.s;
    }
}

// ---------------------------------------------------------------- streaming dequantizer
// Rotation sizes 0, 16 and 32 need no data from other units: each thread
// streams units (row-major order, grid-stride) and keeps the codes and scales of
// kDqDepth units in registers ahead of their use, so that enough small loads
// stay in flight to cover the memory latency.
constexpr int kDqDepth = 4;

__device__ __forceinline__ void advance_unit(int32_t& row, int32_t& j, int32_t drow, int32_t dj,
                                             int32_t upr) {
    j += dj;
    row += drow;
    if (j >= upr) {
        j -= upr;
        ++row;
    }
}

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const uint32_t* o, int nval, bool w32) {
    if (w32 && nval == 32) {  // two 256-bit stores
        asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(o[0]), "r"(o[1]),
                     "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                     : "memory");
        asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 16), "r"(o[8]),
                     "r"(o[9]), "r"(o[10]), "r"(o[11]), "r"(o[12]), "r"(o[13]), "r"(o[14]), "r"(o[15])
                     : "memory");
    } else {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
        d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
        if (nval > 16) {
            d4[2] = make_uint4(o[8], o[9], o[10], o[11]);
            d4[3] = make_uint4(o[12], o[13], o[14], o[15]);
        }
    }
}

template <int FMT, int HAD, bool SIGNED = false>
__global__ void __launch_bounds__(kThreads, 3) dequant_stream_kernel(const DequantParams p, int w32) {
    pdl_wait();
    pdl_trigger();
    // rows < 2^31 and units per row < 2^26: 32-bit unit coordinates
    const int32_t upr = (int32_t)((p.K + 31) / 32);  // units per row
    const int32_t M = (int32_t)p.M;
    const int64_t S = (int64_t)gridDim.x * blockDim.x;
    const int64_t u0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int32_t srow = (int32_t)(S / upr), sj = (int32_t)(S % upr);
    const int64_t D = kDqDepth * S;
    const int32_t drow = (int32_t)(D / upr), dj = (int32_t)(D % upr);
    int32_t row[kDqDepth], jj[kDqDepth];
    row[0] = (int32_t)min64(u0 / upr, (int64_t)M);
    jj[0] = (int32_t)(u0 % upr);
#pragma unroll
    for (int k = 1; k < kDqDepth; ++k) {
        row[k] = row[k - 1];
        jj[k] = jj[k - 1];
        advance_unit(row[k], jj[k], srow, sj, upr);
    }
    RawUnit buf[kDqDepth];
#pragma unroll
    for (int k = 0; k < kDqDepth; ++k)
        if (row[k] < M) load_raw<FMT>(p, row[k], 32 * (int64_t)jj[k], (int)min64(32, p.K - 32 * (int64_t)jj[k]), buf[k]);

    while (row[0] < M) {
#pragma unroll
        for (int k = 0; k < kDqDepth; ++k) {
            if (row[k] >= M) continue;
            const RawUnit cur = buf[k];
            const int64_t r = row[k], col = 32 * (int64_t)jj[k];
            const int nval = (int)min64(32, p.K - col);
            advance_unit(row[k], jj[k], drow, dj, upr);
            if (row[k] < M)
                load_raw<FMT>(p, row[k], 32 * (int64_t)jj[k], (int)min64(32, p.K - 32 * (int64_t)jj[k]), buf[k]);
            float v[32];
            decode_raw<FMT>(cur, v);
            if constexpr (HAD == 16) {
                fwht_reg<16>(v);
                fwht_reg<16>(v + 16);
            } else if constexpr (HAD == 32) {
                fwht_reg<32>(v);
            }
            if constexpr (HAD > 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= p.had_norm;
            }
            if constexpr (SIGNED) {  // period n (16 or 32): columns col + i, col % 32 == 0
                const uint32_t w = HAD == 16 ? (p.signs[0] & 0xffffu) * 0x10001u : p.signs[0];
                apply_signs<32>(v, w);
            }
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = bf16x2_pack(v[2 * i], v[2 * i + 1]);
            store_bf16x32(p.y + r * p.K + col, o, nval, w32 != 0);
        }
    }
}

#ifndef FP4Q_DEQUANT_CTAS_PER_SM
#define FP4Q_DEQUANT_CTAS_PER_SM 4
#endif
constexpr int kDequantCtasPerSm = FP4Q_DEQUANT_CTAS_PER_SM;

// Hadamard sizes 64..512 without CTA barriers: a warp owns a unit of two rows
// x 512 columns.  Lane (r2 = lane / 16, l = lane % 16) decodes columns
// [32 l, 32 l + 32) of row r2 and applies H_32 in registers; the warp then
// exchanges through its own 4 KiB of shared memory (a warp barrier), and lane
// (r2, m) applies H_n2 across the n2 sub-rows of 32 columns of block
// b = m / n2 to its k1w = 32 / n2 columns, tau = m % n2.  For a fixed k2 the
// n2 lanes of a block store 64 consecutive bytes of the row.  The next unit's
// codes and scales are loaded before the current one is worked on.
constexpr int kDqWarpSmem = 4096;  // per warp: 2 rows x 16 sub-rows x 32 fp32

// 16-byte chunk c of sub-row l sits at chunk c ^ dq_swz(l): conflict-free for
// the row writes and for the column reads of every n2.
__device__ __forceinline__ uint32_t dq_swz(uint32_t l) { return (l & 7u) ^ ((l >> 2) & 1u); }

// Decoded unit times one multiplier per 16-block, m = (E4M3 value * s) * c
// (MXFP4: 2^(b-127) * c), applied with the packed f32x2 multiply; c is the
// Hadamard normalisation, moved ahead of the butterflies (a few fp32 ulps from
// the oracle's order, far inside one bf16 ulp).
template <int FMT>
__device__ __forceinline__ void decode_raw_scaled(const RawUnit& u, float c, float* v) {
    float m0, m1;
    if constexpr (FMT == FMT_MXFP4) {
        const uint32_t b = u.e0;
        m0 = (b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u)) * c;
        m1 = m0;
    } else {
        m0 = (e4m3_decode(u.e0) * u.s) * c;
        m1 = (e4m3_decode(u.e1) * u.s) * c;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float m = i < 8 ? m0 : m1;
        const float2 q = __fmul2_rn(e2m1x2_decode((u.w[i >> 2] >> (8 * (i & 3))) & 0xffu), make_float2(m, m));
        v[2 * i] = q.x;
        v[2 * i + 1] = q.y;
    }
}

// Phase A, the exchange and phase B of one unit: the raw unit of lane (r2, l)
// in, the lane's phase-B outputs out (a[k2][i] is column 32 k2 + i of the
// lane's k1w-column slice of block b).  ws is the lane's row in the warp's
// scratch; the caller has synchronised the warp since the scratch was last read.
template <int FMT, int HAD, bool SIGNED>
__device__ __forceinline__ void dq_unit(const DequantParams& p, const RawUnit& cur, bool live, uint8_t* ws,
                                        uint32_t l, uint32_t b, uint32_t k1,
                                        float (&a)[HadShape<HAD>::n2][HadShape<HAD>::k1w]) {
    constexpr int n2 = HadShape<HAD>::n2, k1w = HadShape<HAD>::k1w;
    // phase-B read offset of sub-row sl = b n2 + k2 within the lane's row
    // (swizzled chunk); for n2 >= 8, b n2 is a multiple of 8 and the swizzle
    // depends on k2 alone, a constant of the unrolled loop
    auto rd_off = [&](uint32_t sl, int h) -> uint32_t {
        const uint32_t z = n2 >= 8 ? dq_swz(sl % n2) : dq_swz(sl);
        if constexpr (k1w == 2) return sl * 128u + (((k1 >> 2) ^ z) << 4) + (k1 & 3u) * 4u;
        else return sl * 128u + ((((k1 >> 2) + (uint32_t)h) ^ z) << 4);
    };
    float v[32];
    if (live) {
        decode_raw_scaled<FMT>(cur, p.had_norm, v);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
    }
    fwht_reg<32, true>(v);
    {
        uint8_t* rowp = ws + l * 128u;
        const uint32_t z = dq_swz(l);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<float4*>(rowp + ((ch ^ z) << 4)) =
                make_float4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
    }
    __syncwarp();
#pragma unroll
    for (int k2 = 0; k2 < n2; ++k2) {
        const uint32_t sl = b * n2 + (uint32_t)k2;  // sub-row of this block
        if constexpr (k1w == 2) {
            const float2 q = *reinterpret_cast<const float2*>(ws + rd_off(sl, 0));
            a[k2][0] = q.x;
            a[k2][1] = q.y;
        } else {
#pragma unroll
            for (int h = 0; h < k1w / 4; ++h) {
                const float4 q = *reinterpret_cast<const float4*>(ws + rd_off(sl, h));
                a[k2][4 * h] = q.x;
                a[k2][4 * h + 1] = q.y;
                a[k2][4 * h + 2] = q.z;
                a[k2][4 * h + 3] = q.w;
            }
        }
    }
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int st = 1; st < n2; st <<= 1) {
#pragma unroll
        for (int k2 = 0; k2 < n2; ++k2) {
            if ((k2 & st) == 0) {
#pragma unroll
                for (int i = 0; i < k1w; i += 2) {
                    const float2 x0 = make_float2(a[k2][i], a[k2][i + 1]);
                    const float2 x1 = make_float2(a[k2 + st][i], a[k2 + st][i + 1]);
                    const float2 sm = __fadd2_rn(x0, x1), df = __ffma2_rn(x1, m1, x0);
                    a[k2][i] = sm.x;
                    a[k2][i + 1] = sm.y;
                    a[k2 + st][i] = df.x;
                    a[k2 + st][i + 1] = df.y;
                }
            }
        }
    }
    if constexpr (SIGNED) {
        // output column cb + 32 k2 + i has pattern index (k1 + 32 k2 + i) mod
        // min(n, 128): word k2 mod (period / 32), bit k1 + i
        constexpr int kWords = (HAD < 128 ? HAD : 128) / 32;
#pragma unroll
        for (int k2 = 0; k2 < n2; ++k2) apply_signs<k1w>(a[k2], p.signs[k2 % kWords] >> k1);
    }
}

// bf16 of the lane's phase-B outputs, k1w consecutive columns per k2 (32 columns apart).
template <int HAD>
__device__ __forceinline__ void dq_store_slices(uint16_t* dst0, const float (&a)[HadShape<HAD>::n2][HadShape<HAD>::k1w]) {
    constexpr int n2 = HadShape<HAD>::n2, k1w = HadShape<HAD>::k1w;
#pragma unroll
    for (int k2 = 0; k2 < n2; ++k2) {
        uint16_t* dst = dst0 + 32 * k2;
        if constexpr (k1w == 2) {
            *reinterpret_cast<uint32_t*>(dst) = bf16x2_pack(a[k2][0], a[k2][1]);
        } else if constexpr (k1w == 4) {
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(bf16x2_pack(a[k2][0], a[k2][1]), bf16x2_pack(a[k2][2], a[k2][3]));
        } else {
#pragma unroll
            for (int h = 0; h < k1w / 8; ++h)
                reinterpret_cast<uint4*>(dst)[h] = make_uint4(
                    bf16x2_pack(a[k2][8 * h + 0], a[k2][8 * h + 1]), bf16x2_pack(a[k2][8 * h + 2], a[k2][8 * h + 3]),
                    bf16x2_pack(a[k2][8 * h + 4], a[k2][8 * h + 5]), bf16x2_pack(a[k2][8 * h + 6], a[k2][8 * h + 7]));
        }
    }
}

template <int FMT, int HAD, bool SIGNED = false>
__global__ void __launch_bounds__(kThreads, kDequantCtasPerSm) dequant_warp_kernel(const DequantParams p) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr int n2 = HadShape<HAD>::n2, k1w = HadShape<HAD>::k1w;
    static_assert(HAD >= 64 && n2 * k1w == 32, "block sizes 64..512");
    constexpr int kWarps = kThreads / 32;
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* const ws = smem_raw + warp * kDqWarpSmem + (lane >> 4) * 2048u;  // this lane's row
    const uint32_t r2 = lane >> 4, l = lane & 15;
    const uint32_t b = n2 == 16 ? 0u : l / n2, tau = l % n2, k1 = k1w * tau;
    // unit (row pair rp, 512-column tile ct), ct fastest; 32-bit coordinates
    // (the host keeps rows < 2^31), advanced by the grid stride without division
    const int32_t n_ct = (int32_t)p.n_col_tiles, n_rp = (int32_t)((p.M + 1) / 2);
    const int32_t stride = (int32_t)gridDim.x * kWarps;
    const int32_t drp = stride / n_ct, dct = stride % n_ct;
    const int32_t u0 = (int32_t)blockIdx.x * kWarps + (int32_t)warp;
    int32_t rp = u0 / n_ct, ct = u0 % n_ct;
    auto advance = [&](int32_t& r, int32_t& c) {
        c += dct;
        r += drp;
        if (c >= n_ct) {
            c -= n_ct;
            ++r;
        }
    };
    auto in_range = [&](int32_t r, int32_t c) {  // K % 64 == 0: whole 32-column pieces
        return (int64_t)r * 2 + r2 < p.M && (int64_t)c * kTileCols + 32 * l < p.K;
    };
    RawUnit cur{};
    if (rp < n_rp && in_range(rp, ct)) load_raw<FMT>(p, (int64_t)rp * 2 + r2, (int64_t)ct * kTileCols + 32 * l, 32, cur);
    while (rp < n_rp) {
        const bool live = in_range(rp, ct);
        const int64_t row = (int64_t)rp * 2 + r2;
        const int64_t cb = (int64_t)ct * kTileCols + (int64_t)b * HAD + k1;  // phase-B output column
        int32_t rn = rp, cn = ct;
        advance(rn, cn);
        RawUnit nxt{};
        if (rn < n_rp && in_range(rn, cn)) load_raw<FMT>(p, (int64_t)rn * 2 + r2, (int64_t)cn * kTileCols + 32 * l, 32, nxt);
        __syncwarp();  // the previous unit's reads of this warp's scratch are done
        float a[n2][k1w];
        dq_unit<FMT, HAD, SIGNED>(p, cur, live, ws, l, b, k1, a);
        // the block's columns exist when its first one does (K % n == 0)
        if (row < p.M && cb < p.K) dq_store_slices<HAD>(p.y + row * p.K + cb, a);
        cur = nxt;
        rp = rn;
        ct = cn;
    }
}

// ---------------------------------------------------------------- TMA-fed dequantizer
// The same unit walk and arithmetic as dequant_warp_kernel, for K % 512 == 0
// and the linear scale layout.  Each warp keeps its next units' codes, scale
// bytes and group scales in a private ring of kDqStages shared-memory stages
// filled by 2-D TMA copies (boxes of 2 rows: 256 code bytes, 32 or 16 scale
// bytes, 4 group scales), so the decode never waits on HBM; lane 0 refills a
// stage as soon as every lane has decoded it.
constexpr int kDqStages = 3;
constexpr uint32_t kDqStageBytes = 768;  // codes 2 x 256 | scale bytes 2 x 32 | group scales 2 x 16
constexpr uint32_t kDqRingSmem = kDqWarpSmem + kDqStages * kDqStageBytes + 128;  // + the stage barriers

template <int FMT, int HAD, bool SIGNED = false>
__global__ void __launch_bounds__(kThreads, kDequantCtasPerSm)
    dequant_tma_kernel(const DequantParams p, const __grid_constant__ CUtensorMap codes_map,
                       const __grid_constant__ CUtensorMap scales_map, const __grid_constant__ CUtensorMap g_map) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr int n2 = HadShape<HAD>::n2, k1w = HadShape<HAD>::k1w;
    static_assert(HAD >= 64 && n2 * k1w == 32, "block sizes 64..512");
    constexpr int kWarps = kThreads / 32;
    constexpr uint32_t kScaleBytes = FMT == FMT_MXFP4 ? 32u : 64u;  // both rows' scale bytes
    constexpr uint32_t kTx = 512u + kScaleBytes + (FMT == FMT_DUAL ? 32u : 0u);
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* const wbase = smem_raw + warp * kDqRingSmem;
    uint8_t* const ws = wbase + (lane >> 4) * 2048u;  // this lane's row of the exchange
    uint8_t* const ring = wbase + kDqWarpSmem;
    const uint32_t bar0 = smem_u32(ring + kDqStages * kDqStageBytes);
    const uint32_t r2 = lane >> 4, l = lane & 15;
    const uint32_t b = n2 == 16 ? 0u : l / n2, tau = l % n2, k1 = k1w * tau;
    if (lane == 0) {
        for (int s = 0; s < kDqStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_barrier_init();
        prefetch_tmap(&codes_map);
        prefetch_tmap(&scales_map);
        if constexpr (FMT == FMT_DUAL) prefetch_tmap(&g_map);
    }
    __syncwarp();
    pdl_wait();
    pdl_trigger();
    const int32_t n_ct = (int32_t)p.n_col_tiles, n_rp = (int32_t)((p.M + 1) / 2);
    const int32_t stride = (int32_t)gridDim.x * kWarps;
    const int32_t drp = stride / n_ct, dct = stride % n_ct;
    const int32_t u0 = (int32_t)blockIdx.x * kWarps + (int32_t)warp;
    int32_t rp = u0 / n_ct, ct = u0 % n_ct;
    auto advance = [&](int32_t& r, int32_t& c) {
        c += dct;
        r += drp;
        if (c >= n_ct) {
            c -= n_ct;
            ++r;
        }
    };
    // unit (r, c) into stage s (lane 0); rows past M read as zeros
    auto issue = [&](int s, int32_t r, int32_t c) {
        uint8_t* st = ring + s * kDqStageBytes;
        const uint32_t bar = bar0 + 8 * s;
        mbar_arrive_expect_tx(bar, kTx);
        tma_load_2d(smem_u32(st), &codes_map, c * (kTileCols / 2), 2 * r, bar);
        tma_load_2d(smem_u32(st + 512), &scales_map, c * (int32_t)(kScaleBytes / 2), 2 * r, bar);
        if constexpr (FMT == FMT_DUAL) tma_load_2d(smem_u32(st + 640), &g_map, c * 4, 2 * r, bar);
    };
    int32_t irp = rp, ict = ct;  // the next unit to issue
    if (lane == 0) {
        for (int s = 0; s < kDqStages && irp < n_rp; ++s) {
            issue(s, irp, ict);
            advance(irp, ict);
        }
    } else {
        for (int s = 0; s < kDqStages && irp < n_rp; ++s) advance(irp, ict);
    }
    const float s_t = FMT == FMT_NVFP4 ? __ldg(p.scale_fp32) : 0.0f;
    uint32_t it = 0;
    while (rp < n_rp) {
        const int s = (int)(it % kDqStages);
        const bool ok = mbar_wait(bar0 + 8 * s, (it / kDqStages) & 1u);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                // every copy issued into the ring lands before the CTA may exit
                int32_t r = rp, c = ct;
                for (uint32_t k = it; k < it + kDqStages && r < n_rp; ++k, advance(r, c))
                    (void)mbar_wait(bar0 + 8 * (k % kDqStages), (k / kDqStages) & 1u);
            }
            break;
        }
        const uint8_t* st = ring + s * kDqStageBytes;
        RawUnit cur;
        {
            const uint4 q = *reinterpret_cast<const uint4*>(st + 256 * r2 + 16 * l);
            cur.w[0] = q.x;
            cur.w[1] = q.y;
            cur.w[2] = q.z;
            cur.w[3] = q.w;
            if constexpr (FMT == FMT_MXFP4) {
                cur.e0 = st[512 + 16 * r2 + l];
                cur.e1 = 0u;
                cur.s = 0.0f;
            } else {
                const uint32_t e = *reinterpret_cast<const uint16_t*>(st + 512 + 32 * r2 + 2 * l);
                cur.e0 = e & 0xffu;
                cur.e1 = e >> 8;
                cur.s = FMT == FMT_DUAL ? *reinterpret_cast<const float*>(st + 640 + 16 * r2 + 4 * (l >> 2)) : s_t;
            }
        }
        const int64_t row = (int64_t)rp * 2 + r2;
        const bool live = row < p.M;
        __syncwarp();  // the previous unit's reads of the scratch are done
        float a[n2][k1w];
        dq_unit<FMT, HAD, SIGNED>(p, cur, live, ws, l, b, k1, a);
        // Every lane has used all it loaded from stage s (dq_unit consumed the
        // codes and scales before its first warp barrier): lane 0 refills it.
        if (lane == 0 && irp < n_rp) {
            fence_proxy_async_smem();
            issue(s, irp, ict);
        }
        if (irp < n_rp) advance(irp, ict);
        if (live) dq_store_slices<HAD>(p.y + row * p.K + (int64_t)ct * kTileCols + (int64_t)b * HAD + k1, a);
        advance(rp, ct);
        ++it;
    }
}

}  // namespace fp4q
