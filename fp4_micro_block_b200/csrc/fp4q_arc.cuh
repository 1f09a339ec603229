// fp4q_arc.cuh -- ARCQuant fused kernel for sm_100a: channel reorder + RMSNorm
// + primary NVFP4 quantization + NVFP4 quantization of the residual of the
// outlier channels, written as one [primary K | residual S] GEMM operand
// (ARCQuant summary, "Methodologie" items 1-5).
//
// One warp per row: a row never needs more than its own warp, so there is no
// CTA-wide barrier on the path.  Each warp streams its rows through a private
// ring of row buffers filled by 1-D bulk copies (lane 0 refills a buffer once
// the warp's stores of that row, which consume every value read from it, have
// issued).  Per row:
//   1. sum of squares over the row in natural order (16-byte loads, shuffle
//      reduction) -> rs = 1 / sqrt(mean + eps);
//   2. lane l owns output blocks b = l, l + 32, ... (reordered positions
//      16b..16b+15); for each pair of them it gathers x[perm[p]] from the row
//      buffer, applies rs and gamma[perm[p]] and quantizes the two blocks as
//      one unit (32 consecutive blocks per store instruction);
//   3. at the outlier positions (a per-block bit mask) it forms the residual
//      y - (E2M1val * E4M3val) * s_t into a per-warp buffer indexed by outlier
//      slot; after a warp barrier, lanes quantize the S/16 residual blocks.
// The CTA keeps perm and gamma as one 32-bit word per position (channel index
// | bf16 gamma of that channel), the outlier bit mask per block and the slot of
// every outlier position, built once per CTA.
#pragma once

#include "fp4q_quant.cuh"

namespace fp4q {

#ifndef FP4Q_ARC_MAX_WARPS
#define FP4Q_ARC_MAX_WARPS 14
#endif
constexpr int kArcMaxWarps = FP4Q_ARC_MAX_WARPS;  // launch bound: rows in flight per SM

struct ArcParams {
    int64_t M, K, S;
    const int32_t* perm;      // [K]
    const int32_t* outliers;  // [S] reordered positions
    const uint16_t* gamma;    // bf16 [K]
    const uint8_t* x;         // bf16 rows, byte stride ldx_bytes
    int64_t ldx_bytes;
    float eps;
    uint8_t* codes;           // [M, (K+S)/2]
    uint8_t* scales;          // [M, (K+S)/16] or swizzled
    float* tensor_scale;
    float* partials;
    int n_partials;
    int swizzled;
    int dynamic;
    int warps;                // warps per CTA (one row each at a time)
    int stages;               // row buffers per warp
};

// Shared-memory layout (byte offsets), all 16-byte aligned.
struct ArcLayout {
    int ring, pg, omask, oidx, rslot, res, bars, red, tab, total;
};

__host__ __device__ inline ArcLayout arc_layout(int64_t K, int64_t S, int warps, int stages) {
    ArcLayout l;
    const int row_bytes = (int)K * 2;
    l.ring = 0;
    l.pg = l.ring + warps * stages * row_bytes;                 // u32 [K]
    l.omask = l.pg + (int)K * 4;                                // u32 [K/16]
    l.oidx = l.omask + (int)((K / 16 * 4 + 15) / 16 * 16);      // i16 [K]
    l.rslot = l.oidx + (int)((K * 2 + 15) / 16 * 16);           // i16 [S]
    l.res = l.rslot + (int)((S * 2 + 15) / 16 * 16);            // f32 [warps][S]
    l.bars = l.res + (int)((warps * S * 4 + 15) / 16 * 16);     // u64 [warps][stages]
    l.red = l.bars + (warps * stages * 8 + 15) / 16 * 16;       // f32 [32]
    l.tab = l.red + 128;                                        // float4 [128]
    l.total = l.tab + 128 * 16 + 128;                           // + alignment slack
    return l;
}

template <bool AMAX_ONLY>
__global__ void __launch_bounds__(kArcMaxWarps * 32, 1) arc_kernel(const ArcParams p) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                               ~uintptr_t(127));
    const int K = (int)p.K, S = (int)p.S, nb = K / 16, W = p.warps, SR = p.stages;
    const ArcLayout L = arc_layout(p.K, p.S, W, SR);
    const uint32_t row_bytes = (uint32_t)K * 2u;
    uint32_t* pg = reinterpret_cast<uint32_t*>(smem + L.pg);
    uint32_t* omask = reinterpret_cast<uint32_t*>(smem + L.omask);
    int16_t* oidx = reinterpret_cast<int16_t*>(smem + L.oidx);
    int16_t* rslot = reinterpret_cast<int16_t*>(smem + L.rslot);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    float* red = reinterpret_cast<float*>(smem + L.red);
    float4* tab = reinterpret_cast<float4*>(smem + L.tab);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;

    // ---- per-CTA tables
    bool bad_index = false;
    // pg: word of position q = 16b + 4k4 + t at index 4 (k4 nb + b) + t, so that
    // the 16-byte loads of 32 lanes (blocks b = lane + 32i) are consecutive
    for (int q = tid; q < K; q += nthreads) {
        int c = p.perm[q];
        if ((unsigned)c >= (unsigned)K) {  // not a channel: clamp, flag
            bad_index = true;
            c = 0;
        }
        const int b = q >> 4, k4 = (q >> 2) & 3, t = q & 3;
        pg[4 * (k4 * nb + b) + t] = (uint32_t)c | ((uint32_t)p.gamma[c] << 16);
        oidx[q] = -1;
    }
    for (int b = tid; b < nb; b += nthreads) omask[b] = 0u;
    if (tid < W * SR) mbar_init(smem_u32(&bars[tid]), 1);
    __syncthreads();
    for (int i = tid; i < S; i += nthreads) {  // slot of every outlier position
        int q = p.outliers[i];
        if ((unsigned)q >= (unsigned)K) {
            bad_index = true;
            q = 0;
        }
        oidx[q] = (int16_t)i;  // a position listed twice keeps one slot
        atomicOr(&omask[q >> 4], 1u << (q & 15));
    }
    __syncthreads();
    for (int i = tid; i < S; i += nthreads) {  // slot read by residual element i
        const unsigned q = (unsigned)p.outliers[i];
        rslot[i] = oidx[q < (unsigned)K ? q : 0u];
    }
    if (bad_index) atomicOr(&g_device_error, kErrBadIndex);
    if (tid == 0) fence_barrier_init();

    float s_t = 0.0f;
    if constexpr (!AMAX_ONLY) {
        if (p.dynamic) {
            s_t = tensor_scale_from_partials(p.partials, p.n_partials, red);
            if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = s_t;
        } else {
            s_t = *p.tensor_scale;
        }
        build_table(tab, s_t);
    }
    __syncthreads();

    const ScaleCtx ctx = make_ctx(s_t);
    const int64_t KS = p.K + p.S, kcs = KS / 2, nsc = KS / 16, nC = (nsc + 3) / 4;
    const int64_t gw = (int64_t)blockIdx.x * W + warp, nw = (int64_t)gridDim.x * W;
    const int64_t n_my = p.M > gw ? (p.M - 1 - gw) / nw + 1 : 0;
    uint8_t* ring = smem + L.ring + (size_t)warp * SR * row_bytes;
    uint64_t* wbars = bars + warp * SR;
    float* res = reinterpret_cast<float*>(smem + L.res) + warp * S;
    float my_amax = 0.0f;

    auto issue = [&](int64_t i) {  // lane 0: row i of this warp into buffer i % SR
        const int64_t row = gw + i * nw;
        const uint32_t bar = smem_u32(&wbars[i % SR]);
        mbar_arrive_expect_tx(bar, row_bytes);
        bulk_load_1d(smem_u32(ring + (i % SR) * row_bytes), p.x + row * p.ldx_bytes, row_bytes, bar);
    };
    if (lane == 0)
        for (int64_t i = 0; i < min64(SR, n_my); ++i) issue(i);

    for (int64_t i = 0; i < n_my; ++i) {
        const bool ok = mbar_wait(smem_u32(&wbars[i % SR]), (uint32_t)((i / SR) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                for (int64_t k = i; k < min64(n_my, i + SR); ++k)
                    (void)mbar_wait(smem_u32(&wbars[k % SR]), (uint32_t)((k / SR) & 1));
            }
            break;
        }
        const int64_t row = gw + i * nw;
        const uint8_t* xr = ring + (i % SR) * row_bytes;
        const uint16_t* xs = reinterpret_cast<const uint16_t*>(xr);

        // 1. sum of squares (natural order) and the row's RMS factor
        float ss = 0.0f;
        for (int k = 8 * lane; k < K; k += 256) {
            const uint4 q = *reinterpret_cast<const uint4*>(xr + 2 * k);
            float a;
            a = bf16lo(q.x); ss = fmaf(a, a, ss);
            a = bf16hi(q.x); ss = fmaf(a, a, ss);
            a = bf16lo(q.y); ss = fmaf(a, a, ss);
            a = bf16hi(q.y); ss = fmaf(a, a, ss);
            a = bf16lo(q.z); ss = fmaf(a, a, ss);
            a = bf16hi(q.z); ss = fmaf(a, a, ss);
            a = bf16lo(q.w); ss = fmaf(a, a, ss);
            a = bf16hi(q.w); ss = fmaf(a, a, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = __frcp_rn(__fsqrt_rn(__fdiv_rn(ss, (float)K) + p.eps));

        // 2. reorder + normalise + quantize, two blocks (b, b + 32) per unit;
        // y is kept negated (unit pairs), -y = (x * rs) * (-gamma).
        auto gather = [&](int b, float* ny) {
            if (b >= nb) {
#pragma unroll
                for (int k = 0; k < 16; ++k) ny[k] = 0.0f;
                return;
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const uint4 w4 = *reinterpret_cast<const uint4*>(pg + 4 * (k4 * nb + b));
                const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float xv = bf16lo(xs[wv[t] & 0xffffu]);
                    const float g = __uint_as_float(wv[t] & 0xffff0000u);
                    ny[4 * k4 + t] = (xv * rs) * -g;
                }
            }
        };
        for (int b0 = lane; b0 < nb; b0 += 64) {
            const int b1 = b0 + 32;
            float2 n[16];
            {
                float y0[16], y1[16];
                gather(b0, y0);
                gather(b1, y1);
#pragma unroll
                for (int k = 0; k < 16; ++k) n[k] = make_float2(y0[k], y1[k]);
            }
            const float2 am = amax_pair(n);
            if constexpr (AMAX_ONLY) {
                my_amax = fmaxf(my_amax, b1 < nb ? fmaxf(am.x, am.y) : am.x);
                pin(my_amax);
                continue;
            } else {
                uint32_t w[4];
                const uint32_t e2 = nvfp4_unit<true, false>(n, am, ctx, tab, 1.0f, w);
                uint8_t* cp = p.codes + row * kcs;
                *reinterpret_cast<uint2*>(cp + 8 * b0) = make_uint2(w[0], w[1]);
                if (b1 < nb) *reinterpret_cast<uint2*>(cp + 8 * b1) = make_uint2(w[2], w[3]);
                if (p.swizzled) {
                    p.scales[swizzle_offset(row, b0, nC)] = (uint8_t)(e2 & 0xffu);
                    if (b1 < nb) p.scales[swizzle_offset(row, b1, nC)] = (uint8_t)(e2 >> 8);
                } else {
                    p.scales[row * nsc + b0] = (uint8_t)(e2 & 0xffu);
                    if (b1 < nb) p.scales[row * nsc + b1] = (uint8_t)(e2 >> 8);
                }
                // 3. residuals of the outlier positions of the two blocks
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = h ? b1 : b0;
                    if (b >= nb) continue;
                    const uint32_t m = omask[b];
                    if (m == 0u) continue;
                    const float es = e4m3_decode(h ? (e2 >> 8) : (e2 & 0xffu));
#pragma unroll
                    for (int k = 0; k < 16; k += 2) {
                        // two codes (one byte), E2M1 values, dequantized primary
                        const uint32_t byte = (w[2 * h + (k >> 3)] >> (4 * (k & 7))) & 0xffu;
                        const float2 cv = e2m1x2_decode(byte);
                        const float y0 = -(h ? n[k].y : n[k].x), y1 = -(h ? n[k + 1].y : n[k + 1].x);
                        if (m & (1u << k)) res[max(0, (int)oidx[16 * b + k])] = y0 - (cv.x * es) * s_t;
                        if (m & (2u << k)) res[max(0, (int)oidx[16 * b + k + 1])] = y1 - (cv.y * es) * s_t;
                    }
                }
            }
        }
        if constexpr (!AMAX_ONLY) {
            __syncwarp();
            // residual blocks: slots 16j..16j+15 -> columns K + 16j
            for (int j0 = lane; 16 * j0 < S; j0 += 64) {
                const int j1 = j0 + 32;
                const bool has1 = 16 * j1 < S;
                float2 n[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float r0 = res[rslot[16 * j0 + k]];
                    const float r1 = has1 ? res[rslot[16 * j1 + k]] : 0.0f;
                    n[k] = make_float2(-r0, -r1);
                }
                uint32_t w[4];
                const uint32_t e2 = nvfp4_unit<true, false>(n, amax_pair(n), ctx, tab, 1.0f, w);
                uint8_t* cp = p.codes + row * kcs + p.K / 2;
                *reinterpret_cast<uint2*>(cp + 8 * j0) = make_uint2(w[0], w[1]);
                if (has1) *reinterpret_cast<uint2*>(cp + 8 * j1) = make_uint2(w[2], w[3]);
                const int64_t c0 = nb + j0, c1 = nb + j1;
                if (p.swizzled) {
                    p.scales[swizzle_offset(row, c0, nC)] = (uint8_t)(e2 & 0xffu);
                    if (has1) p.scales[swizzle_offset(row, c1, nC)] = (uint8_t)(e2 >> 8);
                } else {
                    p.scales[row * nsc + c0] = (uint8_t)(e2 & 0xffu);
                    if (has1) p.scales[row * nsc + c1] = (uint8_t)(e2 >> 8);
                }
            }
        }
        // Every value read from the row buffer is consumed by the stores (or
        // the maximum) above, which issue before the refill below; the residual
        // buffer is rewritten for the next row only after this warp barrier.
        __syncwarp();
        if (lane == 0 && i + SR < n_my) issue(i + SR);
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_amax = fmaxf(my_amax, __shfl_xor_sync(0xffffffffu, my_amax, o));
        __syncthreads();
        if (lane == 0) red[warp] = my_amax;
        __syncthreads();
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < nthreads / 32; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

}  // namespace fp4q
