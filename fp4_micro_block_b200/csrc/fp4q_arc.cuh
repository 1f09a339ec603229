// fp4q_arc.cuh -- ARCQuant fused kernel for sm_100a: channel reorder + RMSNorm
// + primary NVFP4 quantization + NVFP4 quantization of the residual of the
// outlier channels, written as one [primary K | residual S] GEMM operand
// (ARCQuant summary, "Methodologie" items 1-5).
//
// One CTA of K/16 threads processes one row at a time; thread b owns output
// block b (reordered positions 16b..16b+15) and keeps that block's channel
// indices and gamma values in registers for the whole kernel.  Rows stream
// through a ring of kArcStages shared-memory buffers filled by 1-D bulk copies
// (TMA) that complete on per-stage mbarriers.
#pragma once

#include "fp4q_device.cuh"

namespace fp4q {

constexpr int kArcStages = 4;

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
};

// Shared-memory layout: [stages: kArcStages * K bf16][res: K fp32][flags: K/32 u32]
//                       [red: 32 fp32][bars: kArcStages u64]
template <bool AMAX_ONLY, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT <= 256 ? 2 : 1) arc_kernel(const ArcParams p) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                               ~uintptr_t(127));
    const int K = (int)p.K;
    const int nb = K / 16;
    const uint32_t row_bytes = (uint32_t)K * 2u;
    uint8_t* stages = smem;
    float* res = reinterpret_cast<float*>(smem + kArcStages * row_bytes);
    uint32_t* flags = reinterpret_cast<uint32_t*>(res + K);
    float* red = reinterpret_cast<float*>(flags + (K + 31) / 32);
    uint64_t* bars = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(red + 32) + 7) & ~uintptr_t(7));

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads >> 5;
    const bool own = tid < nb;

    // This thread's block: channel indices and gamma (fp32), kept for all rows.
    int ch[16];
    float gam[16];
    bool bad_index = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        int c = own ? p.perm[16 * tid + i] : 0;
        if ((unsigned)c >= (unsigned)K) {  // not a channel: clamp, flag
            bad_index = true;
            c = 0;
        }
        ch[i] = c;
        gam[i] = own ? __uint_as_float((uint32_t)p.gamma[c] << 16) : 0.0f;
    }
    // Outlier flags per reordered position (residual exchange), and the residual
    // block this thread quantizes.
    for (int i = tid; i < (K + 31) / 32; i += nthreads) flags[i] = 0u;
    if (tid == 0)
        for (int s = 0; s < kArcStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
    __syncthreads();
    for (int64_t i = tid; i < p.S; i += nthreads) {
        int q = p.outliers[i];
        if ((unsigned)q >= (unsigned)K) {
            bad_index = true;
            q = 0;
        }
        atomicOr(&flags[q >> 5], 1u << (q & 31));
    }
    if (bad_index) atomicOr(&g_device_error, kErrBadIndex);
    if (tid == 0) fence_barrier_init();
    const bool res_owner = (int64_t)tid < p.S / 16;
    __syncthreads();

    float s_t = 0.0f;
    if constexpr (!AMAX_ONLY) {
        if (p.dynamic) {
            float m = 0.0f;
            for (int i = tid; i < p.n_partials; i += nthreads) m = fmaxf(m, p.partials[i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[warp] = m;
            __syncthreads();
            m = 0.0f;
            for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[w]);
            __syncthreads();
            s_t = __fdiv_rn(m, 2688.0f);
            if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = s_t;
        } else {
            s_t = *p.tensor_scale;
        }
    }

    const int64_t n_my = p.M > (int64_t)blockIdx.x ? (p.M - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto issue = [&](int64_t i) {
        const int64_t row = blockIdx.x + i * (int64_t)gridDim.x;
        const uint32_t st = (uint32_t)(i % kArcStages);
        const uint32_t bar = smem_u32(&bars[st]);
        mbar_arrive_expect_tx(bar, row_bytes);
        bulk_load_1d(smem_u32(stages + st * row_bytes), p.x + row * p.ldx_bytes, row_bytes, bar);
    };
    if (tid == 0)
        for (int64_t i = 0; i < min64(kArcStages, n_my); ++i) issue(i);

    const int64_t KS = p.K + p.S;
    float my_amax = 0.0f;

    for (int64_t i = 0; i < n_my; ++i) {
        const uint32_t st = (uint32_t)(i % kArcStages);
        const bool ok = mbar_wait(smem_u32(&bars[st]), (uint32_t)((i / kArcStages) & 1));
        if (!bar_and(1, nthreads, ok)) {
            if (tid == 0) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                for (int64_t k = i; k < min64(n_my, i + kArcStages); ++k)
                    (void)mbar_wait(smem_u32(&bars[k % kArcStages]), (uint32_t)((k / kArcStages) & 1));
            }
            return;
        }
        if (tid == 0 && i >= 1 && i - 1 + kArcStages < n_my) issue(i - 1 + kArcStages);
        const int64_t row = blockIdx.x + i * (int64_t)gridDim.x;
        const uint16_t* xs = reinterpret_cast<const uint16_t*>(stages + st * row_bytes);

        // Sum of squares of the row (natural order, 8 channels per step).
        float ss = 0.0f;
        for (int k = 8 * tid; k < K; k += 8 * nthreads) {
            uint4 q = *reinterpret_cast<const uint4*>(xs + k);
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
        if (lane == 0) red[warp] = ss;
        bar_sync(3, nthreads);
        float tot = 0.0f;
        for (int w = 0; w < nwarps; ++w) tot += red[w];
        const float rs = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)K) + p.eps));

        // Reorder + normalise this thread's block.
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = (bf16lo(xs[ch[k]]) * rs) * gam[k];
        const float amax = amax16(v);

        if constexpr (AMAX_ONLY) {
            if (own) my_amax = fmaxf(my_amax, amax);
            bar_sync(3, nthreads);  // red[] is rewritten by the next row
            continue;
        } else {
            uint32_t e = 0;
            if (own) {
                uint32_t w0, w1;
                e = nvfp4_block16(v, amax, s_t, w0, w1);
                *reinterpret_cast<uint2*>(p.codes + row * (KS / 2) + 8 * tid) = make_uint2(w0, w1);
                if (p.swizzled) p.scales[swizzle_offset(row, tid, (KS / 16 + 3) / 4)] = (uint8_t)e;
                else p.scales[row * (KS / 16) + tid] = (uint8_t)e;
                // Residual of flagged positions: y - (E2M1val * E4M3val) * s_t.
                const uint32_t fl = (flags[(16 * tid) >> 5] >> ((16 * tid) & 31)) & 0xffffu;
                if (fl) {
                    const float ev = e4m3_decode(e);
                    uint32_t cw[2] = {w0, w1};
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        if (fl & (1u << k)) {
                            const uint32_t c = (cw[k >> 3] >> (4 * (k & 7))) & 15u;
                            const float cv = e2m1x2_decode(c).x;
                            const float dq = (cv * ev) * s_t;
                            res[16 * tid + k] = v[k] - dq;
                        }
                    }
                }
            }
            bar_sync(3, nthreads);  // residuals visible; red[] free again
            if (res_owner) {
                float rv[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const unsigned q = (unsigned)__ldg(p.outliers + 16 * tid + k);
                    rv[k] = res[q < (unsigned)K ? q : 0u];
                }
                uint32_t w0, w1;
                const uint32_t er = nvfp4_block16(rv, amax16(rv), s_t, w0, w1);
                *reinterpret_cast<uint2*>(p.codes + row * (KS / 2) + p.K / 2 + 8 * tid) =
                    make_uint2(w0, w1);
                const int64_t c = p.K / 16 + tid;
                if (p.swizzled) p.scales[swizzle_offset(row, c, (KS / 16 + 3) / 4)] = (uint8_t)er;
                else p.scales[row * (KS / 16) + c] = (uint8_t)er;
            }
            // res[] is rewritten for the next row only after the next row's first
            // barrier, which every residual owner reaches after finishing here.
        }
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_amax = fmaxf(my_amax, __shfl_xor_sync(0xffffffffu, my_amax, o));
        __syncthreads();
        if (lane == 0) red[warp] = my_amax;
        __syncthreads();
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

inline int arc_smem_bytes(int64_t K) {
    return 128 + kArcStages * (int)K * 2 + (int)K * 4 + (int)((K + 31) / 32) * 4 + 32 * 4 + 8 +
           kArcStages * 8 + 16;
}

}  // namespace fp4q
