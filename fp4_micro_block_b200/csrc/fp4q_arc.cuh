// fp4q_arc.cuh -- ARCQuant fused kernel for sm_100a: channel reorder + RMSNorm
// + primary quantization + quantization of the residual of the outlier
// channels, written as one [primary K | residual S] GEMM operand (ARCQuant
// summary, "Methodologie" items 1-5), in NVFP4, MXFP4 or INT4
// ("Generalisabilite": the scheme carries over to MXFP4 and INT4; INT4 is the
// NVFP4 container with the integers -7..7 as the grid).
//
// The warps of a pair slot own a PAIR of rows at a time (two warps for NVFP4
// and INT4, one for MXFP4 and for the amax pre-pass): there is no CTA-wide
// barrier on the path, only a named barrier between the warps of a pair.  They
// stream their row pairs through a shared buffer of 4K bytes (K channels),
// filled by two 1-D bulk copies (row 0 in the first half, row 1 in the second),
// and split steps 1 and 2 of a pair between them (alternate 16-byte chunks,
// alternate 32-block groups), which halves the registers a warp holds and
// doubles the warps an SM runs.  Per pair:
//   1. natural order (conflict-free 16-byte reads of both rows): the sum of
//      squares of each row, and one 32-bit word per channel holding the bf16 of
//      row 0 (low half) and of row 1 (high half), written IN PLACE: lane l
//      reads channels 8j..8j+7 of both rows (16 bytes at 16 j of each half)
//      and writes their 8 words back to the same 32 bytes, channels 8j..8j+3
//      into the first half and 8j+4..8j+7 into the second, so the word of
//      channel c sits at 16 (c >> 3) + 4 (c & 3) + ((c >> 2) & 1) * 2K;
//   2. reordered order: lane l of warp w owns the output blocks
//      b = l + 32 w, l + 32 w + 64, ..., one per step; one shared-memory load
//      per position gathers that position's channel for both rows, a packed
//      multiply applies -gamma of the channel, and the two rows' blocks are
//      quantized side by side (NVFP4 and INT4: one unit of two 16-blocks;
//      MXFP4: one 32-block unit per row).  The RMS factor rs of each row is not
//      applied per element: it scales the block maximum and the quotient
//      multiplier of its row (the "fold" of the unit quantizers), so
//      y = z * rs with z = x * gamma;
//   3. at the outlier positions (a bit mask per 16-position group) the
//      residual y - dequant(primary) goes to the pair's slot buffer in position
//      order (a block whose positions are all outliers, as the reorder makes
//      them, in straight-line code); after the pair barrier the buffer takes
//      the next pair, and the residual blocks are quantized (residual column j
//      reads the slot of outlier j; contiguously when the outlier list is in
//      position order): up to 32 blocks all by the pair's last warp in one
//      pass, more alternating between the warps.
// Each warp waits for its pair's copies; the other pairs of the SM (10 for
// NVFP4 and INT4, 12 for MXFP4, one buffer each) hide that latency, and each
// slot's next pair is prefetched into L2 when the current one lands, so the
// copy issued after step 2 reads L2.
// Per CTA (built once): for every position q a 32-bit word (byte offset of the
// word of channel perm[q] << 16 | bf16 gamma of that channel), laid out so that
// the 16-byte loads of 32 lanes (blocks b = lane + 32 i) are consecutive; per
// 16-position group the outlier bit mask and the number of outlier positions
// before the group; the slot of every residual column; the NVFP4 scale table
// (d, RN(1/d)).  The amax pre-pass of the dynamic tensor scale streams the
// rows in natural order through two buffers per warp.
#pragma once

#include "fp4q_quant.cuh"

namespace fp4q {

// Launch bounds (warps per CTA, one CTA per SM).  The NVFP4 quantizer runs up to
// 10 row pairs of two warps (one 16-block of both rows in registers at a time,
// at most 102 registers a thread); the MXFP4 quantizer, whose 32-blocks hold
// twice the values, one warp per pair (12 pairs); the amax pre-pass is a light
// streaming loop with one warp per pair.
template <int FMT, bool AMAX_ONLY>
__host__ __device__ constexpr int arc_max_warps() { return AMAX_ONLY ? 16 : FMT == FMT_MXFP4 ? 12 : 20; }
template <int FMT, bool AMAX_ONLY>
__host__ __device__ constexpr int arc_warps_per_pair() { return (AMAX_ONLY || FMT == FMT_MXFP4) ? 1 : 2; }

struct ArcParams {
    int64_t M, K, S;
    const int32_t* perm;      // [K]
    const int32_t* outliers;  // [S] reordered positions
    const uint16_t* gamma;    // bf16 [K]
    const uint8_t* x;         // bf16 rows, byte stride ldx_bytes
    int64_t ldx_bytes;
    float eps;
    uint8_t* codes;           // [M, (K+S)/2]
    uint8_t* scales;          // [M, (K+S)/B] or swizzled
    float* tensor_scale;      // NVFP4 only
    float* partials;
    int n_partials;
    int swizzled;
    int dynamic;
    int warps;                // warps per CTA (arc_warps_per_pair per row pair)
};

// Shared-memory layout (byte offsets).  CTA part: tab (u32 [K]), om (u32 per
// 16-position group), rslot (u16 [S]), red (f32 [32]), stab (float2 [128]);
// then per pair slot: the pair buffer (2 rows of bf16, then the interleaved
// words; the pre-pass: two stages of 2 rows), residuals (f32 [2][S]), the two
// warps' partial sums of squares, mbarriers.
struct ArcLayout {
    int tab, om, rslot, red, stab, warp0, warp_bytes, land, res, bar, total;
};

__host__ __device__ inline int arc_al(int64_t v) { return (int)((v + 127) / 128 * 128); }

template <bool AMAX_ONLY>
__host__ __device__ inline ArcLayout arc_layout(int64_t K, int64_t S, int slots) {
    ArcLayout l;
    int off = 0;
    l.tab = off;
    off += AMAX_ONLY ? 0 : arc_al(K * 4);
    l.om = off;
    off += AMAX_ONLY ? 0 : arc_al((K / 16) * 4);
    l.rslot = off;
    off += AMAX_ONLY ? 0 : arc_al(S * 2);
    l.red = off;
    off += 128;
    l.stab = off;
    off += AMAX_ONLY ? 0 : 128 * 8;
    l.warp0 = off;
    const int stages = AMAX_ONLY ? 2 : 1;
    int w = 0;
    l.land = w;
    w += arc_al(stages * 2 * K * 2);
    l.res = w;
    w += AMAX_ONLY ? 0 : arc_al(2 * S * 4);
    l.bar = w;  // mbarriers, then the two warps' partial sums (2 x float2) at +64
    w += 128;
    l.warp_bytes = w;
    l.total = off + slots * w + 128;  // + alignment slack of the dynamic buffer
    return l;
}

// Byte offset of the interleaved word of channel c in a pair buffer of K channels.
__host__ __device__ inline uint32_t arc_word_off(uint32_t c, uint32_t K) {
    return 16u * (c >> 3) + 4u * (c & 3u) + ((c >> 2) & 1u) * 2u * K;
}

// Packed f32x2 arithmetic (sm_100a).
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// INT4 codes of the quotients q = n[i] * m of 16 pairs (x: row 0 -> w[0..1],
// y: row 1 -> w[2..3]), optionally clamped to [-7, 7] first: each q is rounded
// to the nearest integer, ties to even, by one IEEE addition of 1.5 * 2^23
// (whose ulp is 1), and the low nibble of the sum's significand is the two's
// complement code.
template <bool CLAMP>
__device__ __forceinline__ void int4_pack_pairs(const float2* n, float2 m, uint32_t (&w)[4]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t a = 0, b = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float2 q = fmul2(n[8 * h + i], m);
            if constexpr (CLAMP) {
                q.x = fminf(fmaxf(q.x, -7.0f), 7.0f);
                q.y = fminf(fmaxf(q.y, -7.0f), 7.0f);
            }
            const float2 k = __fadd2_rn(q, make_float2(12582912.0f, 12582912.0f));  // both rows at once
            const uint32_t ka = __float_as_uint(k.x), kb = __float_as_uint(k.y);
            asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(a) : "r"(ka), "r"(a), "r"(4 * i));
            asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(b) : "r"(kb), "r"(b), "r"(4 * i));
        }
        w[h] = a;
        w[2 + h] = b;
    }
}

// NVFP4 rule for the two blocks of a unit (component x: row 0, y: row 1) with a
// fold per component: the unit holds -z and v = z * fold.  Scale bytes from
// RN(RN(amax(v) * RN(1/6)) * RN(1/s)) and quotients z * RN(RN(1/d) * fold), as
// in nvfp4_unit's table path.  stab[e] = (d, RN(1/d)) for the tensor scale s.
// INT4: the same with RN(1/7) and the integer grid.
template <bool INT4>
__device__ __forceinline__ uint32_t arc_nvfp4_unit(const float2* n, float2 am, const ScaleCtx& c,
                                                   const float2* stab, float2 fold, uint32_t (&w)[4]) {
    am = fmul2(am, fold);
    const uint32_t b0 = __float_as_uint(am.x), b1 = __float_as_uint(am.y);
    const uint32_t tiny = __float_as_uint(0x1p-90f);
    const bool in_range = c.fast && (b0 - 1u) >= tiny - 1u && (b1 - 1u) >= tiny - 1u &&
                          fmaxf(am.x, am.y) <= c.am_max;
    if (!in_range) {
        const uint32_t e0 = nvfp4_block_ieee<false, INT4>(n, am.x, c.s, fold.x, w[0], w[1]);
        const uint32_t e1 = nvfp4_block_ieee<true, INT4>(n, am.y, c.s, fold.y, w[2], w[3]);
        return e0 | (e1 << 8);
    }
    const float k = __uint_as_float(INT4 ? 0x3e124925u : 0x3e2aaaabu);  // RN(1/7), RN(1/6)
    const uint32_t e2 = e4m3x2_encode(fmul2(fmul2(am, make_float2(k, k)), make_float2(c.rs.rn, c.rs.rn)));
    const float2 t0 = stab[e2 & 0xffu], t1 = stab[e2 >> 8];
    const float2 m = fmul2(make_float2(-t0.y, -t1.y), fold);  // n holds -z
    if constexpr (INT4) {
        // A scale byte in the normal range below 448 (8 .. 0x7d: no saturation,
        // relative rounding error at most 2^-4) bounds every |q| by about
        // 7 / (1 - 2^-4) < 7.47, which rounds into -7..7 by itself; other
        // blocks are clamped to [-7, 7] first.
        if ((e2 & 0xffu) - 8u < 0x76u && (e2 >> 8) - 8u < 0x76u) int4_pack_pairs<false>(n, m, w);
        else int4_pack_pairs<true>(n, m, w);
    } else {
        float q0[16], q1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float2 q = fmul2(n[i], m);
            q0[i] = q.x;
            q1[i] = q.y;
        }
        w[0] = e2m1_pack8(q0);
        w[1] = e2m1_pack8(q0 + 8);
        w[2] = e2m1_pack8(q1);
        w[3] = e2m1_pack8(q1 + 8);
    }
    if (t0.x == 0.0f) w[0] = w[1] = 0u;  // zero block scale: all codes +0
    if (t1.x == 0.0f) w[2] = w[3] = 0u;
    return e2;
}

// Block maxima |v| of the two components of 16 pairs as a depth-3 tree of
// three-input maxima (8 instructions per component, like a chain, but a third
// of its latency).
__device__ __forceinline__ float2 amax_pair_tree(const float2* n) {
    float a[6], b[6];
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        a[i] = max3(fabsf(n[3 * i].x), fabsf(n[3 * i + 1].x), fabsf(n[3 * i + 2].x));
        b[i] = max3(fabsf(n[3 * i].y), fabsf(n[3 * i + 1].y), fabsf(n[3 * i + 2].y));
    }
    a[5] = fabsf(n[15].x);
    b[5] = fabsf(n[15].y);
    return make_float2(fmaxf(max3(a[0], a[1], a[2]), max3(a[3], a[4], a[5])),
                       fmaxf(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5])));
}

// Shared-memory loads by 32-bit shared address (the gather's table words and
// pair words).
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    return __byte_perm(a, b, sel);
}

// Hint: bring a 16-byte aligned range (size a multiple of 16) of global memory
// into L2; no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Offset of row `row`'s scales: linear, the row's start; tiled (128 x 4 tiles),
// the part of the tile offset that depends on the row only.
__device__ __forceinline__ int64_t scale_row_base(const ArcParams& p, int64_t row, int64_t nsc, int64_t nC) {
    return p.swizzled ? (row >> 7) * nC * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 : row * nsc;
}

template <int FMT, bool AMAX_ONLY>
__global__ void __launch_bounds__(arc_max_warps<FMT, AMAX_ONLY>() * 32, 1) arc_kernel(const ArcParams p) {
    static_assert(FMT == FMT_NVFP4 || ((FMT == FMT_MXFP4 || FMT == FMT_INT4) && !AMAX_ONLY),
                  "formats of the ARC path");
    constexpr bool I4 = FMT == FMT_INT4;
    constexpr int B = FMT == FMT_MXFP4 ? 32 : 16;  // block size
    constexpr int Q = B / 4;                       // 16-byte table quads per block
    constexpr int SR = AMAX_ONLY ? 2 : 1;          // landing stages per pair slot
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = align_shared<128>(smem_raw);
    constexpr int WPP = arc_warps_per_pair<FMT, AMAX_ONLY>();
    const int K = (int)p.K, S = (int)p.S, nbB = K / B, ng = K / 16, W = p.warps, NP = W / WPP;
    const ArcLayout L = arc_layout<AMAX_ONLY>(p.K, p.S, NP);
    const uint32_t row_bytes = (uint32_t)K * 2u;
    uint32_t* tab = reinterpret_cast<uint32_t*>(smem + L.tab);
    uint32_t* om = reinterpret_cast<uint32_t*>(smem + L.om);
    uint16_t* rslot = reinterpret_cast<uint16_t*>(smem + L.rslot);
    float* red = reinterpret_cast<float*>(smem + L.red);
    float2* stab = reinterpret_cast<float2*>(smem + L.stab);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;

    // ---- this pair slot's buffer and barriers (warps WPP ps .. WPP ps + WPP - 1);
    // its first pairs' copies overlap the building of the CTA tables below
    const int ps = warp / WPP, sub = warp % WPP;
    uint8_t* const wb = smem + L.warp0 + (size_t)ps * L.warp_bytes;
    uint64_t* const bars = reinterpret_cast<uint64_t*>(wb + L.bar);
    float2* const part = reinterpret_cast<float2*>(wb + L.bar + 64);  // the warps' partial sums
    // The warps of a pair meet at a 64-thread named barrier (id 1 + ps; 0 is the
    // CTA's); a vote on it makes every early exit a joint decision.
    auto pair_sync = [&]() {
        if constexpr (WPP > 1) bar_sync(1 + ps, 32 * WPP);
        else __syncwarp();
    };
    auto pair_all = [&](bool v) -> bool {
        v = __all_sync(0xffffffffu, v);
        if constexpr (WPP > 1) v = bar_and(1 + ps, 32 * WPP, v);
        return v;
    };
    const int64_t P = (p.M + 1) / 2;  // row pairs
    // Each CTA takes a contiguous range of P / gridDim.x pairs (the ranges differ
    // by at most one pair), dealt round-robin to its slots: per-CTA loads stay
    // balanced even when there are only two or three pairs per slot.
    const int64_t p_lo = (int64_t)blockIdx.x * P / gridDim.x, p_hi = ((int64_t)blockIdx.x + 1) * P / gridDim.x;
    const int64_t gw = p_lo + ps, nw = NP;
    const int64_t n_my = p_hi > gw ? (p_hi - 1 - gw) / nw + 1 : 0;
    uint8_t* const land = wb + L.land;
    auto issue = [&](int64_t i) {  // lane 0 of the first warp: pair i of the slot into stage i % SR
        const int64_t r0 = 2 * (gw + i * nw);
        const bool two = r0 + 1 < p.M;
        const uint32_t bar = smem_u32(&bars[i % SR]);
        uint8_t* dst = land + (i % SR) * 2 * row_bytes;
        // the buffer was last written through the generic proxy (interleaved
        // words): order those writes before the asynchronous copies
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, two ? 2 * row_bytes : row_bytes);
        bulk_load_1d(smem_u32(dst), p.x + r0 * p.ldx_bytes, row_bytes, bar);
        if (two) bulk_load_1d(smem_u32(dst + row_bytes), p.x + (r0 + 1) * p.ldx_bytes, row_bytes, bar);
    };
    if (sub == 0 && lane == 0) {  // (the CTA barriers below publish the initialisation)
        for (int k = 0; k < SR; ++k) mbar_init(smem_u32(&bars[k]), 1);
        fence_barrier_init();
        for (int64_t i = 0; i < min64(SR, n_my); ++i) issue(i);
    }
    __syncwarp();

    // ---- per-CTA tables
    float s_t = 0.0f;
    int slots_in_order = 1;  // residual column i takes slot i (outlier list in position order)
    if constexpr (!AMAX_ONLY) {
        bool bad_index = false;
        // word of position q = B b + 4 k + t at index 4 (k nbB + b) + t; four
        // positions per thread at a time, so that their loads overlap
        for (int q0 = tid; q0 < K; q0 += 4 * nthreads) {
            int c[4];
            uint32_t g[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = q0 + u * nthreads;
                c[u] = q < K ? __ldg(p.perm + q) : 0;
                if ((unsigned)c[u] >= (unsigned)K) {  // not a channel: clamp, flag
                    bad_index = true;
                    c[u] = 0;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) g[u] = __ldg(p.gamma + c[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = q0 + u * nthreads;
                if (q >= K) continue;
                const int b = q / B, k = (q % B) >> 2, t = q & 3;
                tab[4 * (k * nbB + b) + t] = (arc_word_off((uint32_t)c[u], (uint32_t)K) << 16) | g[u];
            }
        }
        for (int g = tid; g < ng; g += nthreads) om[g] = 0u;
        __syncthreads();
        for (int i = tid; i < S; i += nthreads) {  // outlier bit of every listed position
            int q = p.outliers[i];
            if ((unsigned)q >= (unsigned)K) {
                bad_index = true;
                q = 0;
            }
            atomicOr(&om[q >> 4], 1u << (q & 15));
        }
        __syncthreads();
        if (warp == 0) {  // outlier positions before each group: warp-wide exclusive scan
            const int per = (ng + 31) / 32, g0 = lane * per;
            int cnt = 0;
            for (int g = g0; g < min(ng, g0 + per); ++g) cnt += __popc(om[g] & 0xffffu);
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            int run = inc - cnt;
            for (int g = g0; g < min(ng, g0 + per); ++g) {
                const uint32_t m = om[g] & 0xffffu;
                om[g] = m | ((uint32_t)run << 16);
                run += __popc(m);
            }
        }
        __syncthreads();
        for (int i = tid; i < S; i += nthreads) {  // slot (position rank) of residual column i
            const unsigned q0 = (unsigned)p.outliers[i], q = q0 < (unsigned)K ? q0 : 0u;
            const uint32_t w = om[q >> 4];
            const uint32_t sl = (w >> 16) + __popc(w & ((1u << (q & 15)) - 1u));
            rslot[i] = (uint16_t)sl;
            slots_in_order &= (int)(sl == (uint32_t)i);
        }
        if (bad_index) atomicOr(&g_device_error, kErrBadIndex);
        if constexpr (FMT == FMT_NVFP4 || I4) {
            if (p.dynamic) {
                s_t = tensor_scale_from_partials(p.partials, p.n_partials, red, I4 ? 3136.0f : 2688.0f);
                if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = s_t;
            } else {
                s_t = *p.tensor_scale;
            }
            for (int e = tid; e < 128; e += nthreads) {
                const float d = (e < 127) ? e4m3_decode((uint32_t)e) * s_t : 0.0f;
                const bool ok = d >= 0x1p-100f && d <= 0x1p100f;
                stab[e] = make_float2(d, ok ? __frcp_rn(d) : 0.0f);
            }
        }
    }
    const bool in_order = __syncthreads_and(slots_in_order) != 0;

    const ScaleCtx ctx = make_ctx(s_t);
    const int64_t KS = p.K + p.S, kcs = KS / 2, nsc = KS / B, nC = (nsc + 3) / 4;
    float* const res = reinterpret_cast<float*>(wb + L.res);
    float my_amax = 0.0f;

    for (int64_t i = 0; i < n_my; ++i) {
        const bool ok = mbar_wait(smem_u32(&bars[i % SR]), (uint32_t)((i / SR) & 1));
        if (!pair_all(ok)) {
            if (sub == 0 && lane == 0) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                for (int64_t k = i; k < min64(n_my, i + SR); ++k)
                    (void)mbar_wait(smem_u32(&bars[k % SR]), (uint32_t)((k / SR) & 1));
            }
            break;
        }
        // the slot's next pair into L2 now, so that its copy (issued once this
        // pair's buffer is consumed) does not wait on DRAM
        if (sub == 0 && lane == 0 && i + SR < n_my) {
            const int64_t rn = 2 * (gw + (i + SR) * nw);
            bulk_prefetch_l2(p.x + rn * p.ldx_bytes, row_bytes);
            if (rn + 1 < p.M) bulk_prefetch_l2(p.x + (rn + 1) * p.ldx_bytes, row_bytes);
        }
        const int64_t r0 = 2 * (gw + i * nw);
        const bool two = r0 + 1 < p.M;
        uint8_t* const l0 = land + (i % SR) * 2 * row_bytes;
        uint8_t* const l1 = l0 + row_bytes;

        float2 ss = make_float2(0.0f, 0.0f), sq = make_float2(0.0f, 0.0f);
        if constexpr (AMAX_ONLY) {
            // natural order: sums of squares and max |x gamma| of both rows
            float2 zmax = make_float2(0.0f, 0.0f);
            for (int c = 4 * lane; c < K; c += 128) {
                const uint2 a = *reinterpret_cast<const uint2*>(l0 + 2 * c);
                const uint2 b = two ? *reinterpret_cast<const uint2*>(l1 + 2 * c) : make_uint2(0u, 0u);
                const float2 v0 = make_float2(bf16lo(a.x), bf16lo(b.x)), v1 = make_float2(bf16hi(a.x), bf16hi(b.x));
                const float2 v2 = make_float2(bf16lo(a.y), bf16lo(b.y)), v3 = make_float2(bf16hi(a.y), bf16hi(b.y));
                ss = ffma2(v0, v0, ss);
                sq = ffma2(v1, v1, sq);
                ss = ffma2(v2, v2, ss);
                sq = ffma2(v3, v3, sq);
                // gamma in natural order (2-byte aligned: 16-bit loads)
                const float g0 = bf16lo(__ldg(p.gamma + c)), g1 = bf16lo(__ldg(p.gamma + c + 1));
                const float g2 = bf16lo(__ldg(p.gamma + c + 2)), g3 = bf16lo(__ldg(p.gamma + c + 3));
                const float2 z0 = fmul2(v0, dup2(g0)), z1 = fmul2(v1, dup2(g1));
                const float2 z2 = fmul2(v2, dup2(g2)), z3 = fmul2(v3, dup2(g3));
                zmax.x = fmaxf(zmax.x, max3(fabsf(z0.x), fabsf(z1.x), fmaxf(fabsf(z2.x), fabsf(z3.x))));
                zmax.y = fmaxf(zmax.y, max3(fabsf(z0.y), fabsf(z1.y), fmaxf(fabsf(z2.y), fabsf(z3.y))));
            }
            ss = make_float2(ss.x + sq.x, ss.y + sq.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                ss.x += __shfl_xor_sync(0xffffffffu, ss.x, o);
                ss.y += __shfl_xor_sync(0xffffffffu, ss.y, o);
                zmax.x = fmaxf(zmax.x, __shfl_xor_sync(0xffffffffu, zmax.x, o));
                zmax.y = fmaxf(zmax.y, __shfl_xor_sync(0xffffffffu, zmax.y, o));
            }
            const float rK = (float)K;
            const float2 rs = make_float2(__frcp_rn(__fsqrt_rn(__fdiv_rn(ss.x, rK) + p.eps)),
                                          __frcp_rn(__fsqrt_rn(__fdiv_rn(ss.y, rK) + p.eps)));
            // every value read from the stage is consumed above: refill it
            pair_sync();
            if (sub == 0 && lane == 0 && i + SR < n_my) issue(i + SR);
            my_amax = fmaxf(my_amax, zmax.x * rs.x);
            if (two) my_amax = fmaxf(my_amax, zmax.y * rs.y);
        } else {
            // 1. natural order, in place: sums of squares and the interleaved words
#pragma unroll 4
            for (int j = lane + 32 * sub; 8 * j < K; j += 32 * WPP) {
                const uint4 a = *reinterpret_cast<const uint4*>(l0 + 16 * j);
                const uint4 b = two ? *reinterpret_cast<const uint4*>(l1 + 16 * j) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 lo = make_float2(bf16lo(av[q]), bf16lo(bv[q]));
                    const float2 hi = make_float2(bf16hi(av[q]), bf16hi(bv[q]));
                    ss = ffma2(lo, lo, ss);
                    sq = ffma2(hi, hi, sq);
                }
                *reinterpret_cast<uint4*>(l0 + 16 * j) =
                    make_uint4(prmt(a.x, b.x, 0x5410u), prmt(a.x, b.x, 0x7632u), prmt(a.y, b.y, 0x5410u),
                               prmt(a.y, b.y, 0x7632u));
                *reinterpret_cast<uint4*>(l1 + 16 * j) =
                    make_uint4(prmt(a.z, b.z, 0x5410u), prmt(a.z, b.z, 0x7632u), prmt(a.w, b.w, 0x5410u),
                               prmt(a.w, b.w, 0x7632u));
            }
            ss = make_float2(ss.x + sq.x, ss.y + sq.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                ss.x += __shfl_xor_sync(0xffffffffu, ss.x, o);
                ss.y += __shfl_xor_sync(0xffffffffu, ss.y, o);
            }
            if constexpr (WPP > 1) {
                if (lane == 0) part[sub] = ss;
                pair_sync();  // both warps' interleaved words and partial sums are written
                const float2 o = part[sub ^ 1];
                ss = make_float2(ss.x + o.x, ss.y + o.y);  // the same sum in both warps
            } else {
                __syncwarp();  // every lane's interleaved words are written
            }
            const float rK = (float)K;
            const float2 rs = make_float2(__frcp_rn(__fsqrt_rn(__fdiv_rn(ss.x, rK) + p.eps)),
                                          __frcp_rn(__fsqrt_rn(__fdiv_rn(ss.y, rK) + p.eps)));

            // 2. reordered positions: gather both rows, quantize, store
            const int64_t r1 = r0 + 1;
            uint8_t* cp0 = p.codes + r0 * kcs;
            uint8_t* cp1 = p.codes + r1 * kcs;
            // the two rows' scale bases (linear: the row; tiled: the row's part of
            // the 128 x 4 tile offset) and the column part of a scale's offset
            uint8_t* const sb0 = p.scales + scale_row_base(p, r0, nsc, nC);
            uint8_t* const sb1 = p.scales + scale_row_base(p, r1, nsc, nC);
            auto scol = [&](int64_t c) -> int64_t { return p.swizzled ? ((c >> 2) << 9) + (c & 3) : c; };
            const uint32_t tab_s = smem_u32(tab), l0_s = smem_u32(l0);
            // (-z row 0, -z row 1) of the B positions of block b
            auto gather = [&](int b, float2* v) {
#pragma unroll
                for (int k = 0; k < Q; ++k) {
                    const uint4 tw = lds_v4(tab_s + 16u * (uint32_t)(k * nbB + b));
                    const uint32_t wv[4] = {tw.x, tw.y, tw.z, tw.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint32_t xw = lds_u32(l0_s + (wv[t] >> 16));
                        const float ng_ = -__uint_as_float(wv[t] << 16);
                        v[4 * k + t] = fmul2(make_float2(bf16lo(xw), bf16hi(xw)), dup2(ng_));
                    }
                }
            };
            // quantize + store block b of both rows, and its outlier residuals
            auto emit = [&](int b, const float2* v) {
                if constexpr (FMT == FMT_NVFP4 || I4) {
                    uint32_t w[4];
                    const uint32_t e2 = arc_nvfp4_unit<I4>(v, amax_pair_tree(v), ctx, stab, rs, w);
                    *reinterpret_cast<uint2*>(cp0 + 8 * b) = make_uint2(w[0], w[1]);
                    sb0[scol(b)] = (uint8_t)(e2 & 0xffu);
                    if (two) {
                        *reinterpret_cast<uint2*>(cp1 + 8 * b) = make_uint2(w[2], w[3]);
                        sb1[scol(b)] = (uint8_t)(e2 >> 8);
                    }
                    // 3. residuals of the outlier positions of the block:
                    // y - (grid value * E4M3 value) * s_t, y = z * rs
                    const uint32_t o = om[b];
                    if (o & 0xffffu) {
                        const float es0 = e4m3_decode(e2 & 0xffu), es1 = e4m3_decode(e2 >> 8);
                        auto resid = [&](float nz, float r, float c, float es) { return -nz * r - (c * es) * s_t; };
                        auto pair_at = [&](int k, float2& c0, float2& c1) {  // grid values of k, k + 1 (rows 0, 1)
                            const uint32_t sh = 4 * (k & 7);
                            const uint32_t b0 = (w[k >> 3] >> sh) & 0xffu, b1 = (w[2 + (k >> 3)] >> sh) & 0xffu;
                            c0 = I4 ? int4x2_decode(b0) : e2m1x2_decode(b0);
                            c1 = I4 ? int4x2_decode(b1) : e2m1x2_decode(b1);
                        };
                        const int base = (int)(o >> 16);
                        if ((o & 0xffffu) == 0xffffu && (base & 3) == 0) {
                            // every position of the block is an outlier: slots base .. base + 15
#pragma unroll
                            for (int k = 0; k < 16; k += 4) {
                                float2 c0, c1, d0, d1;
                                pair_at(k, c0, c1);
                                pair_at(k + 2, d0, d1);
                                *reinterpret_cast<float4*>(res + base + k) =
                                    make_float4(resid(v[k].x, rs.x, c0.x, es0), resid(v[k + 1].x, rs.x, c0.y, es0),
                                                resid(v[k + 2].x, rs.x, d0.x, es0), resid(v[k + 3].x, rs.x, d0.y, es0));
                                *reinterpret_cast<float4*>(res + S + base + k) =
                                    make_float4(resid(v[k].y, rs.y, c1.x, es1), resid(v[k + 1].y, rs.y, c1.y, es1),
                                                resid(v[k + 2].y, rs.y, d1.x, es1), resid(v[k + 3].y, rs.y, d1.y, es1));
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; k += 2) {
                                const uint32_t m2 = (o >> k) & 3u;
                                if (m2 == 0u) continue;
                                float2 c0, c1;
                                pair_at(k, c0, c1);
                                const int s0 = base + __popc(o & ((1u << k) - 1u));
                                if (m2 & 1u) {
                                    res[s0] = resid(v[k].x, rs.x, c0.x, es0);
                                    res[S + s0] = resid(v[k].y, rs.y, c1.x, es1);
                                }
                                if (m2 & 2u) {
                                    const int s1 = s0 + (int)(m2 & 1u);
                                    res[s1] = resid(v[k + 1].x, rs.x, c0.y, es0);
                                    res[S + s1] = resid(v[k + 1].y, rs.y, c1.y, es1);
                                }
                            }
                        }
                    }
                } else {  // MXFP4: one 32-block unit per row
                    float2 u0[16], u1[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        u0[k] = make_float2(v[k].x, v[16 + k].x);
                        u1[k] = make_float2(v[k].y, v[16 + k].y);
                    }
                    uint32_t w0[4], w1[4];
                    const uint32_t e0 = mxfp4_unit(u0, rs.x, w0);
                    const uint32_t e1 = mxfp4_unit(u1, rs.y, w1);
                    *reinterpret_cast<uint4*>(cp0 + 16 * b) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                    sb0[scol(b)] = (uint8_t)(e0);
                    if (two) {
                        *reinterpret_cast<uint4*>(cp1 + 16 * b) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                        sb1[scol(b)] = (uint8_t)(e1);
                    }
                    const uint32_t oa = om[2 * b], ob = om[2 * b + 1];
                    if ((oa | ob) & 0xffffu) {
                        const float es0 = e0 ? __uint_as_float(e0 << 23) : __uint_as_float(0x00400000u);
                        const float es1 = e1 ? __uint_as_float(e1 << 23) : __uint_as_float(0x00400000u);
                        auto resid = [&](float nz, float r, float c, float es) { return -nz * r - c * es; };
                        auto pair_at = [&](int kk, float2& c0, float2& c1) {  // grid values of kk, kk + 1
                            const uint32_t sh = 4 * (kk & 7);
                            c0 = e2m1x2_decode((w0[kk >> 3] >> sh) & 0xffu);
                            c1 = e2m1x2_decode((w1[kk >> 3] >> sh) & 0xffu);
                        };
                        const int base = (int)(oa >> 16);
                        if ((oa & ob & 0xffffu) == 0xffffu && (base & 3) == 0) {
                            // every position of the block is an outlier: slots base .. base + 31
#pragma unroll
                            for (int k = 0; k < 32; k += 4) {
                                float2 c0, c1, d0, d1;
                                pair_at(k, c0, c1);
                                pair_at(k + 2, d0, d1);
                                *reinterpret_cast<float4*>(res + base + k) =
                                    make_float4(resid(v[k].x, rs.x, c0.x, es0), resid(v[k + 1].x, rs.x, c0.y, es0),
                                                resid(v[k + 2].x, rs.x, d0.x, es0), resid(v[k + 3].x, rs.x, d0.y, es0));
                                *reinterpret_cast<float4*>(res + S + base + k) =
                                    make_float4(resid(v[k].y, rs.y, c1.x, es1), resid(v[k + 1].y, rs.y, c1.y, es1),
                                                resid(v[k + 2].y, rs.y, d1.x, es1), resid(v[k + 3].y, rs.y, d1.y, es1));
                            }
                        } else {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t o = h ? ob : oa;
#pragma unroll
                                for (int k = 0; k < 16; k += 2) {
                                    const uint32_t m2 = (o >> k) & 3u;
                                    if (m2 == 0u) continue;
                                    const int kk = 16 * h + k;  // position within the block
                                    float2 c0, c1;
                                    pair_at(kk, c0, c1);
                                    const int s0 = (int)(o >> 16) + __popc(o & ((1u << k) - 1u));
                                    if (m2 & 1u) {
                                        res[s0] = resid(v[kk].x, rs.x, c0.x, es0);
                                        res[S + s0] = resid(v[kk].y, rs.y, c1.x, es1);
                                    }
                                    if (m2 & 2u) {
                                        const int s1 = s0 + (int)(m2 & 1u);
                                        res[s1] = resid(v[kk + 1].x, rs.x, c0.y, es0);
                                        res[S + s1] = resid(v[kk + 1].y, rs.y, c1.y, es1);
                                    }
                                }
                            }
                        }
                    }
                }
            };
            // one block of both rows per step; the warps of the pair take
            // alternate groups of 32 blocks
            for (int b = lane + 32 * sub; b < nbB; b += 32 * WPP) {
                float2 va[B];
                gather(b, va);
                emit(b, va);
            }
            // Every residual slot is written, and every value gathered from the
            // buffer has been consumed by the stores above, in both warps: the
            // buffer takes the next pair now, its copy overlapping the residual
            // blocks (which read only the slots; the next pair's first barrier
            // orders them before its residuals are written).
            pair_sync();
            if (sub == 0 && lane == 0 && i + SR < n_my) issue(i + SR);
            // residual blocks: slots of columns B j .. B j + B - 1 -> columns K + B j.
            // Up to 32 blocks all go to the pair's last warp (one pass either way;
            // its partner carried the outlier residuals of the primary blocks),
            // more alternate between the warps.
            const int nrb = S / B;
            const bool last_only = nrb <= 32;
            const int j0 = last_only ? (sub == WPP - 1 ? lane : nrb) : sub + WPP * lane;
            for (int j = j0; j < nrb; j += last_only ? 32 : 32 * WPP) {
                const int64_t col = nbB + j;
                if constexpr (FMT == FMT_NVFP4 || I4) {
                    float2 n[16];
                    if (in_order) {  // slots 16 j .. 16 j + 15
#pragma unroll
                        for (int k = 0; k < 16; k += 4) {
                            const float4 a = *reinterpret_cast<const float4*>(res + 16 * j + k);
                            const float4 c = *reinterpret_cast<const float4*>(res + S + 16 * j + k);
                            n[k] = make_float2(-a.x, -c.x);
                            n[k + 1] = make_float2(-a.y, -c.y);
                            n[k + 2] = make_float2(-a.z, -c.z);
                            n[k + 3] = make_float2(-a.w, -c.w);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int sl = rslot[16 * j + k];
                            n[k] = make_float2(-res[sl], -res[S + sl]);
                        }
                    }
                    uint32_t w[4];
                    const uint32_t e2 = arc_nvfp4_unit<I4>(n, amax_pair_tree(n), ctx, stab, make_float2(1.0f, 1.0f), w);
                    *reinterpret_cast<uint2*>(cp0 + p.K / 2 + 8 * j) = make_uint2(w[0], w[1]);
                    sb0[scol(col)] = (uint8_t)(e2 & 0xffu);
                    if (two) {
                        *reinterpret_cast<uint2*>(cp1 + p.K / 2 + 8 * j) = make_uint2(w[2], w[3]);
                        sb1[scol(col)] = (uint8_t)(e2 >> 8);
                    }
                } else {
                    float2 u0[16], u1[16];
                    if (in_order) {  // slots 32 j .. 32 j + 31
#pragma unroll
                        for (int k = 0; k < 16; k += 4) {
                            const float4 a = *reinterpret_cast<const float4*>(res + 32 * j + k);
                            const float4 b = *reinterpret_cast<const float4*>(res + 32 * j + 16 + k);
                            const float4 c = *reinterpret_cast<const float4*>(res + S + 32 * j + k);
                            const float4 d = *reinterpret_cast<const float4*>(res + S + 32 * j + 16 + k);
                            u0[k] = make_float2(-a.x, -b.x);
                            u0[k + 1] = make_float2(-a.y, -b.y);
                            u0[k + 2] = make_float2(-a.z, -b.z);
                            u0[k + 3] = make_float2(-a.w, -b.w);
                            u1[k] = make_float2(-c.x, -d.x);
                            u1[k + 1] = make_float2(-c.y, -d.y);
                            u1[k + 2] = make_float2(-c.z, -d.z);
                            u1[k + 3] = make_float2(-c.w, -d.w);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int sa = rslot[32 * j + k], sb = rslot[32 * j + 16 + k];
                            u0[k] = make_float2(-res[sa], -res[sb]);
                            u1[k] = make_float2(-res[S + sa], -res[S + sb]);
                        }
                    }
                    uint32_t w0[4], w1[4];
                    const uint32_t e0 = mxfp4_unit(u0, 1.0f, w0);
                    const uint32_t e1 = mxfp4_unit(u1, 1.0f, w1);
                    *reinterpret_cast<uint4*>(cp0 + p.K / 2 + 16 * j) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                    sb0[scol(col)] = (uint8_t)(e0);
                    if (two) {
                        *reinterpret_cast<uint4*>(cp1 + p.K / 2 + 16 * j) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                        sb1[scol(col)] = (uint8_t)(e1);
                    }
                }
            }
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
            for (int w = 0; w < nthreads / 32; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

}  // namespace fp4q
