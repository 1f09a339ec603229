// fp4q_quant.cuh -- persistent TMA-fed quantizer kernels for sm_100a:
// optional block Hadamard rotation (sizes 16..512), then NVFP4 / MXFP4 / dual
// scale quantization, or the amax pre-pass of the dynamic tensor scale.
//
// Work decomposition
//   A tile is 16 rows x 512 columns of the bf16 input (16 KiB), brought into
//   shared memory by eight 2-D TMA box loads of 16 rows x 64 columns each
//   (128-byte swizzle).  A CTA owns a strided subset of the tiles and keeps
//   kStages tiles in flight through a ring of mbarrier-tracked stages.
//   The 256 threads each own one "unit" of 32 consecutive columns of one row:
//     lane l, warp w  ->  row r = (l & 7) + 8*(w & 1),  unit j = (l >> 3) + 4*(w >> 1)
//   so the eight lanes of each shared-memory phase read eight different rows
//   at the same swizzled column: no bank conflicts for any access width.
//
// Block Hadamard of size n = n2 * 32 (Sylvester order, H_n = H_n2 (x) H_32):
//   the n2 threads owning one n-block first read the block "column-major"
//   (for every k2 < n2 their 32/n2 columns k1), apply H_n2 across k2 in
//   registers, exchange through a swizzled fp32 scratch so that each thread
//   holds its 32 contiguous values, then apply H_32 in registers.  n = 16 and
//   32 need no exchange.  The result is scaled by RN(1/sqrt(n)).
#pragma once

#include "fp4q_device.cuh"

namespace fp4q {

#ifndef FP4Q_STAGES
#define FP4Q_STAGES 4
#endif
#ifndef FP4Q_QUANT_CTAS_PER_SM
#define FP4Q_QUANT_CTAS_PER_SM 2
#endif

constexpr int kThreads = 256;
constexpr int kTileRows = 16;
constexpr int kTileCols = 512;
constexpr int kBoxCols = 64;
constexpr int kBoxes = kTileCols / kBoxCols;            // 8
constexpr int kBoxBytes = kTileRows * kBoxCols * 2;     // 2048
constexpr int kTileBytes = kTileRows * kTileCols * 2;   // 16384
constexpr int kStages = FP4Q_STAGES;                    // tiles in the shared-memory ring
constexpr int kQuantCtasPerSm = FP4Q_QUANT_CTAS_PER_SM;
constexpr int kScratchBytes = kTileRows * kTileCols * 4;  // fp32 exchange, 32 KiB

enum : int { FMT_NVFP4 = 0, FMT_MXFP4 = 1, FMT_DUAL = 2 };

struct QuantParams {
    int64_t M, K;
    int64_t n_row_tiles, n_col_tiles, n_tiles;
    uint8_t* codes;       // [M, K/2]
    uint8_t* scales;      // [M, K/B] or swizzled
    float* scale_fp32;    // NVFP4: tensor scale; DUAL: [M, K/128]
    float* partials;      // amax pass: per-CTA maxima out; dynamic quant: in
    int n_partials;       // number of valid partials (dynamic quant)
    int swizzled;         // scale layout
    int dynamic;          // NVFP4: 1 = tensor scale from partials, 0 = read *scale_fp32
    float had_norm;       // RN(1/sqrt(n))
};

template <int HAD>
struct HadShape {
    static constexpr int n2 = HAD >= 64 ? HAD / 32 : 1;  // threads per Hadamard block
    static constexpr int k1w = 32 / n2;                  // columns per k2 row a thread reads
};

// Physical shared-memory byte offset of (row r, tile column c) in a stage.
__device__ __forceinline__ uint32_t tile_off(uint32_t r, uint32_t c) {
    return (c >> 6) * kBoxBytes + swz128(r, (c & 63u) * 2u);
}

// In-register butterflies over v[0..N) with stride s (unnormalised Walsh-Hadamard).
template <int N>
__device__ __forceinline__ void fwht_reg(float* v) {
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
}

// Loads this thread's 32 post-rotation values of unit (r, j) of a staged tile.
template <int HAD>
__device__ __forceinline__ void load_unit(const uint8_t* stage, float* scratch, uint32_t r,
                                          uint32_t j, float had_norm, float* v) {
    if constexpr (HAD <= 32) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint4 q = *reinterpret_cast<const uint4*>(stage + tile_off(r, 32 * j + 8 * c));
            v[8 * c + 0] = bf16lo(q.x);
            v[8 * c + 1] = bf16hi(q.x);
            v[8 * c + 2] = bf16lo(q.y);
            v[8 * c + 3] = bf16hi(q.y);
            v[8 * c + 4] = bf16lo(q.z);
            v[8 * c + 5] = bf16hi(q.z);
            v[8 * c + 6] = bf16lo(q.w);
            v[8 * c + 7] = bf16hi(q.w);
        }
        if constexpr (HAD == 16) {
            fwht_reg<16>(v);
            fwht_reg<16>(v + 16);
        } else if constexpr (HAD == 32) {
            fwht_reg<32>(v);
        }
        if constexpr (HAD > 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= had_norm;
        }
    } else {
        constexpr int n2 = HadShape<HAD>::n2;
        constexpr int k1w = HadShape<HAD>::k1w;
        const uint32_t tau = j % n2;           // position inside the Hadamard block
        const uint32_t blk = j / n2;           // Hadamard block inside the tile row
        const uint32_t col0 = blk * HAD;       // first tile column of the block
        // Phase A: a[k2][i] = x[col0 + 32*k2 + k1w*tau + i]
        float a[n2][k1w];
#pragma unroll
        for (int k2 = 0; k2 < n2; ++k2) {
            const uint32_t c = col0 + 32 * k2 + k1w * tau;
            const uint8_t* p = stage + tile_off(r, c);
            if constexpr (k1w == 2) {
                uint32_t u = *reinterpret_cast<const uint32_t*>(p);
                a[k2][0] = bf16lo(u);
                a[k2][1] = bf16hi(u);
            } else if constexpr (k1w == 4) {
                uint2 u = *reinterpret_cast<const uint2*>(p);
                a[k2][0] = bf16lo(u.x);
                a[k2][1] = bf16hi(u.x);
                a[k2][2] = bf16lo(u.y);
                a[k2][3] = bf16hi(u.y);
            } else {
#pragma unroll
                for (int h = 0; h < k1w / 8; ++h) {
                    uint4 u = *reinterpret_cast<const uint4*>(stage + tile_off(r, c + 8 * h));
                    a[k2][8 * h + 0] = bf16lo(u.x);
                    a[k2][8 * h + 1] = bf16hi(u.x);
                    a[k2][8 * h + 2] = bf16lo(u.y);
                    a[k2][8 * h + 3] = bf16hi(u.y);
                    a[k2][8 * h + 4] = bf16lo(u.z);
                    a[k2][8 * h + 5] = bf16hi(u.z);
                    a[k2][8 * h + 6] = bf16lo(u.w);
                    a[k2][8 * h + 7] = bf16hi(u.w);
                }
            }
        }
        // H_n2 across k2, independently for each of the k1w columns
#pragma unroll
        for (int s = 1; s < n2; s <<= 1) {
#pragma unroll
            for (int k2 = 0; k2 < n2; ++k2) {
                if ((k2 & s) == 0) {
#pragma unroll
                    for (int i = 0; i < k1w; ++i) {
                        float x0 = a[k2][i], x1 = a[k2 + s][i];
                        a[k2][i] = x0 + x1;
                        a[k2 + s][i] = x0 - x1;
                    }
                }
            }
        }
        // Exchange: write row k2 of this block's scratch, read back row tau.
        // Scratch of block (r, blk): n2 rows of 32 floats (128 B), 16-byte chunk
        // index XORed with r & 7.
        uint8_t* sb = reinterpret_cast<uint8_t*>(scratch) +
                      (r * (kTileCols / HAD) + blk) * (uint32_t)(n2 * 128);
        const bool cross_warp = n2 > 4;  // blocks of 256/512 span several warps
        if (cross_warp) bar_sync(2, kThreads);
        else __syncwarp();
#pragma unroll
        for (int k2 = 0; k2 < n2; ++k2) {
            uint8_t* rowp = sb + k2 * 128;
            const uint32_t k1 = k1w * tau;
            if constexpr (k1w == 2) {
                uint32_t off = ((((k1 >> 2) ^ r) & 7u) << 4) + (k1 & 3u) * 4u;
                *reinterpret_cast<float2*>(rowp + off) = make_float2(a[k2][0], a[k2][1]);
            } else {
#pragma unroll
                for (int h = 0; h < k1w / 4; ++h) {
                    uint32_t chunk = (k1 >> 2) + h;
                    *reinterpret_cast<float4*>(rowp + (((chunk ^ r) & 7u) << 4)) =
                        make_float4(a[k2][4 * h], a[k2][4 * h + 1], a[k2][4 * h + 2], a[k2][4 * h + 3]);
                }
            }
        }
        if (cross_warp) bar_sync(2, kThreads);
        else __syncwarp();
        {
            const uint8_t* rowp = sb + tau * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float4 q = *reinterpret_cast<const float4*>(rowp + (((ch ^ r) & 7u) << 4));
                v[4 * ch + 0] = q.x;
                v[4 * ch + 1] = q.y;
                v[4 * ch + 2] = q.z;
                v[4 * ch + 3] = q.w;
            }
        }
        fwht_reg<32>(v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= had_norm;
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
__global__ void __launch_bounds__(kThreads, kQuantCtasPerSm)
    quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned stage ring, then the exchange scratch, then barriers.
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stages = smem;
    float* scratch = reinterpret_cast<float*>(smem + kStages * kTileBytes);
    constexpr int scratch_bytes = (HAD >= 64) ? kScratchBytes : 0;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kTileBytes + scratch_bytes);
    float* red = reinterpret_cast<float*>(bars + kStages);

    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31, warp = tid >> 5;
    const uint32_t r = (lane & 7) + 8 * (warp & 1);
    const uint32_t j = (lane >> 3) + 4 * (warp >> 1);

    const int64_t n_my = p.n_tiles > (int64_t)blockIdx.x
                             ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1
                             : 0;

    if (tid == 0) {
        prefetch_tmap(&tmap_x);
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
        fence_barrier_init();
    }
    __syncthreads();

    // Per-CTA scale of the NVFP4 format.
    float s_t = 0.0f;
    if constexpr (FMT == FMT_NVFP4 && !AMAX_ONLY) {
        if (p.dynamic) {
            s_t = tensor_scale_from_partials(p.partials, p.n_partials, red);
            if (blockIdx.x == 0 && tid == 0) *p.scale_fp32 = s_t;
        } else {
            s_t = *p.scale_fp32;
        }
    }

    auto issue = [&](int64_t i) {  // tile i of this CTA into stage i % kStages
        const int64_t t = blockIdx.x + i * (int64_t)gridDim.x;
        const int64_t rt = t / p.n_col_tiles, ct = t % p.n_col_tiles;
        const int32_t y = (int32_t)(rt * kTileRows);
        const int32_t x0 = (int32_t)(ct * kTileCols);
        const int nb = (int)min64(kBoxes, (p.K - x0 + kBoxCols - 1) / kBoxCols);
        const uint32_t st = (uint32_t)(i % kStages);
        const uint32_t bar = smem_u32(&bars[st]);
        mbar_arrive_expect_tx(bar, (uint32_t)(nb * kBoxBytes));
        const uint32_t dst = smem_u32(stages + st * kTileBytes);
        for (int b = 0; b < nb; ++b) tma_load_2d(dst + b * kBoxBytes, &tmap_x, x0 + b * kBoxCols, y, bar);
    };

    if (tid == 0)
        for (int64_t i = 0; i < min64(kStages, n_my); ++i) issue(i);

    float my_amax = 0.0f;
    for (int64_t i = 0; i < n_my; ++i) {
        const uint32_t st = (uint32_t)(i % kStages);
        const bool ok = mbar_wait(smem_u32(&bars[st]), (uint32_t)((i / kStages) & 1));
        if (!bar_and(1, kThreads, ok)) {
            // A tile never arrived: record it, let the copies still in flight land, leave.
            if (tid == 0) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                for (int64_t k = i; k < min64(n_my, i + kStages); ++k)
                    (void)mbar_wait(smem_u32(&bars[k % kStages]), (uint32_t)((k / kStages) & 1));
            }
            return;
        }
        // The previous stage is free once every thread passed the vote above.
        if (tid == 0 && i >= 1 && i - 1 + kStages < n_my) issue(i - 1 + kStages);

        const int64_t t = blockIdx.x + i * (int64_t)gridDim.x;
        const int64_t rt = t / p.n_col_tiles, ct = t % p.n_col_tiles;
        const int64_t row = rt * kTileRows + r;
        const int64_t col = ct * kTileCols + 32 * (int64_t)j;
        const uint8_t* stage = stages + st * kTileBytes;

        // Units entirely past K skip work, but Hadamard blocks of 256/512 still
        // meet at the exchange barrier: every thread of the CTA calls load_unit.
        float v[32];
        load_unit<HAD>(stage, scratch, r, j, p.had_norm, v);
        const bool live = row < p.M && col < p.K;
        const int nval = (int)min64(32, p.K - col);  // 16 or 32 when live

        if constexpr (AMAX_ONLY) {
            if (live) {
                float m = amax16(v);
                if (nval > 16) m = fmaxf(m, amax16(v + 16));
                my_amax = fmaxf(my_amax, m);
            }
        } else if constexpr (FMT == FMT_NVFP4) {
            if (live) {
                uint32_t w[4];
                const uint32_t e0 = nvfp4_block16(v, amax16(v), s_t, w[0], w[1]);
                uint32_t e1 = 0;
                if (nval > 16) e1 = nvfp4_block16(v + 16, amax16(v + 16), s_t, w[2], w[3]);
                uint8_t* cp = p.codes + row * (p.K / 2) + col / 2;
                if ((p.K & 31) == 0) {  // rows of codes are 16-byte aligned
                    *reinterpret_cast<uint4*>(cp) = make_uint4(w[0], w[1], w[2], w[3]);
                } else {  // K = 16 (mod 32): rows are only 8-byte aligned
                    *reinterpret_cast<uint2*>(cp) = make_uint2(w[0], w[1]);
                    if (nval > 16) *reinterpret_cast<uint2*>(cp + 8) = make_uint2(w[2], w[3]);
                }
                const int64_t nsc = p.K / 16, c0 = col / 16;
                if (p.swizzled) {
                    const int64_t nC = (nsc + 3) / 4;
                    p.scales[swizzle_offset(row, c0, nC)] = (uint8_t)e0;
                    if (nval > 16) p.scales[swizzle_offset(row, c0 + 1, nC)] = (uint8_t)e1;
                } else {
                    p.scales[row * nsc + c0] = (uint8_t)e0;
                    if (nval > 16) p.scales[row * nsc + c0 + 1] = (uint8_t)e1;
                }
            }
        } else if constexpr (FMT == FMT_MXFP4) {
            if (live) {
                uint32_t w[4];
                const uint32_t b = mxfp4_block32(v, w);
                *reinterpret_cast<uint4*>(p.codes + row * (p.K / 2) + col / 2) =
                    make_uint4(w[0], w[1], w[2], w[3]);
                const int64_t nsc = p.K / 32, c0 = col / 32;
                if (p.swizzled) p.scales[swizzle_offset(row, c0, (nsc + 3) / 4)] = (uint8_t)b;
                else p.scales[row * nsc + c0] = (uint8_t)b;
            }
        } else {  // FMT_DUAL: group of 128 = 4 units = lanes l, l^8, l^16, l^24
            float a0 = amax16(v), a1 = amax16(v + 16);
            float g = fmaxf(a0, a1);
            g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 8));
            g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, 16));
            if (live) {
                const float G = __fdiv_rn(g, 2688.0f);
                uint32_t w[4];
                const uint32_t e0 = nvfp4_block16(v, a0, G, w[0], w[1]);
                const uint32_t e1 = nvfp4_block16(v + 16, a1, G, w[2], w[3]);
                *reinterpret_cast<uint4*>(p.codes + row * (p.K / 2) + col / 2) =
                    make_uint4(w[0], w[1], w[2], w[3]);
                const int64_t nsc = p.K / 16, c0 = col / 16;
                if (p.swizzled) {
                    const int64_t nC = (nsc + 3) / 4;
                    *reinterpret_cast<uint16_t*>(p.scales + swizzle_offset(row, c0, nC)) =
                        (uint16_t)(e0 | (e1 << 8));
                } else {
                    *reinterpret_cast<uint16_t*>(p.scales + row * nsc + c0) = (uint16_t)(e0 | (e1 << 8));
                }
                if ((j & 3) == 0) p.scale_fp32[row * (p.K / 128) + col / 128] = G;
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
            for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
            p.partials[blockIdx.x] = m;
        }
    }
}

template <int HAD>
constexpr int quant_smem_bytes() {
    return 1024 + kStages * kTileBytes + (HAD >= 64 ? kScratchBytes : 0) + kStages * 8 + 64;
}

}  // namespace fp4q
