/*
 * fp4q_oracle.c -- plain, slow, scalar CPU oracle for micro-block FP4
 * activation quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
 * the benchmark's CPU-baseline leg load this code.  It shares no source, header,
 * table or helper with the CUDA library; the library never calls it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (IEEE binary32 +,-,*,/ with round-to-nearest-even, no FMA contraction).
 *
 * What it computes, and where the pages fix it:
 *   - NVFP4: 16-element blocks (ARCQuant summary, "Enonce du Probleme", second
 *     bullet: NVFP4 needs block size 16), E2M1 elements (ARCQuant,
 *     "Methodologie" item 1 names the E2M1 mantissa), an E4M3 block scale and an
 *     FP32 per-tensor scale (the nGPT abstract, "Normalized Architectures are
 *     Natively 4-Bit", lists per-tensor scaling as the usual NVFP4 recipe).
 *   - MXFP4: 32-element blocks with a power-of-two shared scale (MR-GPTQ
 *     abstract, point (2): MXFP4's power-of-two scale).
 *   - Dual scale: a coarse FP32 group scale plus fine E4M3 micro-scales
 *     (FP4Quant abstract: "micro-grouped dual-scale FP4 quantization").
 *   - Block Hadamard rotation per contiguous block (MR-GPTQ abstract: block-wise
 *     Hadamard transforms computed on the fly for activations; FP4Quant
 *     abstract: two-level FWHT).  The oracle applies the dense Sylvester matrix.
 *   - ARCQuant fused path: reorder -> RMSNorm -> primary NVFP4 quantization ->
 *     residual NVFP4 quantization of the outlier channels, appended along K
 *     (ARCQuant, "Methodologie" items 1, 2, 3 and 5); the same in MXFP4 and
 *     INT4 ("Generalisabilite": the scheme extends to both formats).
 *
 * Numeric rules (where the pages only name the formats, these are the plain
 * readings of them, each taken where the pages leave the step open):
 *   E2M1   : magnitudes {0,.5,1,1.5,2,3,4,6}; nearest value, ties to the even
 *            code (mantissa bit 0), |v| > 6 saturates to 6, sign always kept
 *            (a negative value that rounds to zero is code 0x8).
 *   E4M3   : OCP E4M3FN, bias 7, max 448, subnormals down to 2^-9, no Inf;
 *            nearest value, ties to even mantissa, saturating at 448.
 *   E8M0   : byte b encodes 2^(b-127); b = clamp(floor(log2 amax) - 2 + 127, 0, 254).
 *   NVFP4  : s_t = amax_tensor / 2688 (2688 = 6*448); per block
 *            r = (amax_b / 6) / s_t, e = E4M3(r), d = E4M3val(e) * s_t,
 *            code_i = E2M1(y_i / d); every operation one binary32 rounding.
 *            d == 0 (or s_t == 0) gives scale byte as encoded and all codes 0.
 *   MXFP4  : code_i = E2M1(y_i * 2^-(b-127)), exact scaling; amax_b == 0 gives
 *            b = 0 and all codes 0.
 *   Dual   : G = amax_128 / 2688 per 128-element group, then the NVFP4 rule per
 *            16-block with G in place of s_t.
 *   INT4   : (ARCQuant summary, "Generalisabilite": the residual scheme extends
 *            to INT4; the pages give no INT4 scale rule, so this is the NVFP4
 *            container with the integer grid in place of E2M1) elements are the
 *            integers -7..7 in 4-bit two's complement; s_t = amax_tensor / 3136
 *            (3136 = 7*448); per 16-block r = (amax_b / 7) / s_t, e = E4M3(r),
 *            d = E4M3val(e) * s_t, code_i = clamp(RNE(fl32(y_i / d)), -7, 7)
 *            (nearest integer, ties to even); d == 0 gives all codes 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* bf16 <-> binary32                                                          */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the top half of a binary32: widening is exact. */
ORC_EXPORT float orc_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* binary32 -> bf16, round to nearest, ties to even (finite inputs). */
ORC_EXPORT uint16_t orc_f32_to_bf16(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7f800000u) == 0x7f800000u) /* Inf / NaN: keep (NaN quieted) */
        return (uint16_t)((u >> 16) | ((u & 0x007fffffu) ? 0x40u : 0u));
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

ORC_EXPORT void orc_bf16_array_to_f32(const uint16_t* x, int64_t n, float* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_bf16_to_f32(x[i]);
}

ORC_EXPORT void orc_f32_array_to_bf16(const float* x, int64_t n, uint16_t* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_f32_to_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit, no Inf/NaN       */
/* ------------------------------------------------------------------------ */

/* Magnitude of code c (0..7), from the bit fields: e = c>>1, m = c&1.
 * e == 0 is subnormal: m * 2^(1-1) * 0.5; otherwise (1 + m/2) * 2^(e-1). */
static double e2m1_mag(int c) {
    int e = c >> 1, m = c & 1;
    if (e == 0) return 0.5 * m;
    return (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
}

ORC_EXPORT float orc_e2m1_decode(uint8_t code) {
    double v = e2m1_mag(code & 7);
    return (float)((code & 8) ? -v : v);
}

/* Nearest E2M1 value to v; ties go to the even code; values beyond 6 saturate
 * (6 is the nearest element of the set); the sign of v is always kept. */
ORC_EXPORT uint8_t orc_e2m1_encode(float v) {
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    int best = 0;
    if (a >= 6.0) {
        best = 7; /* 6 is the nearest member of the set for every larger value */
    } else {
        /* Below 6 the distances are exact in binary64 wherever two candidates
         * are close to a tie (a then has no bits below 2^-26). */
        double bestd = INFINITY;
        for (int c = 0; c < 8; ++c) {
            double d = fabs(a - e2m1_mag(c));
            if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
                best = c;
                bestd = d;
            }
        }
    }
    return (uint8_t)(best | (neg << 3));
}

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP E4M3FN): 1 sign, 4 exponent (bias 7), 3 mantissa, no Inf,        */
/* S.1111.111 is NaN; max finite 448; subnormals m * 2^-9                     */
/* ------------------------------------------------------------------------ */

static double e4m3_mag(int b) { /* b in 0..126 */
    int e = (b >> 3) & 15, m = b & 7;
    if (e == 0) return ldexp((double)m, -9);
    return (1.0 + m / 8.0) * ldexp(1.0, e - 7);
}

ORC_EXPORT float orc_e4m3_decode(uint8_t b) {
    if ((b & 0x7f) == 0x7f) return NAN;
    double v = e4m3_mag(b & 0x7f);
    return (float)((b & 0x80) ? -v : v);
}

/* Nearest finite E4M3 value, ties to even mantissa (= even byte), saturating
 * at 448 (values at or above 448, Inf included, give 0x7E). */
ORC_EXPORT uint8_t orc_e4m3_encode(float r) {
    int neg = signbit(r) ? 1 : 0;
    double a = fabs((double)r);
    int best = 0;
    if (a >= 448.0) {
        best = 0x7e;
    } else {
        double bestd = INFINITY;
        for (int b = 0; b <= 0x7e; ++b) {
            double d = fabs(a - e4m3_mag(b)); /* exact near any tie (a >= 2^-10 there) */
            if (d < bestd || (d == bestd && (b & 1) == 0 && (best & 1) == 1)) {
                best = b;
                bestd = d;
            }
        }
    }
    return (uint8_t)(best | (neg << 7));
}

/* ------------------------------------------------------------------------ */
/* E8M0 shared exponent (MXFP4)                                               */
/* ------------------------------------------------------------------------ */

/* floor(log2(a)) for finite a > 0, from frexp (exact, subnormals included). */
ORC_EXPORT int orc_floor_log2(float a) {
    int ex;
    (void)frexp((double)a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
    return ex - 1;
}

/* Scale byte for a block whose absolute maximum is amax. */
ORC_EXPORT uint8_t orc_e8m0_encode(float amax) {
    if (!(amax > 0.0f)) return 0;
    int E = orc_floor_log2(amax) - 2;
    int b = E + 127;
    if (b < 0) b = 0;
    if (b > 254) b = 254;
    return (uint8_t)b;
}

ORC_EXPORT float orc_e8m0_decode(uint8_t b) {
    if (b == 255) return NAN;
    return (float)ldexp(1.0, (int)b - 127);
}

/* ------------------------------------------------------------------------ */
/* Block scale layouts                                                        */
/* ------------------------------------------------------------------------ */

/* Byte offset of scale element (r, c) in the 128x4-tiled layout consumed by
 * block-scaled tensor-core GEMMs: rows in tiles of 128, scale columns in tiles
 * of 4; each 512-byte tile stores row r%32 at 16*(r%32), row group (r%128)/32
 * at +4*((r%128)/32), column c%4 at +c%4.  nC = ceil(ncols/4). */
ORC_EXPORT int64_t orc_swizzle_offset(int64_t r, int64_t c, int64_t nC) {
    return ((r / 128) * nC + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* Rewrite a linear [M, ncols] scale matrix into the padded 128x4-tiled layout
 * (ceil(M/128)*128 rows x ceil(ncols/4)*4 columns; padding bytes are zero). */
ORC_EXPORT void orc_swizzle_scales(const uint8_t* lin, int64_t M, int64_t ncols, uint8_t* out) {
    int64_t nC = (ncols + 3) / 4;
    int64_t Mp = (M + 127) / 128 * 128;
    memset(out, 0, (size_t)(Mp * nC * 4));
    for (int64_t r = 0; r < M; ++r)
        for (int64_t c = 0; c < ncols; ++c)
            out[orc_swizzle_offset(r, c, nC)] = lin[r * ncols + c];
}

/* ------------------------------------------------------------------------ */
/* Amax and the per-tensor scale                                              */
/* ------------------------------------------------------------------------ */

ORC_EXPORT float orc_amax(const float* y, int64_t M, int64_t K, int64_t ld) {
    float m = 0.0f;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(y[r * ld + k]);
            if (a > m) m = a;
        }
    return m;
}

/* s_t = amax / (6 * 448), one binary32 division. */
ORC_EXPORT float orc_tensor_scale(float amax) { return amax / 2688.0f; }

/* ------------------------------------------------------------------------ */
/* NVFP4 block quantization (one 16-element block)                            */
/* ------------------------------------------------------------------------ */

/* Quantize the 16 values y[0..15] against the FP32 scale s (the per-tensor
 * scale for NVFP4, the group scale for the dual format).  Writes 8 bytes of
 * codes (low nibble = even index) and returns the E4M3 scale byte. */
static uint8_t nvfp4_block(const float* y, float s, uint8_t* codes8) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
    }
    uint8_t e = 0;
    float d = 0.0f;
    if (s > 0.0f) {
        float bs = amax / 6.0f;
        float r = bs / s;
        e = orc_e4m3_encode(r);
        d = orc_e4m3_decode(e) * s;
    }
    for (int i = 0; i < 8; ++i) {
        uint8_t lo = 0, hi = 0;
        if (d != 0.0f) {
            lo = orc_e2m1_encode(y[2 * i] / d);
            hi = orc_e2m1_encode(y[2 * i + 1] / d);
        }
        codes8[i] = (uint8_t)(lo | (hi << 4));
    }
    return e;
}

/* NVFP4 quantization of an fp32 matrix y[M, K] (row stride ld) with per-tensor
 * scale s_t.  codes: [M, K/2] bytes; scales: [M, K/16] E4M3 bytes (linear). */
ORC_EXPORT void orc_nvfp4_quantize(const float* y, int64_t M, int64_t K, int64_t ld, float s_t,
                                   uint8_t* codes, uint8_t* scales) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t b = 0; b < K / 16; ++b)
            scales[r * (K / 16) + b] =
                nvfp4_block(y + r * ld + 16 * b, s_t, codes + r * (K / 2) + 8 * b);
}

/* ------------------------------------------------------------------------ */
/* MXFP4 block quantization                                                   */
/* ------------------------------------------------------------------------ */

ORC_EXPORT void orc_mxfp4_quantize(const float* y, int64_t M, int64_t K, int64_t ld,
                                   uint8_t* codes, uint8_t* scales) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            const float* v = y + r * ld + 32 * b;
            uint8_t* c = codes + r * (K / 2) + 16 * b;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            uint8_t sb = orc_e8m0_encode(amax);
            scales[r * (K / 32) + b] = sb;
            for (int i = 0; i < 16; ++i) {
                uint8_t lo = 0, hi = 0;
                if (amax > 0.0f) {
                    lo = orc_e2m1_encode(ldexpf(v[2 * i], 127 - (int)sb));
                    hi = orc_e2m1_encode(ldexpf(v[2 * i + 1], 127 - (int)sb));
                }
                c[i] = (uint8_t)(lo | (hi << 4));
            }
        }
}

/* ------------------------------------------------------------------------ */
/* Dual scale: FP32 per-128 group scale + E4M3 per-16 micro-scale             */
/* ------------------------------------------------------------------------ */

ORC_EXPORT void orc_dual_quantize(const float* y, int64_t M, int64_t K, int64_t ld,
                                  uint8_t* codes, uint8_t* scales, float* gscales) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t g = 0; g < K / 128; ++g) {
            const float* v = y + r * ld + 128 * g;
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            float G = amax / 2688.0f;
            gscales[r * (K / 128) + g] = G;
            for (int b = 0; b < 8; ++b)
                scales[r * (K / 16) + 8 * g + b] =
                    nvfp4_block(v + 16 * b, G, codes + r * (K / 2) + 64 * g + 8 * b);
        }
}

/* ------------------------------------------------------------------------ */
/* Dequantization                                                             */
/* ------------------------------------------------------------------------ */

/* NVFP4 / dual: value = (E2M1val * E4M3val) * s, s = s_t or the group scale;
 * the first product is exact, the second is one binary32 rounding. */
ORC_EXPORT void orc_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, float s_t,
                                     int64_t M, int64_t K, float* out) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            float p = orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]);
            out[r * K + k] = p * s_t;
        }
}

ORC_EXPORT void orc_dual_dequantize(const uint8_t* codes, const uint8_t* scales,
                                    const float* gscales, int64_t M, int64_t K, float* out) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            float p = orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]);
            out[r * K + k] = p * gscales[r * (K / 128) + k / 128];
        }
}

ORC_EXPORT void orc_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t M,
                                     int64_t K, float* out) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = orc_e2m1_decode(c) * orc_e8m0_decode(scales[r * (K / 32) + k / 32]);
        }
}

/* ------------------------------------------------------------------------ */
/* Block Hadamard rotation (dense Sylvester matrix, binary64)                 */
/* ------------------------------------------------------------------------ */

/* Sylvester-ordered Hadamard entry H_n[i][j] = (-1)^popcount(i & j). */
ORC_EXPORT int orc_hadamard_entry(int i, int j) {
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* y[r, blk*n + i] = (1/sqrt(n)) * sum_j H_n[i][j] * x[r, blk*n + j], for every
 * contiguous n-block along K; accumulated in binary64, rounded once to binary32. */
ORC_EXPORT void orc_hadamard(const float* x, int64_t M, int64_t K, int64_t ld, int n, float* y) {
    double inv = 1.0 / sqrt((double)n);
    for (int64_t r = 0; r < M; ++r)
        for (int64_t b = 0; b < K / n; ++b) {
            const float* xb = x + r * ld + b * n;
            float* yb = y + r * K + b * n;
            for (int i = 0; i < n; ++i) {
                double s = 0.0;
                for (int j = 0; j < n; ++j) s += orc_hadamard_entry(i, j) * (double)xb[j];
                yb[i] = (float)(s * inv);
            }
        }
}

/* ------------------------------------------------------------------------ */
/* RMSNorm and the ARCQuant fused path                                        */
/* ------------------------------------------------------------------------ */

/* Reorder + RMSNorm in binary64, rounded once to binary32:
 *   y[r, p] = x[r, perm[p]] / sqrt(mean_k x[r,k]^2 + eps) * gamma[perm[p]]
 * The mean runs over all K channels of the row (independent of the order). */
ORC_EXPORT void orc_rmsnorm_permute(const float* x, int64_t M, int64_t K, int64_t ld,
                                    const float* gamma, const int32_t* perm, double eps,
                                    float* y) {
    for (int64_t r = 0; r < M; ++r) {
        const float* xr = x + r * ld;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)xr[k] * (double)xr[k];
        double rs = 1.0 / sqrt(ss / (double)K + eps);
        for (int64_t p = 0; p < K; ++p) {
            int32_t c = perm ? perm[p] : (int32_t)p;
            y[r * K + p] = (float)((double)xr[c] * rs * (double)gamma[c]);
        }
    }
}

/* ARCQuant two-stage quantization of an already reordered + normalised fp32
 * matrix y[M, K]:
 *   primary  : NVFP4 of all K columns with tensor scale s_t
 *   residual : for j < S, p = outliers[j]: res_j = y[p] - dq(p), with
 *              dq(p) = (E2M1val * E4M3val) * s_t as in the dequantizer, then
 *              NVFP4 of res in 16-blocks with the same s_t
 *   layout   : row = [primary K columns | residual S columns], i.e. codes
 *              [M, (K+S)/2] and scales [M, (K+S)/16]. */
ORC_EXPORT void orc_arc_quantize(const float* y, int64_t M, int64_t K, int64_t S,
                                 const int32_t* outliers, float s_t, uint8_t* codes,
                                 uint8_t* scales) {
    int64_t KS = K + S;
    float* res = (float*)malloc(sizeof(float) * (size_t)(S > 0 ? S : 1));
    for (int64_t r = 0; r < M; ++r) {
        const float* yr = y + r * K;
        uint8_t* cr = codes + r * (KS / 2);
        uint8_t* sr = scales + r * (KS / 16);
        for (int64_t b = 0; b < K / 16; ++b) sr[b] = nvfp4_block(yr + 16 * b, s_t, cr + 8 * b);
        for (int64_t j = 0; j < S; ++j) {
            int64_t p = outliers[j];
            uint8_t byte = cr[p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15);
            float dq = (orc_e2m1_decode(c) * orc_e4m3_decode(sr[p / 16])) * s_t;
            res[j] = yr[p] - dq;
        }
        for (int64_t b = 0; b < S / 16; ++b)
            sr[K / 16 + b] = nvfp4_block(res + 16 * b, s_t, cr + K / 2 + 8 * b);
    }
    free(res);
}

/* ------------------------------------------------------------------------ */
/* INT4 in the micro-block container (ARCQuant summary, "Generalisabilite")   */
/* ------------------------------------------------------------------------ */

/* Nearest integer to q, ties to the even integer, written out with floor so
 * that it does not depend on the floating-point rounding mode; then clamped to
 * the symmetric range -7..7 and stored as a 4-bit two's complement nibble. */
ORC_EXPORT uint8_t orc_int4_encode(float q) {
    double a = (double)q; /* exact */
    double f = floor(a);
    double frac = a - f;  /* exact: a and f are within 1 of each other */
    double n = f;
    if (a != a) return 0; /* NaN (not produced by finite inputs): code 0 */
    if (frac > 0.5 || (frac == 0.5 && fmod(f, 2.0) != 0.0)) n = f + 1.0;
    if (n > 7.0) n = 7.0;
    if (n < -7.0) n = -7.0;
    return (uint8_t)(((int)n) & 15);
}

/* Two's complement value of a nibble (-8..7; the encoder never writes -8). */
ORC_EXPORT float orc_int4_decode(uint8_t c) {
    int v = c & 15;
    return (float)(v >= 8 ? v - 16 : v);
}

/* s_t = amax / (7 * 448), one binary32 division. */
ORC_EXPORT float orc_int4_tensor_scale(float amax) { return amax / 3136.0f; }

/* One 16-element block against the FP32 scale s: 8 bytes of codes (low nibble
 * = even index) and the E4M3 scale byte, as nvfp4_block with the largest grid
 * value 7 and the integer grid. */
static uint8_t int4_block(const float* y, float s, uint8_t* codes8) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
    }
    uint8_t e = 0;
    float d = 0.0f;
    if (s > 0.0f) {
        float bs = amax / 7.0f;
        float r = bs / s;
        e = orc_e4m3_encode(r);
        d = orc_e4m3_decode(e) * s;
    }
    for (int i = 0; i < 8; ++i) {
        uint8_t lo = 0, hi = 0;
        if (d != 0.0f) {
            lo = orc_int4_encode(y[2 * i] / d);
            hi = orc_int4_encode(y[2 * i + 1] / d);
        }
        codes8[i] = (uint8_t)(lo | (hi << 4));
    }
    return e;
}

/* INT4 quantization of y[M, K] (row stride ld) with tensor scale s_t:
 * codes [M, K/2], scales [M, K/16] E4M3 bytes (linear). */
ORC_EXPORT void orc_int4_quantize(const float* y, int64_t M, int64_t K, int64_t ld, float s_t,
                                  uint8_t* codes, uint8_t* scales) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t b = 0; b < K / 16; ++b)
            scales[r * (K / 16) + b] = int4_block(y + r * ld + 16 * b, s_t, codes + r * (K / 2) + 8 * b);
}

/* value = (integer * E4M3val) * s_t: the first product is exact, the second
 * one binary32 rounding. */
ORC_EXPORT void orc_int4_dequantize(const uint8_t* codes, const uint8_t* scales, float s_t,
                                    int64_t M, int64_t K, float* out) {
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            float p = orc_int4_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]);
            out[r * K + k] = p * s_t;
        }
}

/* ARCQuant two-stage path in INT4: primary INT4 of all K columns with s_t;
 * residual of outlier position p: y[p] - (integer * E4M3val) * s_t, quantized
 * in 16-blocks with the same s_t and appended along K (codes [M, (K+S)/2],
 * scales [M, (K+S)/16]). */
ORC_EXPORT void orc_arc_quantize_int4(const float* y, int64_t M, int64_t K, int64_t S,
                                      const int32_t* outliers, float s_t, uint8_t* codes,
                                      uint8_t* scales) {
    int64_t KS = K + S;
    float* res = (float*)malloc(sizeof(float) * (size_t)(S > 0 ? S : 1));
    for (int64_t r = 0; r < M; ++r) {
        const float* yr = y + r * K;
        uint8_t* cr = codes + r * (KS / 2);
        uint8_t* sr = scales + r * (KS / 16);
        for (int64_t b = 0; b < K / 16; ++b) sr[b] = int4_block(yr + 16 * b, s_t, cr + 8 * b);
        for (int64_t j = 0; j < S; ++j) {
            int64_t p = outliers[j];
            uint8_t byte = cr[p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15);
            float dq = (orc_int4_decode(c) * orc_e4m3_decode(sr[p / 16])) * s_t;
            res[j] = yr[p] - dq;
        }
        for (int64_t b = 0; b < S / 16; ++b)
            sr[K / 16 + b] = int4_block(res + 16 * b, s_t, cr + K / 2 + 8 * b);
    }
    free(res);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar encoders (for the Python binding)                */
/* ------------------------------------------------------------------------ */

/* ARCQuant two-stage path in MXFP4 (ARCQuant summary, "Generalisabilite": the
 * residual scheme carries over to MXFP4; MR-GPTQ abstract: MXFP4's 32-element
 * blocks with a power-of-two scale).  Primary: MXFP4 of every row of y.
 * Residual of outlier position p: r = y[p] - E2M1val(code) * 2^(b - 127), b the
 * primary scale byte of p's block (the product is exact; the difference is one
 * binary32 rounding).  The S residuals are quantized in 32-blocks with their
 * own E8M0 scales and appended along K: codes [M, (K+S)/2], scales
 * [M, (K+S)/32]. */
ORC_EXPORT void orc_arc_quantize_mxfp4(const float* y, int64_t M, int64_t K, int64_t S,
                                       const int32_t* outliers, uint8_t* codes,
                                       uint8_t* scales) {
    int64_t KS = K + S;
    float* res = (float*)malloc(sizeof(float) * (size_t)(S > 0 ? S : 1));
    for (int64_t r = 0; r < M; ++r) {
        const float* yr = y + r * K;
        uint8_t* cr = codes + r * (KS / 2);
        uint8_t* sr = scales + r * (KS / 32);
        orc_mxfp4_quantize(yr, 1, K, K, cr, sr);
        for (int64_t j = 0; j < S; ++j) {
            int64_t p = outliers[j];
            uint8_t byte = cr[p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15);
            float dq = orc_e2m1_decode(c) * orc_e8m0_decode(sr[p / 32]);
            res[j] = yr[p] - dq;
        }
        if (S > 0) orc_mxfp4_quantize(res, 1, S, S, cr + K / 2, sr + K / 32);
    }
    free(res);
}

ORC_EXPORT void orc_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

ORC_EXPORT void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

ORC_EXPORT void orc_e4m3_decode_array(const uint8_t* b, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(b[i]);
}

ORC_EXPORT void orc_e8m0_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e8m0_encode(v[i]);
}

ORC_EXPORT void orc_int4_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_int4_encode(v[i]);
}

ORC_EXPORT void orc_int4_decode_array(const uint8_t* c, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_int4_decode(c[i]);
}
