// fp4q_unit.cuh -- quantization of one 32-value "unit" of a row.
//
// A unit holds 32 consecutive values v[0..31] of one row.  They are kept
// NEGATED, as 16 pairs n[i] = (-v[i], -v[16+i]): the first component belongs
// to block 0 (v[0..15]), the second to block 1 (v[16..31]), so the two
// 16-element NVFP4 blocks of a unit are always processed side by side, and
// Walsh-Hadamard stages of stride 1..8 are "vertical" pair operations.
// Carrying -v costs nothing (the bf16 unpack and the tensor-core rotation flip
// the sign for free) and gives the divisions below the -x operand they use.
//
// The per-element arithmetic is scalar fp32: on sm_100a the packed FFMA2 /
// FMUL2 forms save issue slots but run at half the FMA-pipe rate of scalar
// FFMA, and the quantizer is bound by that pipe.
#pragma once

#include "fp4q_device.cuh"

namespace fp4q {

// Component-wise pair arithmetic (scalar instructions, see above).
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return make_float2(a.x * b.x, a.y * b.y); }
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }

// Negated bf16 -> binary32 (exact): w = (lo, hi) bf16 pair.  w * 2^16 + 2^31
// (mod 2^32) is the low half moved up with its sign bit flipped.
__device__ __forceinline__ float nbf16lo(uint32_t w) { return __uint_as_float(w * 65536u + 0x80000000u); }
__device__ __forceinline__ float nbf16hi(uint32_t w) {
    return __uint_as_float((w & 0xffff0000u) ^ 0x80000000u);
}

// ------------------------------------------------------------------------------
// Division with a split reciprocal (4 FMA-pipe operations per quotient).
//
// For a divisor d > 0 keep rn = RN(1/d), rz = RZ(1/d) (largest float <= 1/d)
// and lo = RN((1 - d*rz) * rz) >= 0, so that rz + lo = 1/d within 2^-45
// relative (1 - d*rz is exact by FMA).  Then
//     q0 = RN(x*rz + RN(x*lo))
// is within (1/2 + 2^-21) ulp of x/d, hence faithful, and Markstein's
// correction theorem (P. Markstein, IBM J. Res. Dev. 34, 1990: with rn within
// half an ulp of 1/d and q0 faithful, the remainder x - q0*d is exact and
// RN(q0 + (x - q0*d)*rn) = RN(x/d)) gives the correctly rounded quotient in one
// step.  lo >= 0 makes x*rz and x*lo carry the sign of x, so a zero x keeps its
// sign through every step.  Preconditions as for div_rn: d in [2^-100, 2^100],
// |x|/d <= 2^100; quotients below 2^-100 may be off by an ulp and still encode
// to a zero E2M1 code of the right sign.
// ------------------------------------------------------------------------------
struct Rcp {
    float rn, rz, lo;
};

__device__ __forceinline__ Rcp make_rcp(float d) {  // d > 0, normal
    Rcp c;
    c.rn = __frcp_rn(d);
    c.rz = fmaf(-d, c.rn, 1.0f) < 0.0f ? __uint_as_float(__float_as_uint(c.rn) - 1u) : c.rn;
    c.lo = fmaf(-d, c.rz, 1.0f) * c.rz;
    return c;
}

// x/d from nx = -x.
__device__ __forceinline__ float div_split(float nx, float d, const Rcp& c) {
    const float t = nx * -c.lo;           // x*lo
    const float q0 = fmaf(nx, -c.rz, t);  // x*rz + x*lo: faithful
    const float e = fmaf(q0, d, nx);      // q0*d - x, exact
    return fmaf(-e, c.rn, q0);            // q0 - e*rn
}

// Split reciprocals of 6 and 2688 (RN, RZ, lo; checked against exact rationals).
__device__ __forceinline__ Rcp rcp6() {
    return Rcp{__uint_as_float(0x3e2aaaabu), __uint_as_float(0x3e2aaaaau), __uint_as_float(0x322aaaaau)};
}
__device__ __forceinline__ Rcp rcp2688() {
    return Rcp{__uint_as_float(0x39c30c31u), __uint_as_float(0x39c30c30u), __uint_as_float(0x2dc30c30u)};
}

// ---------------------------------------------------------------- Walsh-Hadamard
template <int S>
__device__ __forceinline__ void vstage(float2* n) {  // stride S < 16: pairs i, i+S
#pragma unroll
    for (int i = 0; i < 16; ++i)
        if ((i & S) == 0) {
            const float2 a = n[i], b = n[i + S];
            n[i] = add2(a, b);
            n[i + S] = sub2(a, b);
        }
}
__device__ __forceinline__ void hstage(float2* n) {  // stride 16: within each pair
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float a = n[i].x, b = n[i].y;
        n[i] = make_float2(a + b, a - b);
    }
}
// H_16 on both blocks (v[0..15], v[16..31]) / H_32 on the whole unit (unnormalised).
__device__ __forceinline__ void fwht16x2(float2* n) { vstage<1>(n); vstage<2>(n); vstage<4>(n); vstage<8>(n); }
__device__ __forceinline__ void fwht32(float2* n) { fwht16x2(n); hstage(n); }

__device__ __forceinline__ void scale_unit(float2* n, float c) {
    const float2 c2 = dup2(c);
#pragma unroll
    for (int i = 0; i < 16; ++i) n[i] = mul2(n[i], c2);
}

// ---------------------------------------------------------------- amax
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// Block maxima |v| of the two blocks of a unit.
__device__ __forceinline__ float2 amax_pair(const float2* n) {
    float a0 = fmaxf(fabsf(n[0].x), fabsf(n[1].x)), a1 = fmaxf(fabsf(n[0].y), fabsf(n[1].y));
#pragma unroll
    for (int i = 2; i < 16; i += 2) {
        a0 = max3(a0, fabsf(n[i].x), fabsf(n[i + 1].x));
        a1 = max3(a1, fabsf(n[i].y), fabsf(n[i + 1].y));
    }
    return make_float2(a0, a1);
}

// ---------------------------------------------------------------- packing
// Packed E2M1 codes of the quotients q (x/d, both blocks): w[0..1] block 0,
// w[2..3] block 1, low nibble = even index.
__device__ __forceinline__ void pack_codes(const float2* q, uint32_t (&w)[4]) {
    float b0[16], b1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        b0[i] = q[i].x;
        b1[i] = q[i].y;
    }
    w[0] = e2m1_pack8(b0);
    w[1] = e2m1_pack8(b0 + 8);
    w[2] = e2m1_pack8(b1);
    w[3] = e2m1_pack8(b1 + 8);
}

// Two E4M3 bytes (lo = block 0) of the non-negative pair r, and their values.
__device__ __forceinline__ uint32_t e4m3x2_encode(float2 r) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(r.y), "f"(r.x));
    return h;
}
__device__ __forceinline__ float2 e4m3x2_decode(uint32_t e2) {
    uint32_t h2;
    const uint16_t in = (uint16_t)e2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// Constants of the NVFP4 rule for one FP32 scale s (the tensor scale, or a
// group scale of the dual format).  The fast path needs s in [2^-90, 2^90] and,
// per block, 2^-90 <= amax <= 2^62 * s (or amax = 0): then every quotient below
// stays in the normal range, (amax/6)/s <= 2^60, and each decoded block scale
// d = E4M3(e) * s is either 0 or in [2^-99, 2^99], which are the preconditions
// of the split-reciprocal division.
struct ScaleCtx {
    float s;       // the FP32 scale
    Rcp rs;        // split reciprocal of s
    float am_max;  // 2^62 * s
    bool fast;
};

__device__ __forceinline__ ScaleCtx make_ctx(float s) {
    ScaleCtx c;
    c.s = s;
    c.fast = s >= 0x1p-90f && s <= 0x1p90f;
    c.rs = c.fast ? make_rcp(s) : Rcp{0.0f, 0.0f, 0.0f};
    c.am_max = s * 0x1p62f;
    return c;
}

// Per-CTA table of the NVFP4 decoded scales for a fixed s: t[e] = (d, rn, rz,
// lo) with d = E4M3(e) * s and the split reciprocal of d (zeros when d == 0 or
// d is outside [2^-100, 2^100]), for the 128 non-negative E4M3 bytes.
__device__ __forceinline__ void build_table(float4* t, float s) {
    for (int e = threadIdx.x; e < 128; e += blockDim.x) {
        const float d = (e < 127) ? e4m3_decode((uint32_t)e) * s : 0.0f;
        const bool ok = d >= 0x1p-100f && d <= 0x1p100f;
        const Rcp c = ok ? make_rcp(d) : Rcp{0.0f, 0.0f, 0.0f};
        t[e] = make_float4(d, c.rn, c.rz, c.lo);
    }
}

// The NVFP4 rule with IEEE divisions for one block of a unit (component Y of
// the pairs), for units outside the fast range.  Writes two code words and
// returns the scale byte.  INT4: the same rule with the largest grid value 7
// and integer codes.
template <bool Y, bool INT4 = false>
__device__ __forceinline__ uint32_t nvfp4_block_ieee(const float2* n, float a, float s, float fold,
                                                     uint32_t& w0, uint32_t& w1) {
    float d = 0.0f;
    uint32_t e = 0;
    if (s > 0.0f) {
        const float r = __fdiv_rn(__fdiv_rn(a, INT4 ? 7.0f : 6.0f), s);  // a already folded
        e = e4m3_encode(r);
        d = e4m3_decode(e) * s;
    }
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float x = -(Y ? n[i].y : n[i].x) * fold;
        q[i] = d != 0.0f ? __fdiv_rn(x, d) : 0.0f;
    }
    if constexpr (INT4) {
        w0 = d != 0.0f ? int4_pack8(q) : 0u;
        w1 = d != 0.0f ? int4_pack8(q + 8) : 0u;
    } else {
        w0 = d != 0.0f ? e2m1_pack8(q) : 0u;
        w1 = d != 0.0f ? e2m1_pack8(q + 8) : 0u;
    }
    return e;
}

__device__ __forceinline__ uint32_t nvfp4_unit_ieee(const float2* n, float2 am, float s, float fold,
                                                    uint32_t (&w)[4]) {
    const uint32_t e0 = nvfp4_block_ieee<false>(n, am.x, s, fold, w[0], w[1]);
    const uint32_t e1 = nvfp4_block_ieee<true>(n, am.y, s, fold, w[2], w[3]);
    return e0 | (e1 << 8);
}

// NVFP4 rule for the two blocks of a unit against the FP32 scale of `c`:
//   r = (amax_b / 6) / s,  e = E4M3(r),  d = E4M3(e) * s,  code = E2M1(v / d).
// The unit holds z with v = z * fold (fold > 0: a Hadamard normalisation
// applied here per block instead of per element); am is the amax of z.
// EXACT: v / d is the correctly rounded quotient (div_split), and fold must be
//        a power of two so that the folding is exact (the quantize-only paths,
//        whose codes are bit-exact).
// !EXACT: scale and quotient are products with rounded reciprocals (below),
//        within a few ulp of the exact ones (the rotated paths, whose inputs are
//        themselves fp32 approximations of the rotation and whose acceptance
//        is a tolerance).  `tab` must be the table of c.s (TABLE) or of s = 1.
// Returns the two scale bytes (block 0 low) and writes the codes to w.
template <bool TABLE, bool EXACT>
__device__ __forceinline__ uint32_t nvfp4_unit(const float2* n, float2 am, const ScaleCtx& c,
                                               const float4* tab, float fold, uint32_t (&w)[4]) {
    am.x *= fold;
    am.y *= fold;
    const uint32_t b0 = __float_as_uint(am.x), b1 = __float_as_uint(am.y);
    const uint32_t tiny = __float_as_uint(0x1p-90f);  // amax == 0 passes, 0 < amax < 2^-90 fails
    const bool in_range = c.fast && (b0 - 1u) >= tiny - 1u && (b1 - 1u) >= tiny - 1u &&
                          fmaxf(am.x, am.y) <= c.am_max;
    if (!in_range) return nvfp4_unit_ieee(n, am, c.s, fold, w);
    if constexpr (!EXACT) {
        // Scale bytes from RN(RN(amax * RN(1/6)) * RN(1/s)), within 3 ulp of
        // (amax/6)/s: a byte can differ only for r within 3 ulp of an E4M3
        // rounding boundary.  Quotients z * RN(rn * fold), rn = RN(1/d) from the
        // table (TABLE: d = E4M3(e) * s) or RN(1/E4M3(e)) * RN(1/s) from a
        // table built for s = 1 (the dual format's per-group s).
        const float k6 = __uint_as_float(0x3e2aaaabu);  // RN(1/6)
        const float r0 = (am.x * k6) * c.rs.rn, r1 = (am.y * k6) * c.rs.rn;
        const uint32_t e2 = e4m3x2_encode(make_float2(r0, r1));
        const float4 t0 = tab[e2 & 0xffu], t1 = tab[e2 >> 8];
        const float g = TABLE ? fold : c.rs.rn * fold;
        const float2 m = make_float2(-(t0.y * g), -(t1.y * g));  // n holds -z
        float q0[16], q1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float2 q = __fmul2_rn(n[i], m);
            q0[i] = q.x;
            q1[i] = q.y;
        }
        w[0] = e2m1_pack8(q0);
        w[1] = e2m1_pack8(q0 + 8);
        w[2] = e2m1_pack8(q1);
        w[3] = e2m1_pack8(q1 + 8);
        if (t0.x == 0.0f) w[0] = w[1] = 0u;  // zero block scale: all codes +0
        if (t1.x == 0.0f) w[2] = w[3] = 0u;
        return e2;
    }
    const Rcp r6 = rcp6();
    const float bs0 = div_split(-am.x, 6.0f, r6), bs1 = div_split(-am.y, 6.0f, r6);
    const float r0 = div_split(-bs0, c.s, c.rs), r1 = div_split(-bs1, c.s, c.rs);
    const uint32_t e2 = e4m3x2_encode(make_float2(r0, r1));
    float d0, d1;
    Rcp c0, c1;
    if constexpr (TABLE) {
        const float4 t0 = tab[e2 & 0xffu], t1 = tab[e2 >> 8];
        d0 = t0.x; c0 = Rcp{t0.y, t0.z, t0.w};
        d1 = t1.x; c1 = Rcp{t1.y, t1.z, t1.w};
    } else {
        const float2 dd = e4m3x2_decode(e2);
        d0 = dd.x * c.s;
        d1 = dd.y * c.s;
        c0 = d0 != 0.0f ? make_rcp(d0) : Rcp{0.0f, 0.0f, 0.0f};
        c1 = d1 != 0.0f ? make_rcp(d1) : Rcp{0.0f, 0.0f, 0.0f};
    }
    if (fold != 1.0f) {  // divide z by d / 2^-k
        const float inv = 1.0f / fold;  // exact: a power of two
        d0 *= inv;
        d1 *= inv;
        c0 = Rcp{c0.rn * fold, c0.rz * fold, c0.lo * fold};
        c1 = Rcp{c1.rn * fold, c1.rz * fold, c1.lo * fold};
    }
    float q0[16], q1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        q0[i] = div_split(n[i].x, d0, c0);
        q1[i] = div_split(n[i].y, d1, c1);
    }
    w[0] = e2m1_pack8(q0);
    w[1] = e2m1_pack8(q0 + 8);
    w[2] = e2m1_pack8(q1);
    w[3] = e2m1_pack8(q1 + 8);
    if (d0 == 0.0f) w[0] = w[1] = 0u;  // zero block scale: all codes +0
    if (d1 == 0.0f) w[2] = w[3] = 0u;
    return e2;
}

// MXFP4 of a whole unit (one 32-block) of v = z * fold (fold > 0, see
// nvfp4_unit; am of v = RN(amax(z) * fold) since rounding is monotone):
// byte = clamp(floor(log2 amax) - 2 + 127, 0, 254) from the exponent field,
// codes = E2M1(z * RN(fold * 2^(127-byte))), which is RN(v * 2^(127-byte))
// exactly when fold = 1 and within an ulp otherwise.
__device__ __forceinline__ uint32_t mxfp4_unit(const float2* n, float fold, uint32_t (&w)[4]) {
    const float2 a = amax_pair(n);
    const float am = fmaxf(a.x, a.y) * fold;
    if (am == 0.0f) {
        w[0] = w[1] = w[2] = w[3] = 0u;
        return 0u;
    }
    const uint32_t ef = __float_as_uint(am) >> 23;
    const uint32_t b = ef >= 2u ? ef - 2u : 0u;
    const float nm = -__uint_as_float((254u - b) << 23) * fold;  // -2^(127-b) * fold
    // codes in element order: v[i] = -n[i].x * 2^(127-b), v[16+i] = -n[i].y * ...
    float v[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // packed f32x2 multiply: the same RN products
        const float2 q = __fmul2_rn(n[i], make_float2(nm, nm));
        v[i] = q.x;
        v[16 + i] = q.y;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e2m1_pack8(v + 8 * i);
    return b;
}

}  // namespace fp4q
