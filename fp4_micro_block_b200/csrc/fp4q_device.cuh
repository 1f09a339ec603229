// fp4q_device.cuh -- device building blocks of the sm_100a quantizer kernels:
// the micro-scaling formats (E2M1 / E4M3 / E8M0) through the Blackwell
// conversion instructions, the correctly rounded division used for every
// element, bounded mbarrier waits and TMA tile loads.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fp4q {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------------------------
// Device error word (the library's only device state).  Bit 0: a bounded wait on
// a tile's arrival barrier ran out.  Bit 1: an index argument (channel order,
// outlier position) was outside [0, K) and was clamped.  Read and cleared by
// fp4q_device_error().
// ------------------------------------------------------------------------------
__device__ unsigned int g_device_error;

constexpr unsigned int kErrWaitTimeout = 1u;
constexpr unsigned int kErrBadIndex = 2u;  // a channel / outlier index outside [0, K)
// Upper bound of try_wait polls before a wait gives up (each poll may suspend
// the thread for a short, hardware-chosen time).  Far above any real latency.
// The test build (FP4Q_TEST_HOOKS) cuts it short so that a test can make a
// wait run out quickly.
#ifdef FP4Q_TEST_HOOKS
constexpr uint32_t kWaitPolls = 1u << 14;
#else
constexpr uint32_t kWaitPolls = 1u << 22;
#endif

// ------------------------------------------------------------------------------
// Format conversions
// ------------------------------------------------------------------------------

// bf16 pair (low half = lower address) -> two binary32 (exact).
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Four bytes of packed E2M1 codes from eight values (v[0] -> low nibble of byte 0).
// cvt.rn.satfinite.e2m1x2.f32 d, a, b puts E2M1(a) in the high nibble and E2M1(b)
// in the low nibble: round to nearest even, saturate to +-6, keep the sign.
__device__ __forceinline__ uint32_t e2m1_pack8(const float* v) {
    uint32_t w;
    asm("{ .reg .b8 t0, t1, t2, t3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
        "mov.b32 %0, {t0, t1, t2, t3}; }"
        : "=r"(w)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return w;
}

// E4M3 (OCP E4M3FN) of a non-negative binary32: nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode(float r) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(r));
    return h & 0xffu;
}

// E4M3 byte -> binary32 (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
    uint32_t h2;
    uint16_t in = (uint16_t)(b & 0xffu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// Two E2M1 codes (one byte, low nibble first) -> two binary32 (exact).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
    uint32_t h2;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte));
    float2 r;
    r.x = __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
    r.y = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    return r;
}

// INT4 (4-bit two's complement, the symmetric range -7..7): four bytes of
// codes from eight quotients q (q[0] -> low nibble of byte 0).  Each q is
// clamped to [-7, 7] and rounded to the nearest integer, ties to even, by one
// IEEE addition of 1.5 * 2^23 (whose ulp is 1); the integer is then the low
// bits of the sum's significand (2^22 + k for k in -7..7), its low nibble the
// two's complement code.
__device__ __forceinline__ uint32_t int4_pack8(const float* q) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float c = fminf(fmaxf(q[i], -7.0f), 7.0f);
        const uint32_t k = __float_as_uint(__fadd_rn(c, 12582912.0f));
        asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(w) : "r"(k), "r"(w), "r"(4 * i));
    }
    return w;
}

// Two INT4 codes (one byte, low nibble first) -> two binary32 (exact): a
// nibble n holds k = (n ^ 8) - 8; n ^ 8 goes into the low significand bits of
// 1.5 * 2^23 (whose ulp is 1), and 1.5 * 2^23 + 8 is subtracted.
__device__ __forceinline__ float2 int4x2_decode(uint32_t byte) {
    const float lo = __uint_as_float((byte & 0xfu) ^ 0x4b400008u) - 12582920.0f;
    const float hi = __uint_as_float(((byte >> 4) & 0xfu) ^ 0x4b400008u) - 12582920.0f;
    return make_float2(lo, hi);
}

// Binary32 -> bf16 bits, round to nearest even (finite values).
__device__ __forceinline__ uint32_t bf16x2_pack(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------------------------------------
// Correctly rounded division x / d with a precomputed reciprocal.
//
// Markstein's correction theorem (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34, 1990):
// if y is within half an ulp of 1/d and q is within one ulp of x/d, then
// q' = RN(q + (x - q*d) * y), with the remainder x - q*d exact by FMA, is the
// correctly rounded quotient.  q0 = RN(x*y) can be up to 1.5 ulp away, so one
// correction first makes it faithful and a second one makes it correctly
// rounded.  The remainder is formed as (q*d - x) and subtracted so that the
// sign of a zero quotient follows x (x = -0 gives -0).
// Preconditions (checked by the callers per block): y = RN(1/d) is normal,
// 2^-100 <= d <= 2^100 and |x|/d <= 2^100.  Quotients below 2^-100 in magnitude
// may be off by an ulp; they encode to a zero E2M1 code of the right sign
// either way.
// ------------------------------------------------------------------------------
__device__ __forceinline__ float div_rn(float x, float d, float y) {
    float q = x * y;
    float e = fmaf(q, d, -x);
    q = fmaf(-e, y, q);
    e = fmaf(q, d, -x);
    q = fmaf(-e, y, q);
    return q;
}

__device__ __forceinline__ bool div_fast_ok(float d, float amax) {
    return d >= 0x1p-100f && d <= 0x1p100f && amax <= d * 0x1p100f;
}

// ------------------------------------------------------------------------------
// Block quantizers (registers in, packed codes out)
// ------------------------------------------------------------------------------

__device__ __forceinline__ float amax16(const float* v) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    return m;
}

// NVFP4 block of 16 against the FP32 scale s (tensor or group scale):
// r = (amax/6)/s, e = E4M3(r), d = E4M3val(e)*s, code_i = E2M1(v_i/d).
// Returns the E4M3 byte; writes 8 bytes of codes as two words.
__device__ __forceinline__ uint32_t nvfp4_block16(const float* v, float amax, float s,
                                                  uint32_t& w0, uint32_t& w1) {
    uint32_t e = 0;
    float d = 0.0f;
    if (s > 0.0f) {
        float bs = __fdiv_rn(amax, 6.0f);
        float r = __fdiv_rn(bs, s);
        e = e4m3_encode(r);
        d = e4m3_decode(e) * s;
    }
    if (d == 0.0f) {
        w0 = 0u;
        w1 = 0u;
        return e;
    }
    float q[16];
    if (div_fast_ok(d, amax)) {
        float y = __frcp_rn(d);
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = div_rn(v[i], d, y);
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], d);
    }
    w0 = e2m1_pack8(q);
    w1 = e2m1_pack8(q + 8);
    return e;
}

// MXFP4 block of 32: byte = clamp(floor(log2 amax) - 2 + 127, 0, 254) read off the
// exponent field; codes = E2M1(v * 2^(127-byte)) (exact scaling).
__device__ __forceinline__ uint32_t mxfp4_block32(const float* v, uint32_t* w) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    uint32_t ef = __float_as_uint(amax) >> 23;  // amax >= 0, finite
    uint32_t b = ef >= 2u ? ef - 2u : 0u;      // subnormal / tiny amax clamps to 0
    if (amax == 0.0f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = 0u;
        return 0u;
    }
    float mult = __uint_as_float((254u - b) << 23);  // 2^(127-b), b <= 252: normal
    float q[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) q[i] = v[i] * mult;
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e2m1_pack8(q + 8 * i);
    return b;
}

// ------------------------------------------------------------------------------
// Scale layouts
// ------------------------------------------------------------------------------

__device__ __forceinline__ int64_t swizzle_offset(int64_t r, int64_t c, int64_t nC) {
    return ((r >> 7) * nC + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// ------------------------------------------------------------------------------
// mbarrier + TMA
// ------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// The first byte of the dynamic shared buffer `base` aligned to A bytes, by
// pointer arithmetic on the shared array: the compiler keeps the result (and
// every pointer derived from it) in the shared address space.  Rounding the
// address through an integer instead loses that, and every load and store
// through the pointer becomes a generic one (slower, and waited for on the
// long scoreboard).
template <uint32_t A>
__device__ __forceinline__ uint8_t* align_shared(uint8_t* base) {
    return base + ((A - (smem_u32(base) & (A - 1))) & (A - 1));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity; false if it never completed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitPolls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int32_t x, int32_t y,
                                             uint32_t src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// At most the most recent bulk group still reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void sts_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Barrier among the first `n` threads of the CTA with an AND vote.
__device__ __forceinline__ bool bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, %3, p; "
        "selp.u32 %0, 1, 0, q; }"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Programmatic dependent launch: every kernel is launched so that it may start
// while the previous kernel of the stream is finishing.  pdl_wait() blocks
// until that kernel has completed and its writes are visible, and comes before
// the first global read or write; pdl_trigger() lets the next kernel launch
// (it still waits for this one to complete before touching memory).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 128-byte TMA swizzle: the 16-byte chunk index inside a 128-byte row is XORed
// with the row index modulo 8 (box bases are 1024-byte aligned).
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t byte_in_row) {
    return row * 128u + ((((byte_in_row >> 4) ^ row) & 7u) << 4) + (byte_in_row & 15u);
}

}  // namespace fp4q
