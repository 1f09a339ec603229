/*
 * fp4q.h -- C ABI of the B200 (sm_100a) micro-block FP4 activation quantizer.
 *
 * The library turns bf16 activations [M tokens x K channels] into 4-bit E2M1
 * codes plus block scales, in the two hardware micro-scaling formats and a
 * dual-scale variant, optionally after a block Hadamard rotation or the
 * ARCQuant reorder + RMSNorm + residual path (which also writes 4-bit integer
 * codes, FP4Q_INT4), and back again.
 *
 * Common conventions
 * ------------------
 *  - Every pointer argument is a DEVICE pointer to memory the caller allocated
 *    and owns (unless stated otherwise).  The library allocates nothing, holds
 *    no pointer after a call returns, and enqueues its kernels on `stream` only
 *    (NULL = the legacy default stream).  Calls are asynchronous.
 *  - bf16 matrices are row-major with a row stride `ld*` given in ELEMENTS.
 *  - Packed codes are row-major uint8 [M, K/2]: two E2M1 codes per byte, the
 *    code of the even column in the LOW nibble.  E2M1 code c: bit 3 = sign,
 *    magnitude (c & 7) -> {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  FP4Q_INT4 packs
 *    4-bit two's complement integers the same way.
 *  - Scale matrices are uint8 [M, K/B] row-major (FP4Q_SCALES_LINEAR) or the
 *    128x4-tiled layout of block-scaled tensor-core GEMMs
 *    (FP4Q_SCALES_SWIZZLED, see fp4q_scales_bytes): rows padded to a multiple
 *    of 128, scale columns to a multiple of 4, padding written as zero.
 *  - Validation happens on the host before anything is launched.  On any
 *    error the call returns a status != FP4Q_OK and launches nothing.
 *    Requirements shared by the quantizers: M >= 0, K >= 64, ldx >= K,
 *    ldx % 8 == 0, x 16-byte aligned; M == 0 is a no-op returning FP4Q_OK.
 *  - Kernel launch failures return FP4Q_ERR_CUDA.  Faults that happen later on
 *    the device surface through the CUDA error state of the stream.  A device-
 *    side bounded wait that runs out records a code read by fp4q_device_error().
 *  - The library is reentrant: it keeps no state between calls apart from the
 *    device error word described at fp4q_device_error().
 *
 * Numeric rules (identical in every entry point):
 *  - E2M1 rounding: nearest grid value, ties to the even code, saturation at
 *    +-6, sign kept (a negative value rounding to zero gives code 0x8).
 *  - NVFP4 (16-element blocks; ARCQuant summary, "Enonce du Probleme": NVFP4
 *    needs block size 16; E4M3 scales with an FP32 per-tensor scale, the usual
 *    NVFP4 recipe named in the nGPT abstract "Normalized Architectures are
 *    Natively 4-Bit"):  s_t = amax/2688;  per block r = (amax_b/6)/s_t,
 *    e = E4M3 round-to-nearest-even saturating at 448, d = E4M3(e)*s_t,
 *    code = E2M1(y/d) with y/d correctly rounded.  d == 0 gives zero codes.
 *  - MXFP4 (32-element blocks, power-of-two scale; MR-GPTQ abstract, point
 *    (2)): scale byte b = clamp(floor(log2 amax_b) - 2 + 127, 0, 254),
 *    code = E2M1(y * 2^(127-b)) (exact scaling); amax_b == 0 gives b = 0 and
 *    zero codes.
 *  - Dual scale (FP4Quant abstract, "micro-grouped dual-scale FP4"): an FP32
 *    group scale G = amax_128/2688 per 128 contiguous elements, then the NVFP4
 *    rule per 16-block with G in place of s_t.
 *  - INT4 (ARCQuant summary, "Generalisabilite": the ARCQuant scheme extends
 *    to INT4; the pages give no INT4 rule, so this is the NVFP4 container with
 *    the integer grid): codes are the integers -7..7 as 4-bit two's complement
 *    (low nibble = even column; -8 is never written); s_t = amax/3136
 *    (3136 = 7*448); per 16-block r = (amax_b/7)/s_t, e = E4M3(r),
 *    d = E4M3(e)*s_t, code = y/d rounded to the nearest integer (ties to even)
 *    and clamped to +-7.  Produced by fp4q_arc_quantize, read by
 *    fp4q_dequantize.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* fp4q_stream_t;

typedef enum fp4q_status {
    FP4Q_OK = 0,
    FP4Q_ERR_INVALID_ARG = 1, /* null pointer, bad size or enum value          */
    FP4Q_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. K too large)  */
    FP4Q_ERR_ALIGNMENT = 3,   /* pointer or row stride misaligned              */
    FP4Q_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed             */
    FP4Q_ERR_DEVICE = 5       /* a kernel's bounded wait ran out (see below)   */
} fp4q_status;

typedef enum fp4q_format {
    FP4Q_NVFP4 = 0,      /* B = 16, E4M3 block scale, FP32 tensor scale          */
    FP4Q_MXFP4 = 1,      /* B = 32, E8M0 shared exponent                          */
    FP4Q_NVFP4_DUAL = 2, /* B = 16, E4M3 micro-scale, FP32 scale per 128 elements */
    FP4Q_INT4 = 3        /* B = 16, integers -7..7, E4M3 block scale, FP32 tensor
                            scale (fp4q_arc_quantize and fp4q_dequantize only)   */
} fp4q_format;

typedef enum fp4q_scale_layout {
    FP4Q_SCALES_LINEAR = 0,   /* uint8 [M, K/B] row-major                            */
    FP4Q_SCALES_SWIZZLED = 1  /* 128x4 tiles: byte of (r, c) at
                                 ((r/128)*nC + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4,
                                 nC = ceil((K/B)/4)                                   */
} fp4q_scale_layout;

typedef enum fp4q_tscale_mode {
    FP4Q_TSCALE_DYNAMIC = 0, /* compute s_t = amax/2688 (INT4: amax/3136) of the
                                quantized tensor and WRITE it to *tensor_scale (two
                                passes over x)                                       */
    FP4Q_TSCALE_STATIC = 1   /* READ s_t from *tensor_scale (a calibrated scale;
                                one pass).  s_t <= 0 gives zero scales and codes.    */
} fp4q_tscale_mode;

/* Bytes of scratch the DYNAMIC tensor-scale mode needs (per-CTA partial maxima).
 * A constant; any M, K.  The workspace may be reused as soon as the call's
 * kernels have finished on the stream. */
#define FP4Q_WORKSPACE_BYTES ((size_t)16384)
size_t fp4q_workspace_bytes(int64_t M, int64_t K);

/* Size in bytes of the scale buffer a quantizer writes for an [M, ncols]
 * matrix of ncols = K/B blocks (ARC: (K+S)/16) in the given layout.  The
 * SWIZZLED size is ceil(M/128)*128 * ceil(ncols/4)*4.  Returns -1 on bad args. */
int64_t fp4q_scales_bytes(int64_t M, int64_t ncols, fp4q_scale_layout layout);

/* fp4q_quantize_nvfp4 -- NVFP4 quantization of a bf16 matrix.
 *   x            bf16 [M, ldx], K columns used.          (read)
 *   codes        uint8 [M, K/2].                         (written)
 *   scales       E4M3 bytes, [M, K/16] or swizzled.      (written)
 *   tensor_scale 1 float: written (DYNAMIC) or read (STATIC).
 *   workspace    >= fp4q_workspace_bytes() device bytes, DYNAMIC mode only
 *                (may be NULL in STATIC mode).
 * Requires K % 16 == 0.
 * Defined by: ARCQuant summary, "Methodologie" item 2 (primary stage: standard
 * block NVFP4 quantization) and "Enonce du Probleme" (block size 16). */
fp4q_status fp4q_quantize_nvfp4(const void* x, int64_t M, int64_t K, int64_t ldx,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                void* workspace, size_t workspace_bytes,
                                fp4q_stream_t stream);

/* fp4q_quantize_nvfp4_noalloc -- fp4q_quantize_nvfp4 in DYNAMIC tensor-scale
 * mode for callers that cannot allocate device memory: for example a host
 * framework that hands the library only its input and output tensors and gives
 * plugins no device allocator, or a service that fixes its device memory at
 * start-up and may not grow it afterwards.  Such a caller has no way to provide
 * the `workspace` of the dynamic mode, so this variant keeps that scratch (the
 * per-CTA partial maxima of the amax pre-pass) in a 16 KiB array of static
 * device memory inside the library, which every GPU that loads the library
 * holds until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.  (Not a method of the pages: they have no counterpart.)
 *   Arguments and results are those of fp4q_quantize_nvfp4 with
 *   mode = FP4Q_TSCALE_DYNAMIC: *tensor_scale is written.
 *   Limit: at most 4096 partial maxima, one per CTA of the amax pre-pass,
 *   whose grid is min(row tiles x column tiles, CTAs per SM x SMs, 4096); so
 *   every M and K accepted by fp4q_quantize_nvfp4 fits, and a grid above the
 *   limit would return FP4Q_ERR_UNSUPPORTED before anything is launched.
 *   Set-up: a call looks up the array's device address (cudaGetSymbolAddress)
 *   on the current device whenever `stream` is not capturing, and caches it;
 *   a call on a capturing stream uses the address cached by the last
 *   uncaptured call on that device.  So make the first call on a device
 *   before any stream capture, and, after cudaDeviceReset (which re-creates
 *   the context and so the array), make one uncaptured call before capturing
 *   again; a first call under capture returns FP4Q_ERR_CUDA.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents.  Nothing in it needs clearing (each call's pre-pass writes
 *   every entry its quantizer reads), but calls that overlap on the GPU (for
 *   example on two streams at once) race on it and must be serialised. */
fp4q_status fp4q_quantize_nvfp4_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx,
                                        uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                        fp4q_scale_layout layout, fp4q_stream_t stream);

/* fp4q_quantize_mxfp4 -- MXFP4 quantization of a bf16 matrix.
 *   x       bf16 [M, ldx].                     (read)
 *   codes   uint8 [M, K/2].                    (written)
 *   scales  E8M0 bytes, [M, K/32] or swizzled. (written)
 * Requires K % 32 == 0.
 * Defined by: MR-GPTQ abstract (MXFP4 and its power-of-two scale). */
fp4q_status fp4q_quantize_mxfp4(const void* x, int64_t M, int64_t K, int64_t ldx,
                                uint8_t* codes, uint8_t* scales, fp4q_scale_layout layout,
                                fp4q_stream_t stream);

/* fp4q_hadamard_quantize -- block Hadamard rotation, then quantization.
 *   y[r, b*n + i] = (1/sqrt(n)) * sum_j H_n[i][j] x[r, b*n + j]  for every
 *   contiguous n-block along K, H_n the Sylvester matrix
 *   H_n[i][j] = (-1)^popcount(i & j); then `format` quantization of y.
 *   had_size   n in {0 (no rotation), 16, 32, 64, 128, 256, 512}.
 *   format     FP4Q_NVFP4: scale_fp32 = 1 float tensor scale (DYNAMIC: written,
 *              STATIC: read).  FP4Q_MXFP4: scale_fp32 unused (may be NULL).
 *              FP4Q_NVFP4_DUAL: scale_fp32 = float [M, K/128] group scales,
 *              written; `mode` ignored.
 *   codes/scales as above; workspace as for fp4q_quantize_nvfp4.
 * Requires K % n == 0 and K % B == 0 (K % 128 == 0 for the dual format).
 * Defined by: MR-GPTQ abstract (block-wise Hadamard transforms, computed on the
 * fly for activations) and FP4Quant abstract (two-level FWHT, micro-grouped
 * dual-scale quantization). */
fp4q_status fp4q_hadamard_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                                   int had_size, fp4q_format format,
                                   uint8_t* codes, uint8_t* scales, float* scale_fp32,
                                   fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                   void* workspace, size_t workspace_bytes,
                                   fp4q_stream_t stream);

/* fp4q_hadamard_quantize_signed -- fp4q_hadamard_quantize with a random-sign
 * rotation: y = (1/sqrt(n)) H_n D x per contiguous n-block, D = diag(+-1), the
 * randomized Hadamard transform that NVFP4 training recipes apply before
 * quantizing (named as such in the nGPT abstract, "Normalized Architectures
 * are Natively 4-Bit").
 *   signs  HOST pointer to ceil(p/32) uint32 words, p = min(had_size, 128):
 *          bit j (word j/32, bit j%32) set negates input channel j of every
 *          p consecutive channels (D repeats with period p; for n = 256, 512 the
 *          rotation is H_(n/128) (x) (H_128 D_128)).  Read during the call.
 * Other arguments as for fp4q_hadamard_quantize; had_size in {16..512}.
 * Requires K % 128 == 0 (the tensor-core rotation), else FP4Q_ERR_UNSUPPORTED. */
fp4q_status fp4q_hadamard_quantize_signed(const void* x, int64_t M, int64_t K, int64_t ldx,
                                          int had_size, const uint32_t* signs, fp4q_format format,
                                          uint8_t* codes, uint8_t* scales, float* scale_fp32,
                                          fp4q_tscale_mode mode, fp4q_scale_layout layout,
                                          void* workspace, size_t workspace_bytes,
                                          fp4q_stream_t stream);

/* fp4q_arc_quantize -- ARCQuant fused reorder + RMSNorm + primary quantization
 * + residual quantization of the outlier channels, in NVFP4, MXFP4 or INT4.
 *   For each row: y[p] = x[perm[p]] / sqrt(mean_k x[k]^2 + eps) * gamma[perm[p]]
 *   (p = 0..K-1), primary = Q(y); for j < S, the residual
 *   res[j] = y[outliers[j]] - dq(outliers[j]), quantized in the same format.
 *     FP4Q_NVFP4: blocks of 16, E4M3 scales, one tensor scale s_t for both
 *       halves; dq = (E2M1 value * E4M3 value) * s_t.
 *     FP4Q_MXFP4: blocks of 32, E8M0 scales; dq = E2M1 value * 2^(b - 127).
 *       tensor_scale, mode and workspace are unused (may be NULL / 0).
 *     FP4Q_INT4: blocks of 16, E4M3 scales, one tensor scale s_t (amax/3136
 *       in DYNAMIC mode); dq = (integer * E4M3 value) * s_t.
 *   Output row = [primary K columns | residual S columns]:
 *   codes uint8 [M, (K+S)/2], scales [M, (K+S)/B] (or swizzled).
 *   gamma     bf16 [K], indexed by ORIGINAL channel.
 *   perm      int32 [K], perm[p] = original channel placed at position p
 *             (a permutation of 0..K-1; entries outside [0, K) are replaced
 *             by 0 and reported through fp4q_device_error(), code 2).
 *   outliers  int32 [S], positions in the REORDERED order (0 <= o < K, same
 *             out-of-range handling as perm); the
 *             calibrated choice is 0..S-1 (channels sorted by descending
 *             calibration absmax).  May be NULL when S == 0.
 *   tensor_scale / mode / workspace as for fp4q_quantize_nvfp4 (NVFP4 and
 *   INT4); DYNAMIC uses the amax of y.
 * Requires K % B == 0, S % B == 0, 0 <= S <= K, K <= 16384, eps >= 0, and that
 * one warp's buffers fit in shared memory (12 K + 8 S bytes plus the CTA's
 * 4 K + S/8 + 1.3 KiB, within 227 KiB), else FP4Q_ERR_UNSUPPORTED.
 * Defined by: ARCQuant summary, "Methodologie" items 1 (reorder by absolute
 * maximum, subset S), 2 (two-stage quantization), 3 (residual channels
 * concatenated along K) and 5 (one fused kernel: reorder, RMSNorm, primary and
 * residual quantization, GEMM-ready channel layout); "Generalisabilite" (the
 * scheme extends to MXFP4 and INT4). */
fp4q_status fp4q_arc_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                              const void* gamma, float eps, const int32_t* perm,
                              const int32_t* outliers, int64_t S, fp4q_format format,
                              uint8_t* codes, uint8_t* scales, float* tensor_scale,
                              fp4q_tscale_mode mode, fp4q_scale_layout layout,
                              void* workspace, size_t workspace_bytes,
                              fp4q_stream_t stream);

/* fp4q_dequantize -- codes + scales back to bf16, optionally followed by the
 * inverse block Hadamard (the normalised Sylvester matrix is its own inverse).
 *   value = (E2M1 value * E4M3 value) * s (s = *scale_fp32 for NVFP4, the
 *   group scale for the dual format), E2M1 value * 2^(b-127) for MXFP4, or
 *   (integer * E4M3 value) * *scale_fp32 for INT4, computed in FP32, then (if
 *   inv_had_size) rotated, then rounded to bf16 (nearest even).
 *   codes      uint8 [M, K/2]; scales [M, K/B] or swizzled, per `layout`.
 *   scale_fp32 NVFP4, INT4: 1 float; dual: float [M, K/128]; MXFP4: unused.
 *   y          bf16 [M, K] (row stride K).  (written)
 *   inv_had_size 0 or n in {16, 32, 64, 128, 256, 512}, K % n == 0 (INT4: 0
 *              only, else FP4Q_ERR_UNSUPPORTED).
 * Requires K % B == 0 (K % 128 for dual), K >= 64, 16-byte aligned codes and y.
 * Defined by: FP4Quant abstract (the receiving side of FP4-compressed
 * activations: unpack, rescale, inverse FWHT). */
fp4q_status fp4q_dequantize(fp4q_format format, const uint8_t* codes, const uint8_t* scales,
                            const float* scale_fp32, int64_t M, int64_t K,
                            fp4q_scale_layout layout, int inv_had_size, void* y,
                            fp4q_stream_t stream);

/* fp4q_gemm_nvfp4 -- the consumer of NVFP4 activations: a block-scaled GEMM on
 * the tensor cores,
 *   D[m, n] = a_scale * b_scale *
 *             sum_k (E2M1(A[m,k]) * E4M3(SA[m,k/16])) * (E2M1(B[n,k]) * E4M3(SB[n,k/16]))
 * with the products accumulated in FP32.
 *   a_codes   uint8 [M, K/2], a_scales the SWIZZLED scale buffer of A (as
 *             fp4q_quantize_nvfp4 / fp4q_arc_quantize write it), a_scale 1 float.
 *   b_codes   uint8 [N, K/2], b_scales SWIZZLED, b_scale 1 float (the weights,
 *             quantized the same way).
 *   d         [M, N] row-major, FP32 (d_bf16 = 0) or bf16 rounded to nearest
 *             even (d_bf16 = 1).   (written)
 * Requires K % 256 == 0 and N % 256 == 0 (else FP4Q_ERR_UNSUPPORTED); any M;
 * 16-byte aligned codes, scales and d.  The ARCQuant operand is consumed with
 * K + S in place of K against weights [W | W_S].
 * Defined by: ARCQuant summary, "Methodologie" items 3-4 (one GEMM over the
 * augmented reduction dimension K + S, the residual channels concatenated
 * along K) and MR-GPTQ abstract (kernels consuming NVFP4 activations on B200). */
fp4q_status fp4q_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_scale,
                            const uint8_t* b_codes, const uint8_t* b_scales, const float* b_scale,
                            int64_t M, int64_t N, int64_t K, void* d, int d_bf16,
                            fp4q_stream_t stream);

/* fp4q_dequantize_signed -- fp4q_dequantize followed by the inverse of a
 * random-sign rotation: x = D (1/sqrt(n)) H_n y (the normalised H is its own
 * inverse and D = D^-1).  signs: HOST pointer, the pattern given to
 * fp4q_hadamard_quantize_signed (period min(inv_had_size, 128)).  inv_had_size
 * must be non-zero; other arguments as for fp4q_dequantize. */
fp4q_status fp4q_dequantize_signed(fp4q_format format, const uint8_t* codes, const uint8_t* scales,
                                   const float* scale_fp32, int64_t M, int64_t K,
                                   fp4q_scale_layout layout, int inv_had_size, const uint32_t* signs,
                                   void* y, fp4q_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp4q_status_string(fp4q_status status);

/* Reads and clears the device error word of the CURRENT device: 0 if no kernel
 * recorded an error since the last read, else a bit mask (1 = a bounded wait
 * on a tile's arrival barrier ran out; 2 = an index argument of
 * fp4q_arc_quantize was outside [0, K) and was clamped).  Synchronizes the
 * device.  Returns -1 if the read itself failed. */
int fp4q_device_error(void);

/* Self-check of the division used by the quantizers (no page counterpart: it
 * exists so that tests can compare the kernels' correctly rounded quotient
 * against CUDA's IEEE division).  For i < n: q_fast[i] = x[i]/d[i] by the
 * kernels' method, q_ieee[i] = the IEEE quotient.  All device pointers. */
fp4q_status fp4q_selftest_div(const float* x, const float* d, int64_t n, float* q_fast,
                              float* q_ieee, fp4q_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
