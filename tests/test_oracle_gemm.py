"""Pins of the oracle's consumer GEMM (the block-scaled NVFP4 product of two
quantized tensors; ARCQuant summary, Methodologie items 3-4: one GEMM over the
augmented reduction dimension K + S).

The oracle dequantizes with its own decoders and multiplies in float64; here
the product is recomputed exactly with rational arithmetic from ml_dtypes'
decoders, and the augmented GEMM is checked against the primary GEMM plus the
residual correction."""
from fractions import Fraction

import ml_dtypes
import numpy as np

import oracle
import workloads

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _exact_values(codes, scales):
    u = oracle.unpack_codes(codes)
    e = u.view(F4).astype(np.float64)
    s = np.repeat(np.asarray(scales, np.uint8).view(F8).astype(np.float64), 16, axis=1)
    return [[Fraction(float(a)) * Fraction(float(b)) for a, b in zip(er, sr)] for er, sr in zip(e, s)]


def test_gemm_equals_exact_rational_product():
    a = workloads.nvfp4_outliers(3, 64, seed=50)
    b = workloads.nvfp4_outliers(4, 64, seed=51, gain=5.0)
    ca, sa, ta = oracle.quantize_nvfp4(a)
    cb, sb, tb = oracle.quantize_nvfp4(b)
    D, Dabs = oracle.nvfp4_gemm(ca, sa, ta, cb, sb, tb)
    A, B = _exact_values(ca, sa), _exact_values(cb, sb)
    s = Fraction(float(ta)) * Fraction(float(tb))
    for i in range(3):
        for j in range(4):
            exact = s * sum(x * y for x, y in zip(A[i], B[j]))
            mag = s * sum(abs(x * y) for x, y in zip(A[i], B[j]))
            assert abs(Fraction(float(D[i, j])) - exact) <= Fraction(2) ** -50 * mag
            assert abs(Fraction(float(Dabs[i, j])) - mag) <= Fraction(2) ** -50 * mag


def test_augmented_gemm_is_primary_plus_residual_correction():
    """[Q(y) | Q(r)] [W | W_S]^T = Q(y) W^T + Q(r) W_S^T: the GEMM over K + S
    adds the residual's correction on the outlier channels only."""
    M, K, S, N = 6, 128, 32, 5
    x, gamma, perm, outl = workloads.arc_activations(M, K, seed=52, S=S, calib_rows=64)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl)
    w = workloads.nvfp4_outliers(N, K, seed=53)
    w_aug = np.concatenate([w, w[:, outl]], axis=1)
    cw, sw, tw = oracle.quantize_nvfp4(w_aug)
    D, _ = oracle.nvfp4_gemm(codes, scales, s_t, cw, sw, tw)
    Dp, _ = oracle.nvfp4_gemm(codes[:, : K // 2], scales[:, : K // 16], s_t, cw[:, : K // 2],
                              sw[:, : K // 16], tw)
    Dr, _ = oracle.nvfp4_gemm(codes[:, K // 2:], scales[:, K // 16:], s_t, cw[:, K // 2:],
                              sw[:, K // 16:], tw)
    np.testing.assert_allclose(D, Dp + Dr, rtol=1e-12, atol=1e-12)
