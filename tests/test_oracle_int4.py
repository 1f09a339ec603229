"""Pins of the oracle's INT4 variant of the ARCQuant two-stage path.

ARCQuant summary, "Generalisabilite": the residual scheme extends to the INT4
format.  The pages give no INT4 scale rule; the reading the oracle takes is the
NVFP4 container (16-element blocks, E4M3 block scale, FP32 tensor scale) with
the symmetric integer grid -7..7 in place of E2M1, so s_t = amax / (7 * 448)
and each block's scale targets amax_b / 7.

Each test checks the oracle against something other than its own code path:
numpy's round-half-even ``rint``, numpy's int8 arithmetic shift for two's
complement, ml_dtypes' E4M3 decoder, exhaustive nearest-integer search with
exact rationals, closed forms on inputs built to lie on the grid, the
round-to-nearest error bound, and the linearity identity of the augmented GEMM.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle
import workloads

F8 = ml_dtypes.float8_e4m3fn
E4_VALS = [Fraction(float(v)) for v in np.arange(127, dtype=np.uint8).view(F8).astype(np.float64)]


def lib_e4m3(b):
    return np.asarray(b, np.uint8).view(F8).astype(np.float64)


def lib_int4(nibbles):
    """Two's complement of 4-bit values by numpy's int8 arithmetic shift."""
    return ((np.asarray(nibbles, np.uint8) << 4).astype(np.int8) >> 4).astype(np.int64)


def nearest_e4m3_byte(ratio: np.float32) -> int:
    """Nearest finite E4M3 byte (0..126) to ratio >= 0 by exact rationals, ties
    to the even byte (even mantissa)."""
    r = Fraction(float(ratio))
    ds = [abs(r - v) for v in E4_VALS]
    best = min(ds)
    want = [i for i, dv in enumerate(ds) if dv == best]
    return ([i for i in want if i % 2 == 0] or want)[0]


def nearest_int4(q: np.float32) -> int:
    """The integer in -7..7 nearest to q by exact rationals, ties to even."""
    fq = Fraction(float(q))
    cands = sorted((abs(fq - k), k) for k in range(-7, 8))
    best = [k for dv, k in cands if dv == cands[0][0]]
    return ([k for k in best if k % 2 == 0] or best)[0]


def brute_block(blk: np.ndarray, s_t: np.float32):
    """(scale byte, [16 integers]) of one block by exhaustive search."""
    blk = np.asarray(blk, np.float32)
    if not s_t > 0:
        return 0, [0] * 16
    ratio = (np.float32(np.abs(blk).max()) / np.float32(7.0)) / np.float32(s_t)
    e = nearest_e4m3_byte(ratio)
    d = np.float32(np.float32(lib_e4m3(np.uint8(e))) * np.float32(s_t))
    if d == 0:
        return e, [0] * 16
    return e, [nearest_int4(np.float32(v) / d) for v in blk]


def test_int4_encode_matches_numpy_rint():
    quarter = np.arange(-48, 49, dtype=np.float32) / 4  # every half-integer tie in [-12, 12]
    rng = np.random.default_rng(70)
    rand = (rng.standard_normal(20000) * 5).astype(np.float32)
    edge = np.array([0.0, -0.0, 7.4999995, 7.5, -7.5, 8.0, -8.0, 1e30, -1e30, np.inf, -np.inf],
                    np.float32)
    v = np.concatenate([quarter, rand, edge])
    want = (np.clip(np.rint(v.astype(np.float64)), -7, 7).astype(np.int64)) & 15
    np.testing.assert_array_equal(oracle.int4_encode(v), want.astype(np.uint8))
    # ties go to the even integer: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, -3.5 -> -4
    np.testing.assert_array_equal(lib_int4(oracle.int4_encode([0.5, 1.5, 2.5, -3.5])), [0, 2, 2, -4])


def test_int4_decode_twos_complement():
    c = np.arange(16, dtype=np.uint8)
    np.testing.assert_array_equal(oracle.int4_decode(c), lib_int4(c).astype(np.float32))
    # the encoder's range is symmetric: -8 (nibble 8) is never written
    assert 8 not in set(oracle.int4_encode(np.linspace(-100, 100, 4001)).tolist())


def test_int4_grid_inputs_are_fixed_points():
    """A block whose values are integers times an exactly representable d, with
    its maximum at 7 d, quantizes to exactly those integers (closed form)."""
    ints = np.array([0, 1, -1, 2, -2, 3, -3, 4, -4, 5, -5, 6, -6, 7, -7, 0], np.float32)
    for s_t, e_byte in ((1.0, 0x40), (0.25, 0x50), (2.0 ** -6, 0x70)):
        # d = E4M3(e) * s_t = 2; amax = 14 -> r = (14 / 7) / s_t = 2 / s_t = E4M3 value of e
        y = (ints * 2.0).astype(np.float32)[None, :]
        codes, scales = oracle.int4_quantize(y, s_t)
        assert int(scales[0, 0]) == e_byte
        np.testing.assert_array_equal(lib_int4(oracle.unpack_codes(codes))[0], ints.astype(np.int64))
        np.testing.assert_array_equal(oracle.int4_dequantize(codes, scales, s_t), y)


@pytest.mark.parametrize("seed,scale", [(71, 1.0), (72, 1e-3), (73, 300.0)])
def test_int4_quantize_by_brute_force(seed, scale):
    rng = np.random.default_rng(seed)
    M, K = 4, 128
    y = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    y[1, 16:32] = 0.0                                    # an all-zero block
    y[2, :16] *= np.float32(40.0)                        # a block far above the rest
    s_t = np.float32(np.abs(y).max() / np.float32(3136.0))
    assert np.float32(oracle.int4_tensor_scale(np.abs(y).max())) == s_t
    codes, scales = oracle.int4_quantize(y, s_t)
    u = lib_int4(oracle.unpack_codes(codes))
    for r in range(M):
        for b in range(K // 16):
            e, ints = brute_block(y[r, 16 * b:16 * b + 16], s_t)
            assert int(scales[r, b]) == e, (r, b)
            assert u[r, 16 * b:16 * b + 16].tolist() == ints, (r, b)


def test_int4_tensor_scale_puts_the_maximum_on_the_top_integer():
    """s_t = amax / 3136: the block holding the tensor maximum gets the largest
    E4M3 scale 448 and the maximum element the code +-7."""
    rng = np.random.default_rng(74)
    y = rng.standard_normal((8, 256)).astype(np.float32)
    r, c = np.unravel_index(np.argmax(np.abs(y)), y.shape)
    s_t = oracle.int4_tensor_scale(oracle.amax(y))
    codes, scales = oracle.int4_quantize(y, s_t)
    assert int(scales[r, c // 16]) == 0x7E
    assert abs(int(lib_int4(oracle.unpack_codes(codes))[r, c])) == 7


def test_int4_round_trip_error_bound():
    """Round to nearest: |y - dq| <= d / 2 wherever |y / d| <= 7.5, else the
    clamp error |y| - 7 d, plus the binary32 roundings of y / d and of dq."""
    x = workloads.nvfp4_outliers(256, 1024, seed=75)
    y = oracle.bf16_to_f32(x)
    s_t = np.float32(oracle.int4_tensor_scale(oracle.amax(y)))
    codes, scales = oracle.int4_quantize(y, s_t)
    dq = oracle.int4_dequantize(codes, scales, s_t).astype(np.float64)
    want = (lib_int4(oracle.unpack_codes(codes)) *
            np.repeat(lib_e4m3(scales), 16, axis=1)).astype(np.float32) * s_t
    np.testing.assert_array_equal(dq, want.astype(np.float64))  # value = (int * E4M3) * s_t
    d = np.repeat(lib_e4m3(scales), 16, axis=1).astype(np.float32) * s_t
    d = d.astype(np.float64)
    y64 = y.astype(np.float64)
    v = np.abs(y64) / np.where(d > 0, d, 1)
    bound = np.where(v > 7.5, np.abs(y64) - 7 * d, d / 2)
    err = np.abs(y64 - dq)
    assert np.all(err <= bound * (1 + 2.0 ** -20) + 2.0 ** -23 * np.abs(y64) + 1e-45)
    # with normal E4M3 scales no element needs the clamp (|y / d| < 7 (1 + 2^-4) < 7.5)
    normal = np.repeat((scales & 0x78) != 0, 16, axis=1)
    assert np.all(v[normal] < 7.5)


def test_arc_int4_two_stage_by_brute_force():
    """INT4 variant of the two-stage path: primary half = INT4 of y with
    s_t = amax / 3136; residual half = INT4 with the same s_t of
    r = fl32(y - dq) on the outlier positions, dq = (integer * E4M3) * s_t
    decoded with numpy and ml_dtypes; both halves by exhaustive search."""
    M, K, S = 6, 256, 32
    x, gamma, perm, outl = workloads.arc_activations(M, K, seed=76, S=S, calib_rows=64)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl, fmt="int4")
    s_t = np.float32(s_t)
    assert s_t == np.float32(np.float32(np.abs(y).max()) / np.float32(3136.0))
    assert codes.shape == (M, (K + S) // 2) and scales.shape == (M, (K + S) // 16)
    u = lib_int4(oracle.unpack_codes(codes))
    for row in range(M):
        for b in range(K // 16):
            e, ints = brute_block(y[row, 16 * b:16 * b + 16], s_t)
            assert int(scales[row, b]) == e and u[row, 16 * b:16 * b + 16].tolist() == ints
    prod = (u[:, :K] * np.repeat(lib_e4m3(scales[:, :K // 16]), 16, axis=1)).astype(np.float32)
    dq = (prod * s_t).astype(np.float32)
    r = (y[:, outl] - dq[:, outl]).astype(np.float32)
    for row in range(M):
        for b in range(S // 16):
            e, ints = brute_block(r[row, 16 * b:16 * b + 16], s_t)
            assert int(scales[row, K // 16 + b]) == e, (row, b)
            assert u[row, K + 16 * b:K + 16 * b + 16].tolist() == ints, (row, b)
    # the residual stage is within half a step of r, and two stages beat one
    d_res = (np.repeat(lib_e4m3(scales[:, K // 16:]), 16, axis=1) * float(s_t))
    res = u[:, K:] * d_res
    assert np.all(np.abs(r - res) <= d_res / 2 * (1 + 2.0 ** -20) + 2.0 ** -23 * np.abs(r))
    yo = y.astype(np.float64)[:, outl]
    assert np.linalg.norm(yo - dq[:, outl] - res) < 0.5 * np.linalg.norm(yo - dq[:, outl])
    # linearity of the augmented GEMM with the INT4 operand
    W = np.random.default_rng(77).standard_normal((K, 5))
    full = np.concatenate([dq.astype(np.float64), res], axis=1)
    corrected = dq.astype(np.float64).copy()
    corrected[:, outl] += res
    np.testing.assert_allclose(full @ np.concatenate([W, W[outl]], axis=0), corrected @ W,
                               rtol=1e-12, atol=1e-12)


def test_arc_int4_without_outliers_is_plain_int4():
    x, gamma, perm, _ = workloads.arc_activations(5, 128, seed=78, S=16, calib_rows=32)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, np.zeros(0, np.int32), fmt="int4")
    c1, s1 = oracle.int4_quantize(y, s_t)
    np.testing.assert_array_equal(codes, c1)
    np.testing.assert_array_equal(scales, s1)


def test_arc_int4_alignment_window():
    """Alignment factor phi = d / (amax / 7) of the INT4 two-stage path: within
    1 +- 2^-4 for normal E4M3 scales, so two stages stay within (1 + 2^-3)^2,
    the ARCQuant summary's 1.266 ("Analyse de la Borne d'Erreur Theorique")."""
    x, gamma, perm, outl = workloads.arc_activations(64, 1024, seed=79, S=64, calib_rows=64)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl, fmt="int4")
    pp, pr, np_, nr = oracle.arc_alignment(y, outl, s_t, codes, scales, fmt="int4")
    assert np.nanmax(np.abs(pp[np_] - 1)) <= 2.0 ** -4 + 2.0 ** -20
    assert np.nanmax(np.abs(pr[nr] - 1)) <= 2.0 ** -4 + 2.0 ** -20
    # worst two-stage product over rows whose blocks are all normal
    worst = np.nanmax(np.where(np_, pp, np.nan), axis=1) * np.nanmax(np.where(nr, pr, np.nan), axis=1)
    assert np.nanmax(worst) <= 1.265625 + 1e-9
