"""Pins of the oracle's quantizers, Hadamard, RMSNorm and ARCQuant layout.

Each test checks the oracle against something other than its own code path:
idempotence on inputs built to lie on the format grid, the error bound of
round-to-nearest (half a grid step times the block scale), brute-force nearest
search with exact rationals, library routines (scipy's Hadamard matrix, torch's
rms_norm, ml_dtypes decoders), closed forms, and the linearity identity of the
augmented GEMM.  The methods are the ones the pages describe: NVFP4 blocks of 16
with a per-tensor scale (ARCQuant summary, Enonce du Probleme; nGPT abstract),
MXFP4 with a power-of-two scale and block Hadamard rotations (MR-GPTQ abstract),
micro-grouped dual scales and a two-level FWHT (FP4Quant abstract), and the
two-stage primary + residual quantization appended along K (ARCQuant,
Methodologie items 2-4).
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import workloads

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def lib_decode_codes(codes_packed):
    """Decode packed E2M1 codes with ml_dtypes (low nibble = even index)."""
    u = oracle.unpack_codes(codes_packed)
    return u.view(F4).astype(np.float64)


def lib_decode_e4m3(b):
    return np.asarray(b, np.uint8).view(F8).astype(np.float64)


def grid_step(v):
    """Spacing of the E2M1 grid around |v| (0.5 on [0,2], 1 on [2,4], 2 on [4,6])."""
    a = np.abs(v)
    return np.where(a <= 2, 0.5, np.where(a <= 4, 1.0, 2.0))


# ----------------------------------------------------------------------------- NVFP4

def _on_grid_nvfp4(rng, M, K, s_t):
    """Codes/scales whose dequantized matrix re-quantizes to itself: every block
    holds a +-6 element (so amax_b = 6 * scale) and one block has scale 448 (so
    the tensor amax / 2688 recovers s_t exactly)."""
    nb = K // 16
    codes = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    pos = rng.integers(0, 16, size=(M, nb))
    for r in range(M):
        for b in range(nb):
            codes[r, 16 * b + pos[r, b]] = 7 | (rng.integers(0, 2) << 3)
    scales = rng.integers(1, 0x7F, size=(M, nb), dtype=np.uint8)
    scales[0, 0] = 0x7E
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales


@pytest.mark.parametrize("s_t", [2.0 ** -7, 1.5 * 2.0 ** -9, 0.75])
def test_nvfp4_idempotent_on_grid(s_t):
    rng = np.random.default_rng(20)
    codes, scales = _on_grid_nvfp4(rng, 8, 256, s_t)
    # build the values from the library decoders, exactly, in float64
    y = lib_decode_codes(codes) * np.repeat(lib_decode_e4m3(scales), 16, axis=1) * s_t
    y32 = y.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), y)  # exactly representable
    s2 = oracle.tensor_scale(oracle.amax(y32))
    assert s2 == np.float32(s_t)
    c2, sc2 = oracle.nvfp4_quantize(y32, s2)
    np.testing.assert_array_equal(sc2, scales)
    # -0 and +0 both decode to 0: compare decoded values, and all non-zero codes bitwise
    u1, u2 = oracle.unpack_codes(codes), oracle.unpack_codes(c2)
    nz = (u1 & 7) != 0
    np.testing.assert_array_equal(u1[nz], u2[nz])
    assert np.all((u2[~nz] & 7) == 0)


def test_nvfp4_error_bound_and_brute_force_scale():
    x = workloads.nvfp4_outliers(64, 256, seed=21)
    codes, scales, s_t = oracle.quantize_nvfp4(x)
    y = oracle.bf16_to_f32(x).astype(np.float64)
    # the per-tensor scale: amax / 2688 (one binary32 division)
    assert s_t == np.float32(np.float32(np.abs(y).max()) / np.float32(2688.0))
    # block scale = nearest E4M3 (ties even) to (amax_b/6)/s_t, by exhaustive search
    e4_vals = [Fraction(float(v)) for v in lib_decode_e4m3(np.arange(127))]
    amax_b = np.abs(y).reshape(64, -1, 16).max(axis=2).astype(np.float32)
    r = (amax_b / np.float32(6.0)) / np.float32(s_t)
    for rv, got in zip(r.reshape(-1).tolist(), scales.reshape(-1).tolist()):
        fr = Fraction(rv)
        ds = [abs(fr - v) for v in e4_vals]
        best = min(ds)
        assert ds[got] == best
        if ds.count(best) > 1:
            assert got % 2 == 0
    # error bound: |y - dq| <= step/2 * d  (d = scale * s_t)
    d = np.repeat(lib_decode_e4m3(scales), 16, axis=1) * float(s_t)
    dq = lib_decode_codes(codes) * d
    v = y / d
    assert np.all(np.abs(y - dq) <= grid_step(np.minimum(np.abs(v), 6.0)) / 2 * d * (1 + 1e-6))


def test_nvfp4_codes_nearest_by_brute_force():
    rng = np.random.default_rng(22)
    y = (rng.standard_normal((4, 64)) * np.exp(rng.uniform(-3, 3, (4, 1)))).astype(np.float32)
    s_t = oracle.tensor_scale(oracle.amax(y))
    codes, scales = oracle.nvfp4_quantize(y, s_t)
    u = oracle.unpack_codes(codes)
    dscale = (lib_decode_e4m3(scales) * s_t).astype(np.float32)  # one binary32 rounding
    grid = {c: Fraction(float(v))
            for c, v in enumerate(np.arange(16, dtype=np.uint8).view(F4).astype(np.float64))}
    for r in range(4):
        for k in range(64):
            d = dscale[r, k // 16]
            q = Fraction(float(np.float32(y[r, k]) / np.float32(d)))  # correctly rounded quotient
            neg = np.signbit(np.float32(y[r, k]) / np.float32(d))
            cands = [(abs(q - grid[c]), c) for c in range(16) if bool(c & 8) == bool(neg)]
            best = min(cands)[0]
            assert abs(q - grid[int(u[r, k])]) == best


def test_nvfp4_zero_tensor_and_zero_blocks():
    y = np.zeros((2, 32), np.float32)
    c, s, st = oracle.quantize_nvfp4(oracle.f32_to_bf16(y))
    assert st == 0 and not c.any() and not s.any()
    y[0, :16] = 1.0
    c, s = oracle.nvfp4_quantize(y, oracle.tensor_scale(1.0))
    assert s[0, 1] == 0 and not c[0, 8:].any() and s[0, 0] == 0x7E


# ----------------------------------------------------------------------------- MXFP4

def test_mxfp4_idempotent_on_grid():
    rng = np.random.default_rng(23)
    M, K = 6, 256
    codes = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    for r in range(M):
        for b in range(K // 32):
            codes[r, 32 * b + rng.integers(0, 32)] = rng.choice([6, 7, 14, 15])  # |v| in {4, 6}
    # scale bytes whose decoded values stay normal binary32 for every code
    scales = rng.integers(4, 251, size=(M, K // 32), dtype=np.uint8)
    scales[0, :2] = [4, 250]
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    y = lib_decode_codes(packed) * np.exp2(np.repeat(scales.astype(np.float64) - 127, 32, axis=1))
    y32 = y.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), y)
    c2, s2 = oracle.mxfp4_quantize(y32)
    np.testing.assert_array_equal(s2, scales)
    u1, u2 = oracle.unpack_codes(packed), oracle.unpack_codes(c2)
    nz = (u1 & 7) != 0
    np.testing.assert_array_equal(u1[nz], u2[nz])


def test_mxfp4_error_bound_and_scale_range():
    x = workloads.mxfp4_student_t(64, 512, seed=24)
    codes, scales = oracle.quantize_mxfp4(x)
    y = oracle.bf16_to_f32(x).astype(np.float64)
    amax_b = np.abs(y).reshape(64, -1, 32).max(axis=2)
    ratio = amax_b * np.exp2(127.0 - scales)
    assert np.all((ratio >= 4) & (ratio < 8))  # shared exponent floor(log2 amax) - 2
    d = np.exp2(np.repeat(scales.astype(np.float64), 32, axis=1) - 127)
    dq = lib_decode_codes(codes) * d
    v = np.abs(y / d)
    sat = v > 6
    assert np.all(np.abs(y - dq)[~sat] <= (grid_step(v) / 2 * d)[~sat])
    assert np.all(np.abs(y - dq)[sat] < 2 * d[sat])  # saturated: (|v| - 6) d < 2 d
    # dequantizer: decoded values are exact products
    np.testing.assert_array_equal(oracle.mxfp4_dequantize(codes, scales).astype(np.float64), dq)


# ----------------------------------------------------------------------------- dual

def test_dual_idempotent_on_grid():
    rng = np.random.default_rng(25)
    M, K = 4, 512
    G = 2.0 ** -6
    codes = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    scales = rng.integers(1, 0x7F, size=(M, K // 16), dtype=np.uint8)
    for r in range(M):
        for b in range(K // 16):
            codes[r, 16 * b + rng.integers(0, 16)] = 7
        for g in range(K // 128):
            scales[r, 8 * g + rng.integers(0, 8)] = 0x7E
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    y = lib_decode_codes(packed) * np.repeat(lib_decode_e4m3(scales), 16, axis=1) * G
    y32 = y.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), y)
    c2, s2, g2 = oracle.dual_quantize(y32)
    assert np.all(g2 == np.float32(G))
    np.testing.assert_array_equal(s2, scales)
    u1, u2 = oracle.unpack_codes(packed), oracle.unpack_codes(c2)
    nz = (u1 & 7) != 0
    np.testing.assert_array_equal(u1[nz], u2[nz])


def test_dual_error_bound():
    x = workloads.dual_gain(32, 1024, seed=26)
    y = oracle.bf16_to_f32(x)
    codes, scales, g = oracle.dual_quantize(y)
    y = y.astype(np.float64)
    amax_g = np.abs(y).reshape(32, -1, 128).max(axis=2)
    np.testing.assert_array_equal(g, (amax_g.astype(np.float32) / np.float32(2688)))
    d = np.repeat(lib_decode_e4m3(scales), 16, axis=1) * np.repeat(g.astype(np.float64), 128, axis=1)
    dq = lib_decode_codes(codes) * d
    v = np.abs(y) / np.where(d > 0, d, 1)
    ok = d > 0
    assert np.all((np.abs(y - dq) <= grid_step(np.minimum(v, 6)) / 2 * d * (1 + 1e-6))[ok])
    np.testing.assert_allclose(oracle.dual_dequantize(codes, scales, g), dq.astype(np.float32),
                               rtol=0, atol=0)


def test_nvfp4_dequantize_matches_library_decoders():
    x = workloads.nvfp4_outliers(16, 128, seed=27)
    codes, scales, s_t = oracle.quantize_nvfp4(x)
    prod = lib_decode_codes(codes) * np.repeat(lib_decode_e4m3(scales), 16, axis=1)
    want = (prod.astype(np.float32) * np.float32(s_t))
    np.testing.assert_array_equal(oracle.nvfp4_dequantize(codes, scales, s_t), want)


# ----------------------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("n", [16, 32, 64, 128, 256, 512])
def test_hadamard_matrix_matches_scipy(n):
    H = np.array([[oracle.hadamard_entry(i, j) for j in range(n)] for i in range(n)])
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(n))
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n, dtype=H.dtype))


@pytest.mark.parametrize("n", [16, 32, 128, 512])
def test_hadamard_transform_matches_dense_scipy(n):
    rng = np.random.default_rng(28)
    x = rng.standard_normal((5, 2 * n)).astype(np.float32)
    y = oracle.hadamard(x, n)
    H = scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(n)
    ref = (x.astype(np.float64).reshape(5, 2, n) @ H.T).reshape(5, 2 * n)
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=2 ** -23, atol=1e-30)
    # involution of the normalised matrix
    np.testing.assert_allclose(oracle.hadamard(y, n), x, rtol=0, atol=4e-6 * np.abs(x).max())


def test_two_level_fwht_equals_one_level():
    """H_512 = H_16 (x) H_32: applying the in-block size-32 level and then the
    strided size-16 level gives the single 512 transform (FP4Quant's two levels)."""
    rng = np.random.default_rng(29)
    x = rng.standard_normal((3, 512))
    H32 = scipy.linalg.hadamard(32) / np.sqrt(32)
    H16 = scipy.linalg.hadamard(16) / np.sqrt(16)
    z = x.reshape(3, 16, 32) @ H32.T             # level 1: contiguous 32-blocks
    z = np.einsum("ij,rjk->rik", H16, z)          # level 2: across the 16 blocks
    y = oracle.hadamard(x.astype(np.float32), 512)
    np.testing.assert_allclose(y, z.reshape(3, 512), rtol=1e-6, atol=1e-6)


# ----------------------------------------------------------------------------- RMSNorm / ARC

def test_rmsnorm_permute_matches_torch():
    x, gamma, perm, outl = workloads.arc_activations(16, 512, seed=30, S=32)
    y = oracle.arc_prepare(x, gamma, perm, eps=1e-6)
    xt = torch.from_numpy(oracle.bf16_to_f32(x).astype(np.float64))
    gt = torch.from_numpy(oracle.bf16_to_f32(gamma).astype(np.float64))
    p = torch.from_numpy(perm.astype(np.int64))
    ref = torch.nn.functional.rms_norm(xt[:, p], (512,), weight=gt[p], eps=1e-6)
    np.testing.assert_allclose(y, ref.numpy().astype(np.float32), rtol=2 ** -23, atol=0)


def test_arc_outliers_are_the_scaled_channels():
    x, gamma, perm, outl = workloads.arc_activations(64, 512, seed=31, S=32)
    xv = np.abs(oracle.bf16_to_f32(x)).max(axis=0)
    top = set(np.argsort(-xv)[:32].tolist())
    assert len(top & set(perm[:32].tolist())) >= 30


def test_arc_residual_layout_and_linearity():
    x, gamma, perm, outl = workloads.arc_activations(8, 256, seed=32, S=32)
    M, K, S = 8, 256, 32
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl)
    assert codes.shape == (M, (K + S) // 2) and scales.shape == (M, (K + S) // 16)
    # primary half equals plain NVFP4 of the prepared matrix
    c1, s1 = oracle.nvfp4_quantize(y, s_t)
    np.testing.assert_array_equal(codes[:, : K // 2], c1)
    np.testing.assert_array_equal(scales[:, : K // 16], s1)
    # decode both halves with the library decoders
    dq = lib_decode_codes(codes) * np.repeat(lib_decode_e4m3(scales), 16, axis=1) * float(s_t)
    prim, res = dq[:, :K], dq[:, K:]
    yo = y.astype(np.float64)[:, outl]
    r_true = yo - prim[:, outl]
    # residual codes approximate the primary error of the outlier channels to
    # round-to-nearest accuracy: half a grid step times the residual block's
    # scale d (saturated elements: (|v| - 6) d), plus the binary32 rounding of
    # the residual itself (2^-24 |r|)
    d_res = np.repeat(lib_decode_e4m3(scales[:, K // 16:]), 16, axis=1) * float(s_t)
    v = np.abs(r_true) / d_res
    bound = np.where(v > 6, v - 6, grid_step(v) / 2) * d_res
    assert np.all(np.abs(r_true - res) <= bound * (1 + 1e-6) + 2.0 ** -24 * np.abs(r_true))
    # two-stage error is below the primary error on the outliers (on aggregate)
    assert np.linalg.norm(yo - prim[:, outl] - res) < 0.5 * np.linalg.norm(yo - prim[:, outl])
    # linearity of the augmented GEMM: [Q(x) | Q(r)] @ [W ; W_S] equals (Q(x) + Q(r) on S) @ W
    rng = np.random.default_rng(33)
    W = rng.standard_normal((K, 7))
    W_aug = np.concatenate([W, W[outl]], axis=0)
    corrected = prim.copy()
    corrected[:, outl] += res
    np.testing.assert_allclose(dq @ W_aug, corrected @ W, rtol=1e-12, atol=1e-12)



def test_arc_residual_half_by_brute_force():
    """The residual columns are the NVFP4 quantization, with the primary's s_t,
    of r = fl32(y - dq) on the outlier positions (ARCQuant, Methodologie item 2:
    residual = original - primary), found here by exhaustive search with exact
    rationals: the scale byte nearest (ties even) to (amax_r / 6) / s_t, then
    each code nearest (ties to the even code, sign kept) to fl32(r / d)."""
    M, K, S = 6, 128, 32
    x, gamma, perm, outl = workloads.arc_activations(M, K, seed=35, S=S, calib_rows=64)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl)
    s_t = np.float32(s_t)
    prod = (lib_decode_codes(codes[:, : K // 2]) *
            np.repeat(lib_decode_e4m3(scales[:, : K // 16]), 16, axis=1)).astype(np.float32)
    dq = prod * s_t  # binary32 product (the first one is exact)
    r = (y[:, outl] - dq[:, outl]).astype(np.float32)
    e4_vals = [Fraction(float(v)) for v in lib_decode_e4m3(np.arange(127))]
    grid = {c: Fraction(float(v))
            for c, v in enumerate(np.arange(16, dtype=np.uint8).view(F4).astype(np.float64))}
    u = oracle.unpack_codes(codes[:, K // 2:])
    for row in range(M):
        for b in range(S // 16):
            blk = r[row, 16 * b:16 * b + 16]
            ratio = (np.float32(np.abs(blk).max()) / np.float32(6.0)) / s_t
            ds = [abs(Fraction(float(ratio)) - v) for v in e4_vals]
            best = min(ds)
            want = [i for i, dv in enumerate(ds) if dv == best]
            want = [i for i in want if i % 2 == 0] or want
            assert int(scales[row, K // 16 + b]) == want[0]
            d = np.float32(lib_decode_e4m3(np.uint8(want[0])) * s_t)
            for k in range(16):
                q32 = np.float32(blk[k]) / d if d > 0 else np.float32(0)
                q = Fraction(float(q32))
                neg = bool(np.signbit(q32))
                cands = sorted((abs(q - grid[c]), c) for c in range(16) if bool(c & 8) == neg)
                best_c = [c for dv, c in cands if dv == cands[0][0]]
                best_c = [c for c in best_c if c % 2 == 0] or best_c
                if d == 0:
                    assert u[row, 16 * b + k] == 0
                else:
                    assert u[row, 16 * b + k] == best_c[0], (row, b, k)


def _floor_log2_exact(a: float) -> int:
    """floor(log2 a) for a > 0 by exact rational comparison."""
    fa = Fraction(a)
    e = 0
    while Fraction(2) ** e > fa:
        e -= 1
    while Fraction(2) ** (e + 1) <= fa:
        e += 1
    return e


def test_arc_mxfp4_two_stage_by_brute_force():
    """MXFP4 variant of the two-stage path (ARCQuant summary, Generalisabilite:
    the scheme carries over to MXFP4; MR-GPTQ abstract: 32-element blocks with a
    power-of-two scale).  Primary half: MXFP4 of y.  Residual half: MXFP4 of
    r = fl32(y - dq) on the outlier positions, dq = E2M1val * 2^(b-127) decoded
    with ml_dtypes; the residual scale byte is floor(log2 amax_r) - 2 + 127 by
    exact rational search, each code the nearest grid value (ties to the even
    code, sign kept) of r * 2^(127-b), which is exact."""
    M, K, S = 6, 256, 64
    x, gamma, perm, outl = workloads.arc_activations(M, K, seed=36, S=S, calib_rows=64)
    codes, scales, s_t, y = oracle.arc(x, gamma, perm, outl, fmt="mxfp4")
    assert s_t is None and codes.shape == (M, (K + S) // 2) and scales.shape == (M, (K + S) // 32)
    c1, s1 = oracle.mxfp4_quantize(y)
    np.testing.assert_array_equal(codes[:, : K // 2], c1)
    np.testing.assert_array_equal(scales[:, : K // 32], s1)
    dq = lib_decode_codes(codes[:, : K // 2]) * np.exp2(
        np.repeat(scales[:, : K // 32].astype(np.float64), 32, axis=1) - 127)
    assert np.array_equal(dq.astype(np.float32).astype(np.float64), dq)  # exact in binary32
    r = (y[:, outl] - dq[:, outl].astype(np.float32)).astype(np.float32)
    grid = {c: Fraction(float(v))
            for c, v in enumerate(np.arange(16, dtype=np.uint8).view(F4).astype(np.float64))}
    u = oracle.unpack_codes(codes[:, K // 2:])
    for row in range(M):
        for b in range(S // 32):
            blk = r[row, 32 * b:32 * b + 32]
            am = float(np.abs(blk).max())
            want_b = 0 if am == 0 else min(254, max(0, _floor_log2_exact(am) - 2 + 127))
            assert int(scales[row, K // 32 + b]) == want_b
            for k in range(32):
                if am == 0:
                    assert u[row, 32 * b + k] == 0
                    continue
                v = Fraction(float(blk[k])) * Fraction(2) ** (127 - want_b)
                neg = bool(np.signbit(blk[k]))
                cands = sorted((abs(abs(v) - grid[c & 7]), c) for c in range(16)
                               if bool(c & 8) == neg)
                best = [c for dv, c in cands if dv == cands[0][0]]
                best = [c for c in best if c % 2 == 0] or best
                assert u[row, 32 * b + k] == best[0], (row, b, k)
    # error bound of the residual stage, and the two stages beat one on the outliers
    res = lib_decode_codes(codes[:, K // 2:]) * np.exp2(
        np.repeat(scales[:, K // 32:].astype(np.float64), 32, axis=1) - 127)
    d = np.exp2(np.repeat(scales[:, K // 32:].astype(np.float64), 32, axis=1) - 127)
    v = np.abs(r.astype(np.float64)) / d
    bound = np.where(v > 6, v - 6, grid_step(v) / 2) * d
    assert np.all(np.abs(r - res) <= bound * (1 + 1e-9))
    yo = y.astype(np.float64)[:, outl]
    assert np.linalg.norm(yo - dq[:, outl] - res) < 0.5 * np.linalg.norm(yo - dq[:, outl])
    # linearity of the augmented GEMM with the MXFP4 operand
    W = np.random.default_rng(37).standard_normal((K, 5))
    full = np.concatenate([dq, res], axis=1)
    corrected = dq.copy()
    corrected[:, outl] += res
    np.testing.assert_allclose(full @ np.concatenate([W, W[outl]], axis=0), corrected @ W,
                               rtol=1e-12, atol=1e-12)

# ----------------------------------------------------------------------------- swizzle

def test_swizzle_is_a_bijection_with_zero_padding():
    for M, n in [(1, 1), (128, 4), (130, 9), (300, 64), (256, 272)]:
        offs = {oracle.swizzle_offset(r, c, n) for r in range(M) for c in range(n)}
        assert len(offs) == M * n
        size = oracle.swizzled_size(M, n)
        assert max(offs) < size
        lin = np.random.default_rng(34).integers(1, 255, (M, n), dtype=np.uint8)
        sw = oracle.swizzle_scales(lin)
        assert sw.size == size and np.count_nonzero(sw) == M * n


def test_swizzle_tile_structure():
    """Within one 128x4 tile: row r%32 strides 16 bytes, row group (r%128)/32
    strides 4, the scale column strides 1; tiles run along the scale columns."""
    n = 16
    assert oracle.swizzle_offset(0, 0, n) == 0
    assert oracle.swizzle_offset(0, 3, n) == 3
    assert oracle.swizzle_offset(1, 0, n) == 16
    assert oracle.swizzle_offset(31, 0, n) == 496
    assert oracle.swizzle_offset(32, 0, n) == 4
    assert oracle.swizzle_offset(127, 3, n) == 511
    assert oracle.swizzle_offset(0, 4, n) == 512
    assert oracle.swizzle_offset(128, 0, n) == 512 * 4


def test_swizzle_matches_the_block_scaled_gemm_library_layout():
    """The 128x4 tiled scale layout against vLLM's helper that lays out NVFP4
    block scales for the CUTLASS / FlashInfer block-scaled GEMMs (plain torch
    reshapes; its final device copy is bypassed on this CPU-only host)."""
    from unittest import mock

    torch = pytest.importorskip("torch")
    try:
        from vllm.model_executor.layers.quantization.utils.nvfp4_utils import swizzle_blockscale
    except Exception as e:  # not importable here
        pytest.skip(f"vllm helper unavailable: {type(e).__name__}")
    with mock.patch.object(torch.Tensor, "cuda", lambda self, *a, **k: self):
        for M, n in [(1, 1), (128, 4), (130, 9), (300, 64), (256, 272)]:
            lin = np.random.default_rng(M + n).integers(1, 127, (M, n), dtype=np.uint8)
            ref = swizzle_blockscale(torch.from_numpy(lin).view(torch.float8_e4m3fn))
            want = ref.contiguous().view(torch.uint8).numpy().reshape(-1)
            assert np.array_equal(oracle.swizzle_scales(lin), want), (M, n)


# ----------------------------------------------------------------------------- random-sign rotation

def _pattern(words, p):
    """+-1 per channel of the period from the bit mask (independent of the oracle's helper)."""
    bits = np.unpackbits(np.asarray(words, np.uint32).view(np.uint8), bitorder="little")[:p]
    return 1.0 - 2.0 * bits.astype(np.float64)


@pytest.mark.parametrize("n", [16, 32, 128, 512])
def test_random_sign_hadamard_matches_scipy(n):
    """H_n D per block against scipy's Hadamard matrix times the sign diagonal
    (period min(n, 128)); orthonormal (norms kept) and inverted by D H."""
    rng = np.random.default_rng(40 + n)
    K = 2 * n
    x = rng.standard_normal((3, K)).astype(np.float32)
    words = workloads.random_signs(min(n, 128), seed=n)
    d = np.tile(_pattern(words, min(n, 128)), K // min(n, 128))
    H = scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(n)
    ref = ((x.astype(np.float64) * d).reshape(3, K // n, n) @ H.T).reshape(3, K)
    y = oracle.hadamard(x, n, words)
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=2 ** -23, atol=1e-30)
    np.testing.assert_allclose(np.linalg.norm(y.reshape(3, -1, n), axis=2),
                               np.linalg.norm(x.reshape(3, -1, n).astype(np.float64), axis=2), rtol=1e-6)
    # the inverse through the dequantizer's path: D H y = x
    back = oracle.hadamard(y, n) * d.astype(np.float32)
    np.testing.assert_allclose(back, x, rtol=0, atol=4e-6 * np.abs(x).max())
