"""Pins of the oracle's format encoders/decoders against independent sources.

The oracle (plain C, ``oracle/fp4q_oracle.c``) is checked here against things
other than itself: the ml_dtypes and torch implementations of the OCP
FP4 (E2M1) and FP8 (E4M3FN) formats, exact rational arithmetic (``fractions``),
and brute-force nearest-value search.  The formats are the ones the pages name:
E2M1 elements (ARCQuant summary, Methodologie item 1), E4M3 block scales for
NVFP4 and the power-of-two (E8M0) scale of MXFP4 (MR-GPTQ abstract, point (2)).
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _neighbours(values, n_ulp=6):
    """Every binary32 within n_ulp ulps of each value (both signs)."""
    out = []
    for v in values:
        b = np.array([v], np.float32).view(np.int32)[0]
        for d in range(-n_ulp, n_ulp + 1):
            out.append(np.array([b + d], np.int32).view(np.float32)[0])
    out = np.array(out, np.float32)
    out = out[np.isfinite(out)]
    return np.concatenate([out, -out])


E2M1_POINTS = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0,
               6.5, 7.0, 8.0, 1e-30, 1e30]


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ours = oracle.e2m1_decode(codes)
    ref = codes.view(F4).astype(np.float32)
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_e2m1_value_set_is_the_fp4_grid():
    vals = sorted(set(np.abs(oracle.e2m1_decode(np.arange(16))).tolist()))
    assert vals == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_matches_ml_dtypes_around_every_midpoint():
    v = _neighbours(E2M1_POINTS)
    ours = oracle.e2m1_encode(v)
    ref = v.astype(F4).view(np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_e2m1_encode_matches_ml_dtypes_random():
    rng = np.random.default_rng(10)
    v = np.concatenate([
        rng.uniform(-8, 8, 200000),
        np.exp(rng.uniform(-20, 5, 100000)) * rng.choice([-1, 1], 100000),
    ]).astype(np.float32)
    np.testing.assert_array_equal(oracle.e2m1_encode(v), v.astype(F4).view(np.uint8))


def test_e2m1_encode_special_values():
    v = np.array([0.0, -0.0, np.inf, -np.inf, 1e38, -1e38, 1e-45, -1e-45], np.float32)
    assert oracle.e2m1_encode(v).tolist() == [0x0, 0x8, 0x7, 0xF, 0x7, 0xF, 0x0, 0x8]


def test_e2m1_encode_is_nearest_by_brute_force():
    """Exact-rational nearest search over the 15 distinct values, ties to the even code."""
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.uniform(-7, 7, 3000), _neighbours(E2M1_POINTS, 2)]).astype(np.float32)
    grid = [(c, Fraction(float(oracle.e2m1_decode(np.uint8(c))))) for c in range(16)]
    got = oracle.e2m1_encode(v)
    for x, g in zip(v.tolist(), got.tolist()):
        fx = Fraction(x)
        cands = [(abs(fx - val), c & 1, c) for c, val in grid
                 if (c & 8) == (8 if np.signbit(np.float32(x)) else 0)]
        best = min(cands)
        assert abs(fx - grid[g][1]) == best[0]
        if sum(1 for d, _, _ in cands if d == best[0]) > 1:  # a tie: the even code wins
            assert (g & 1) == 0


def test_e4m3_decode_all_bytes_matches_ml_dtypes_and_torch():
    b = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(b)
    ref = b.view(F8).astype(np.float32)
    tref = torch.from_numpy(b).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert nan.tolist() == np.isnan(ours).tolist() == np.isnan(tref).tolist()
    assert sorted(np.nonzero(nan)[0].tolist()) == [0x7F, 0xFF]
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), tref[~nan].view(np.uint32))
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_encode_matches_libraries_in_range():
    """Inside the finite range (|r| <= 464, where no library overflows) the
    oracle's round-to-nearest-even equals ml_dtypes and torch."""
    pts = oracle.e4m3_decode(np.arange(127, dtype=np.uint8)).astype(np.float64)
    mids = (pts[1:] + pts[:-1]) / 2
    v = _neighbours(np.concatenate([pts, mids, [464.0]]).astype(np.float32).tolist(), 4)
    rng = np.random.default_rng(12)
    v = np.concatenate([v, np.exp(rng.uniform(np.log(1e-5), np.log(460), 200000)).astype(np.float32)])
    v = v[np.abs(v) <= 464]
    ours = oracle.e4m3_encode(v)
    np.testing.assert_array_equal(ours, v.astype(F8).view(np.uint8))
    tref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, tref)


def test_e4m3_encode_saturates():
    v = np.array([448.0, 463.9, 464.0, 470.0, 1e6, np.inf], np.float32)
    assert oracle.e4m3_encode(v).tolist() == [0x7E] * 6
    assert oracle.e4m3_encode(np.array([-1e6], np.float32)).tolist() == [0xFE]


def _floor_log2_exact(a: float) -> int:
    f = Fraction(a)
    e = 0
    while Fraction(2) ** (e + 1) <= f:
        e += 1
    while Fraction(2) ** e > f:
        e -= 1
    return e


def test_e8m0_exponent_by_exact_search():
    rng = np.random.default_rng(13)
    vals = np.concatenate([
        np.exp(rng.uniform(np.log(1e-44), np.log(3e38), 3000)),
        [2.0 ** k for k in range(-149, 128)],
        [np.nextafter(np.float32(2.0 ** k), np.float32(0)) for k in range(-120, 120)],
    ]).astype(np.float32)
    vals = vals[vals > 0]
    for a in vals.tolist():
        assert oracle.floor_log2(a) == _floor_log2_exact(a), a
    b = oracle.e8m0_encode(vals).astype(np.int64)
    E = np.array([_floor_log2_exact(a) for a in vals.tolist()]) - 2
    np.testing.assert_array_equal(b, np.clip(E + 127, 0, 254))
    # amax * 2^-E lies in [4, 8) wherever the byte is not clamped
    ok = (E + 127 >= 0) & (E + 127 <= 254)
    ratio = vals[ok].astype(np.float64) * np.exp2(-(b[ok] - 127).astype(np.float64))
    assert np.all((ratio >= 4) & (ratio < 8))


def test_e8m0_zero_block_and_decode():
    assert oracle.e8m0_encode(np.array([0.0], np.float32)).tolist() == [0]
    assert oracle.e8m0_decode(np.array([127, 0, 254], np.uint8)).tolist() == [
        1.0, 2.0 ** -127, 2.0 ** 127]


def test_bf16_round_trip_matches_torch():
    rng = np.random.default_rng(14)
    x = np.concatenate([rng.standard_normal(100000) * 10,
                        np.exp(rng.uniform(-80, 80, 100000))]).astype(np.float32)
    # exact ties: the low 16 bits = 0x8000
    ties = (rng.integers(0, 2**31, 1000, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    x = np.concatenate([x, ties.astype(np.uint32).view(np.float32)])
    x = x[np.isfinite(x)]
    ours = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = oracle.bf16_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())
