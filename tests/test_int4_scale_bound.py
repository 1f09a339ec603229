"""The bound behind the unclamped INT4 fast path of the fused ARC kernel.

INT4 (the symmetric integers -7..7 in the NVFP4 container, block scale
E4M3(amax / 7 / s_t)) clamps each quotient q = v / (E4M3 scale * s_t) to
[-7, 7] before rounding it to the nearest integer.  The kernel skips the clamp
for a block whose scale byte lies in 8..0x7d: a normal E4M3 value below 448, so
that the scale was neither saturated nor subnormal.  Then rounding moved the
scale down by at most 2^-4 of the rounded value (three fraction bits), and
every |q| stays below 7 * (1 + 2^-4) = 7.4375 plus a few fp32 roundings, under
7.5, so rounding alone lands in -7..7 and the clamp changes nothing.

These tests follow the kernel's fp32 steps in numpy (RN(1/7), the split
reciprocal's nearest part RN(1/s_t), the E4M3 encoding, d = RN(E4M3(e) * s_t),
RN(1/d), the RMS fold) with the oracle's E4M3 coder, and check:
  * the bound on random and on worst-case inputs (a value just below the
    rounding midpoint above each normal E4M3 value, which rounds down);
  * that the excluded bytes do need the clamp (a saturated 448 and a
    subnormal scale both give quotients above 7.5);
  * that on the same inputs the unclamped rounding equals the oracle's INT4
    encoder, which clamps.
"""
import numpy as np

import oracle

F = np.float32
K7 = F(1.0) / F(7.0)  # RN(1/7) = 0x3e124925


def _quotient_max(amax, s_t, fold):
    """Largest |q| of a block whose largest |v| is amax, by the kernel's steps."""
    amax, s_t, fold = F(amax), F(s_t), F(fold)
    am = (amax * fold).astype(F)                   # block amax of v * fold
    x = ((am * K7).astype(F) * (F(1.0) / s_t).astype(F)).astype(F)
    e = oracle.e4m3_encode(x)
    d = (oracle.e4m3_decode(e) * s_t).astype(F)
    with np.errstate(divide="ignore", over="ignore"):
        m = ((F(1.0) / d).astype(F) * fold).astype(F)
        q = (amax * m).astype(F)
    return e, q


def _in_window(e):
    return (e.astype(np.int64) - 8 >= 0) & (e.astype(np.int64) - 8 < 0x76)


def test_random_blocks_stay_below_7_5():
    rng = np.random.default_rng(11)
    n = 400_000
    s_t = np.exp2(rng.uniform(-40, 40, n)).astype(F)
    fold = np.exp2(rng.uniform(-12, 12, n)).astype(F)
    x = np.exp2(rng.uniform(-10, 9.2, n))          # E4M3 argument, subnormal to saturated
    amax = (x * 7.0 * s_t / fold).astype(F)
    e, q = _quotient_max(amax, s_t, fold)
    win = _in_window(e)
    assert win.sum() > n // 2 and (~win).sum() > n // 20
    assert np.all(np.abs(q[win]) < 7.5)
    assert np.abs(q[win]).max() <= 7.4375 * (1 + 2.0**-20)


def test_worst_case_just_below_each_midpoint():
    vals = oracle.e4m3_decode(np.arange(8, 0x7e, dtype=np.uint8)).astype(np.float64)
    nxt = oracle.e4m3_decode(np.arange(9, 0x7f, dtype=np.uint8)).astype(np.float64)
    mid = (vals + nxt) / 2
    for s_t, fold in ((1.0, 1.0), (2.0**-17 * 3, 1.0), (0.37, 5.5), (1e4, 2.0**-7)):
        x = np.nextafter(mid.astype(F), F(0))      # just below: rounds down to vals
        amax = (x.astype(np.float64) * 7.0 * s_t / fold).astype(F)
        e, q = _quotient_max(amax, F(s_t), F(fold))
        win = _in_window(e)  # (a few ulps of the fp32 steps may cross a midpoint)
        assert win.mean() > 0.95
        assert np.all(np.abs(q[win]) < 7.5), np.abs(q[win]).max()
        assert np.abs(q[win]).max() > 7.3  # the worst case is reached, near 7.4375


def test_excluded_bytes_need_the_clamp():
    # saturated: the E4M3 argument far above 448 keeps the byte at 0x7e
    e, q = _quotient_max(F(7.0 * 1000.0), F(1.0), F(1.0))
    assert int(np.ravel(e)[0]) == 0x7E and float(np.ravel(q)[0]) > 7.5
    # subnormal: 0.0029 rounds to one subnormal step 2^-9 (byte 1)
    e, q = _quotient_max(F(7.0 * 0.0029), F(1.0), F(1.0))
    assert int(np.ravel(e)[0]) < 8 and float(np.ravel(q)[0]) > 7.5


def test_unclamped_rounding_equals_the_clamping_encoder():
    rng = np.random.default_rng(12)
    n = 50_000
    s_t = np.exp2(rng.uniform(-20, 20, n)).astype(F)
    x = np.exp2(rng.uniform(-6, 8.7, n))           # inside the window
    amax = (x * 7.0 * s_t).astype(F)
    e, qmax = _quotient_max(amax, s_t, F(1.0))
    win = _in_window(e)
    # quotients of every value up to the block maximum, both signs
    frac = rng.uniform(-1, 1, n).astype(F)
    q = (qmax * frac).astype(F)[win]
    q = np.concatenate([q, qmax[win], -qmax[win]])
    rounded = np.rint(q.astype(np.float64))        # ties to even, no clamp
    assert np.all(np.abs(rounded) <= 7)
    assert np.array_equal(oracle.int4_decode(oracle.int4_encode(q)), rounded.astype(F))
