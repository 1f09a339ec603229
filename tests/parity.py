"""Comparison helpers for the GPU-vs-oracle parity tests.

Two bars, as the method fixes them:
  * quantize-only paths (NVFP4, MXFP4, dual scale without rotation) and every
    dequantizer without rotation: packed codes, scale bytes and fp32 scales are
    BIT-EXACT;
  * paths with a Hadamard rotation or RMSNorm (the GPU computes the transform
    in fp32 butterflies / fp32 normalisation, the oracle in binary64 rounded
    once): the dequantized values agree within |delta| <= 1e-3 * block scale,
    at most 1e-4 of the codes are off by one grid step, and at most 1e-4 of the
    blocks carry a scale byte one E4M3 step apart (a block amax sitting on an
    E4M3 rounding boundary); elements of such blocks must still meet the
    round-to-nearest error bound against the oracle's unquantized value.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

E2M1_MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bf16_torch_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_torch_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def code_values(codes_packed: np.ndarray) -> np.ndarray:
    u = oracle.unpack_codes(codes_packed)
    mag = E2M1_MAG[u & 7]
    return np.where(u & 8, -mag, mag)


def block_scale(fmt: str, scales: np.ndarray, scale, K: int) -> np.ndarray:
    """Per-element block scale d (float64) from scale bytes (+ fp32 scale)."""
    if fmt == "mxfp4":
        return np.exp2(np.repeat(scales.astype(np.float64), 32, axis=1)[:, :K] - 127)
    e = np.repeat(oracle.e4m3_decode(scales).astype(np.float64), 16, axis=1)[:, :K]
    if fmt == "dual":
        g = np.repeat(np.asarray(scale, np.float64), 128, axis=1)[:, :K]
        return (e * g)
    return e * float(np.asarray(scale).reshape(-1)[0])


def unswizzle(buf: np.ndarray, M: int, ncols: int) -> np.ndarray:
    nC = (ncols + 3) // 4
    r = np.arange(M)[:, None]
    c = np.arange(ncols)[None, :]
    off = ((r // 128) * nC + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    return buf.reshape(-1)[off]


def assert_bitexact(name: str, got: np.ndarray, want: np.ndarray):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, f"{name}: shape {got.shape} != {want.shape}"
    if got.dtype.kind == "f":
        got = got.view(np.uint32 if got.dtype.itemsize == 4 else np.uint16)
        want = want.view(got.dtype)
    bad = np.argwhere(got != want)
    if bad.size:
        idx = tuple(bad[0])
        raise AssertionError(f"{name}: {len(bad)} mismatches, first at {idx}: "
                             f"got {got[idx]!r} want {want[idx]!r}")


def assert_tolerant(fmt: str, K: int, gpu, orc, y_orc: np.ndarray, *, frac: float = 1e-4,
                    name: str = ""):
    """gpu/orc = (codes, scales_linear, scale_fp32).  y_orc: oracle's unquantized fp32."""
    cg, sg, fg = gpu
    co, so, fo = orc
    dg = block_scale(fmt, sg, fg, K)
    do = block_scale(fmt, so, fo, K)
    vg = code_values(cg) * dg
    vo = code_values(co) * do
    n = vg.size
    allow = max(1, math.ceil(frac * n))
    scale_diff = np.repeat(sg != so, 16 if fmt != "mxfp4" else 32, axis=1)[:, :K]
    n_blocks = sg.size
    n_blocks_diff = int((sg != so).sum())
    assert n_blocks_diff <= max(1, math.ceil(frac * n_blocks)), (
        f"{name}: {n_blocks_diff} of {n_blocks} scale bytes differ")
    if n_blocks_diff:
        diff_bytes = np.abs(sg.astype(np.int64) - so.astype(np.int64))[sg != so]
        assert np.all(diff_bytes <= 1), f"{name}: scale bytes differ by more than one step"
    close = np.abs(vg - vo) <= 1e-3 * np.maximum(do, 1e-300)
    # elements of same-scale blocks that disagree: must be one grid step apart
    bad = ~close & ~scale_diff
    nbad = int(bad.sum())
    assert nbad <= allow, f"{name}: {nbad} of {n} codes differ (allowed {allow})"
    if nbad:
        ug = oracle.unpack_codes(cg)[bad]
        uo = oracle.unpack_codes(co)[bad]
        # position on the signed grid: -7..-1, 0, 1..7
        pg = np.where(ug & 8, -(ug & 7).astype(np.int64), (ug & 7).astype(np.int64))
        po = np.where(uo & 8, -(uo & 7).astype(np.int64), (uo & 7).astype(np.int64))
        assert np.all(np.abs(pg - po) <= 1), f"{name}: codes more than one grid step apart"
    # elements of blocks whose scale differs: round-to-nearest bound against y_orc
    if n_blocks_diff:
        y = y_orc.astype(np.float64)[scale_diff]
        v = np.abs(y) / np.maximum(dg[scale_diff], 1e-300)
        step = np.where(v <= 2, 0.5, np.where(v <= 4, 1.0, 2.0))
        err = np.abs(vg[scale_diff] - y)
        bound = np.where(v > 6, (v - 6 + 1e-3) * dg[scale_diff], (step / 2 + 1e-3) * dg[scale_diff])
        assert np.all(err <= bound * (1 + 1e-6)), f"{name}: error bound violated in rescaled blocks"
    return {"codes_off": nbad, "blocks_rescaled": n_blocks_diff, "n": n}


def assert_roundtrip_close(got_bits: np.ndarray, want_bits: np.ndarray, n: int, name: str = "",
                           max_frac: float = 3e-2):
    """bf16 outputs of an inverse-Hadamard dequantizer against the oracle's.

    The GPU rotates in fp32 butterflies, the oracle in binary64 rounded once;
    the difference before the final bf16 rounding is a few fp32 ulps of the
    Hadamard block's magnitude.  So each element may differ by one bf16 ulp of
    itself (a rounding flip) plus 2^-18 of the block's largest magnitude (a
    cancelled, near-zero element), and at most `max_frac` of them may differ.
    The dequantized inputs carry only a few significant bits, so binary64 sums
    are often exact where fp32 butterflies are not, and single-ulp bf16 flips
    are far more frequent than for random data: about 1.3% of the outputs for
    n = 16 when the fp32 butterflies are replayed on the host in numpy.  The
    element-wise one-ulp bound is the check that catches a wrong sign, index
    or scale."""
    got = oracle.bf16_to_f32(got_bits).astype(np.float64)
    want = oracle.bf16_to_f32(want_bits).astype(np.float64)
    M, K = want.shape
    blk = np.abs(want).reshape(M, K // n, n).max(axis=2)
    blk = np.repeat(blk, n, axis=1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), np.abs(got)) + 1e-300)) - 7)
    diff = np.abs(got - want)
    bound = ulp + 2.0 ** -18 * blk
    bad = diff > bound
    assert not bad.any(), (f"{name}: {int(bad.sum())} elements beyond one bf16 ulp; first "
                           f"{np.argwhere(bad)[0]}: got {got[bad][0]} want {want[bad][0]}")
    assert (diff > 0).mean() <= max_frac, f"{name}: {(diff > 0).mean():.2e} of elements differ"
