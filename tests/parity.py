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


def code_values(codes_packed: np.ndarray, fmt: str = "nvfp4") -> np.ndarray:
    u = oracle.unpack_codes(codes_packed)
    if fmt == "int4":  # 4-bit two's complement integers
        return oracle.int4_decode(u).astype(np.float64)
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


def tolerant_counts(fmt: str, K: int, gpu, orc, y_orc: np.ndarray, name: str = "") -> dict:
    """Element-wise part of the tolerance rule; returns the counts that the
    fraction limits apply to.  gpu/orc = (codes, scales_linear, scale_fp32);
    y_orc: the oracle's unquantized fp32 values."""
    cg, sg, fg = gpu
    co, so, fo = orc
    dg = block_scale(fmt, sg, fg, K)
    do = block_scale(fmt, so, fo, K)
    vg = code_values(cg, fmt) * dg
    vo = code_values(co, fmt) * do
    scale_diff = np.repeat(sg != so, 16 if fmt != "mxfp4" else 32, axis=1)[:, :K]
    n_blocks_diff = int((sg != so).sum())
    if n_blocks_diff:
        diff_bytes = np.abs(sg.astype(np.int64) - so.astype(np.int64))[sg != so]
        assert np.all(diff_bytes <= 1), f"{name}: scale bytes differ by more than one step"
    close = np.abs(vg - vo) <= 1e-3 * np.maximum(do, 1e-300)
    # elements of same-scale blocks that disagree: must be one grid step apart
    bad = ~close & ~scale_diff
    nbad = int(bad.sum())
    if nbad:
        if fmt == "int4":  # the integer is its own grid position
            pg = code_values(cg, fmt)[bad].astype(np.int64)
            po = code_values(co, fmt)[bad].astype(np.int64)
        else:
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
        err = np.abs(vg[scale_diff] - y)
        if fmt == "int4":  # unit steps, clamp at 7
            bound = np.where(v > 7, (v - 7 + 1e-3) * dg[scale_diff], (0.5 + 1e-3) * dg[scale_diff])
        else:
            step = np.where(v <= 2, 0.5, np.where(v <= 4, 1.0, 2.0))
            bound = np.where(v > 6, (v - 6 + 1e-3) * dg[scale_diff], (step / 2 + 1e-3) * dg[scale_diff])
        assert np.all(err <= bound * (1 + 1e-6)), f"{name}: error bound violated in rescaled blocks"
    return {"codes_off": nbad, "blocks_rescaled": n_blocks_diff, "n": int(vg.size),
            "n_blocks": int(sg.size)}


def check_fractions(c: dict, frac: float = 1e-4, name: str = "") -> dict:
    """The fraction limits of the tolerance rule on (summed) counts."""
    allow = max(1, math.ceil(frac * c["n"]))
    assert c["blocks_rescaled"] <= max(1, math.ceil(frac * c["n_blocks"])), (
        f"{name}: {c['blocks_rescaled']} of {c['n_blocks']} scale bytes differ")
    assert c["codes_off"] <= allow, f"{name}: {c['codes_off']} of {c['n']} codes differ (allowed {allow})"
    return c


def assert_tolerant(fmt: str, K: int, gpu, orc, y_orc: np.ndarray, *, frac: float = 1e-4,
                    name: str = ""):
    """gpu/orc = (codes, scales_linear, scale_fp32).  y_orc: oracle's unquantized fp32."""
    return check_fractions(tolerant_counts(fmt, K, gpu, orc, y_orc, name), frac, name)


def add_counts(a: dict | None, b: dict) -> dict:
    return dict(b) if a is None else {k: a[k] + b[k] for k in a}


def arc_counts(fmt: str, K: int, outl, gpu, orc_primary, y_orc: np.ndarray, name: str = "") -> dict:
    """Tolerance counts of an ARCQuant output row block [primary K | residual S].

    The primary columns are compared with the oracle's quantization of y.  The
    residual columns are compared with the oracle's quantization of the
    residual of the kernel's OWN primary codes, r = y - dq(primary), since the
    residual is defined against the primary value actually produced (ARCQuant
    summary, Methodologie item 2); a primary code one step off (allowed by the
    rule) would otherwise shift its residual by a whole primary step.
    gpu = (codes [M, (K+S)/2], linear scales [M, (K+S)/B], s_t or None);
    orc_primary = (codes [M, K/2], scales [M, K/B], s_t or None)."""
    cg, sg, fg = gpu
    co, so, fo = orc_primary
    B = 32 if fmt == "mxfp4" else 16
    c = tolerant_counts(fmt, K, (cg[:, :K // 2], sg[:, :K // B], fg), (co, so, fo), y_orc, name)
    S = len(outl)
    if S == 0:
        return c
    if fmt == "mxfp4":
        dq = oracle.mxfp4_dequantize(cg[:, :K // 2], sg[:, :K // B])
    elif fmt == "int4":
        dq = oracle.int4_dequantize(cg[:, :K // 2], sg[:, :K // B], float(np.asarray(fg).reshape(-1)[0]))
    else:
        dq = oracle.nvfp4_dequantize(cg[:, :K // 2], sg[:, :K // B], float(np.asarray(fg).reshape(-1)[0]))
    r = (np.asarray(y_orc, np.float32)[:, outl] - dq[:, outl]).astype(np.float32)
    if fmt == "mxfp4":
        cr, sr = oracle.mxfp4_quantize(r)
    elif fmt == "int4":
        cr, sr = oracle.int4_quantize(r, fo)
    else:
        cr, sr = oracle.nvfp4_quantize(r, fo)
    c2 = tolerant_counts(fmt, S, (cg[:, K // 2:], sg[:, K // B:], fg), (cr, sr, fo), r, name + "-residual")
    return add_counts(c, c2)


def _bf16_boundary_distance(w: np.ndarray) -> np.ndarray:
    """Distance (float64) from each fp32 value to the nearest bf16 rounding
    boundary: the midpoints between |w|'s two bf16 neighbours and between the
    lower neighbour and the bf16 value below it."""
    a = np.abs(np.asarray(w, np.float32))
    u = a.view(np.uint32)
    lo_b = u & np.uint32(0xFFFF0000)
    lo = lo_b.view(np.float32).astype(np.float64)
    hi = (lo_b + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    below = np.where(lo_b > 0, lo_b - np.uint32(0x10000), np.uint32(0)).view(np.float32).astype(np.float64)
    below = np.where(lo_b > 0, below, -lo)
    a64 = a.astype(np.float64)
    return np.minimum(np.abs((lo + hi) / 2 - a64), a64 - (below + lo) / 2)


def assert_roundtrip(got_bits: np.ndarray, want_f32: np.ndarray, n: int, name: str = "") -> dict:
    """bf16 output of an inverse-Hadamard dequantizer against the oracle.

    `want_f32` is the oracle's value w: the binary64 product H_n * dq rounded
    once to fp32.  The kernels compute the same product in fp32 (one rounding
    of the folded multiplier at decode, then log2(n) butterfly stages).  Each
    rounding adds an error of at most 2^-24 of the value it rounds; an
    unnormalised butterfly stage multiplies the l2 norm of an error vector by
    sqrt(2), so the errors of all stages, carried to the output, stay below
    (log2(n) + 6) * 2^-24 * ||w_block||_2 in every element (3 decode roundings
    and a margin of 3).  With the 2^-24 |w| of the oracle's own fp32 rounding
    this is the window delta.  Consequences checked here:
      * an element whose w lies farther than delta from every bf16 rounding
        boundary is BIT-EXACT (both sides round the same value the same way);
      * inside the window the two results may be the two bf16 neighbours of
        the boundary: |got - w| <= one bf16 ulp + delta.
    The dequantized inputs carry few significant bits, so many outputs are
    exact bf16 midpoints (ties the oracle rounds to even, the kernel sees a
    few fp32 ulps to one side): this window holds about 1-3 % of the elements,
    and it is the only place a difference is allowed."""
    got = oracle.bf16_to_f32(got_bits).astype(np.float64)
    w = np.asarray(want_f32, np.float32)
    want_bits = oracle.f32_to_bf16(w)
    M, K = w.shape
    w64 = w.astype(np.float64)
    L = int(round(math.log2(n)))
    blk = np.sqrt(np.square(w64).reshape(M, K // n, n).sum(axis=2))
    delta = (L + 6) * 2.0 ** -24 * np.repeat(blk, n, axis=1) + 2.0 ** -24 * np.abs(w64)
    window = _bf16_boundary_distance(w) <= delta
    g_bits = np.asarray(got_bits, np.uint16)
    outside_bad = (g_bits != want_bits) & ~window
    assert not outside_bad.any(), (
        f"{name}: {int(outside_bad.sum())} elements outside the rounding window differ; first "
        f"{np.argwhere(outside_bad)[0]}: got {got[outside_bad][0]} want "
        f"{oracle.bf16_to_f32(want_bits)[outside_bad][0]}")
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(w64), np.abs(got)) + 1e-300)) - 7)
    inside_bad = window & (np.abs(got - w64) > ulp + delta)
    assert not inside_bad.any(), (f"{name}: {int(inside_bad.sum())} window elements beyond one "
                                  f"bf16 ulp + delta")
    return {"window": int(window.sum()), "differ": int((g_bits != want_bits).sum()), "n": w.size}


def block_l2_identity(x_bits, xhat_bits, dq_y, y_orc, w_orc, n: int, name: str = ""):
    """Per n-block l2 identity of the round trip (orthonormal H):
    ||x^ - x||_2 = ||y^ - y||_2 with x the bf16 input, y = H x its rotation
    (oracle, fp32), y^ the dequantized codes and x^ = H y^.
      * w_orc = oracle's H y^ (fp32): equal to ||y^ - y|| within 1e-5 relative
        (plus the fp32 roundings of y and w, 2^-23 ||x_block||);
      * the kernel's bf16 x^: within the a-priori bound of its bf16 rounding
        and fp32 error, ||1/2 ulp_bf16(w) + delta||_2 of the block, which does
        not depend on the kernel's output."""
    x = oracle.bf16_to_f32(x_bits).astype(np.float64)
    M, K = x.shape
    nb = K // n
    blocks = lambda a: np.asarray(a, np.float64).reshape(M, nb, n)
    e_y = np.sqrt(np.square(blocks(dq_y) - blocks(y_orc)).sum(axis=2))
    e_w = np.sqrt(np.square(blocks(w_orc) - blocks(x)).sum(axis=2))
    nx = np.sqrt(np.square(blocks(x)).sum(axis=2))
    tol_w = 1e-5 * e_y + 2.0 ** -23 * nx
    assert np.all(np.abs(e_w - e_y) <= tol_w), (
        f"{name}: oracle inverse breaks the l2 identity, worst "
        f"{np.max(np.abs(e_w - e_y) - tol_w)}")
    xh = oracle.bf16_to_f32(xhat_bits).astype(np.float64)
    e_g = np.sqrt(np.square(blocks(xh) - blocks(x)).sum(axis=2))
    w64 = blocks(w_orc)
    L = int(round(math.log2(n)))
    wn = np.sqrt(np.square(w64).sum(axis=2))
    half_ulp = np.exp2(np.floor(np.log2(np.abs(w64) + 1e-300)) - 8)
    per = half_ulp + (L + 6) * 2.0 ** -24 * wn[..., None] + 2.0 ** -24 * np.abs(w64)
    bound = np.sqrt(np.square(per).sum(axis=2)) + tol_w
    assert np.all(np.abs(e_g - e_y) <= bound), (
        f"{name}: kernel round trip breaks the l2 identity, worst excess "
        f"{np.max(np.abs(e_g - e_y) - bound)}")
    return {"rel_err_median": float(np.median(e_y / np.maximum(nx, 1e-300)))}
