"""Python binding of the plain C oracle (``fp4q_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the package smoke check in
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``.  The
CUDA library and its Python binding never import this package; the two share no
code.  Arrays are numpy; bf16 tensors travel as ``uint16`` bit patterns.

Each helper below composes the scalar C steps in the order the pages give them;
the C file's header states the numeric rules and where they come from.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_LIB = None


def lib() -> C.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, f32, f64 = C.c_int64, C.c_float, C.c_double
        p = C.c_void_p
        sig = {
            "orc_bf16_to_f32": (f32, [C.c_uint16]),
            "orc_f32_to_bf16": (C.c_uint16, [f32]),
            "orc_bf16_array_to_f32": (None, [p, i64, p]),
            "orc_f32_array_to_bf16": (None, [p, i64, p]),
            "orc_e2m1_decode": (f32, [C.c_uint8]),
            "orc_e2m1_encode": (C.c_uint8, [f32]),
            "orc_e4m3_decode": (f32, [C.c_uint8]),
            "orc_e4m3_encode": (C.c_uint8, [f32]),
            "orc_floor_log2": (C.c_int, [f32]),
            "orc_e8m0_encode": (C.c_uint8, [f32]),
            "orc_e8m0_decode": (f32, [C.c_uint8]),
            "orc_swizzle_offset": (i64, [i64, i64, i64]),
            "orc_swizzle_scales": (None, [p, i64, i64, p]),
            "orc_amax": (f32, [p, i64, i64, i64]),
            "orc_tensor_scale": (f32, [f32]),
            "orc_nvfp4_quantize": (None, [p, i64, i64, i64, f32, p, p]),
            "orc_mxfp4_quantize": (None, [p, i64, i64, i64, p, p]),
            "orc_dual_quantize": (None, [p, i64, i64, i64, p, p, p]),
            "orc_nvfp4_dequantize": (None, [p, p, f32, i64, i64, p]),
            "orc_dual_dequantize": (None, [p, p, p, i64, i64, p]),
            "orc_mxfp4_dequantize": (None, [p, p, i64, i64, p]),
            "orc_hadamard_entry": (C.c_int, [C.c_int, C.c_int]),
            "orc_hadamard": (None, [p, i64, i64, i64, C.c_int, p]),
            "orc_rmsnorm_permute": (None, [p, i64, i64, i64, p, p, f64, p]),
            "orc_arc_quantize": (None, [p, i64, i64, i64, p, f32, p, p]),
            "orc_arc_quantize_mxfp4": (None, [p, i64, i64, i64, p, p, p]),
            "orc_e2m1_encode_array": (None, [p, i64, p]),
            "orc_e4m3_encode_array": (None, [p, i64, p]),
            "orc_e4m3_decode_array": (None, [p, i64, p]),
            "orc_e8m0_encode_array": (None, [p, i64, p]),
            "orc_int4_encode": (C.c_uint8, [f32]),
            "orc_int4_decode": (f32, [C.c_uint8]),
            "orc_int4_tensor_scale": (f32, [f32]),
            "orc_int4_quantize": (None, [p, i64, i64, i64, f32, p, p]),
            "orc_int4_dequantize": (None, [p, p, f32, i64, i64, p]),
            "orc_arc_quantize_int4": (None, [p, i64, i64, i64, p, f32, p, p]),
            "orc_int4_encode_array": (None, [p, i64, p]),
            "orc_int4_decode_array": (None, [p, i64, p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


# --------------------------------------------------------------------------- formats

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float32)
    lib().orc_bf16_array_to_f32(_ptr(bits), bits.size, _ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = _f32(x)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_array_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_encode(v) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().orc_e2m1_decode(c) for c in range(16)], np.float32)
    return table[codes & 15]


def e4m3_encode(v) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, np.float32)
    lib().orc_e4m3_decode_array(_ptr(b), b.size, _ptr(out))
    return out


def e8m0_encode(amax) -> np.ndarray:
    v = _f32(amax)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e8m0_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e8m0_decode(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    return np.array([lib().orc_e8m0_decode(int(x)) for x in b.reshape(-1)],
                    np.float32).reshape(b.shape)


def floor_log2(a: float) -> int:
    return int(lib().orc_floor_log2(float(a)))


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[M, K/2] packed bytes -> [M, K] 4-bit codes (low nibble = even index)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


# --------------------------------------------------------------------------- layouts

def swizzle_offset(r: int, c: int, n_cols: int) -> int:
    return int(lib().orc_swizzle_offset(r, c, (n_cols + 3) // 4))


def swizzled_size(M: int, n_cols: int) -> int:
    return ((M + 127) // 128 * 128) * ((n_cols + 3) // 4 * 4)


def swizzle_scales(lin: np.ndarray) -> np.ndarray:
    lin = np.ascontiguousarray(lin, dtype=np.uint8)
    M, n = lin.shape
    out = np.empty(swizzled_size(M, n), np.uint8)
    lib().orc_swizzle_scales(_ptr(lin), M, n, _ptr(out))
    return out


# --------------------------------------------------------------------------- steps

def amax(y: np.ndarray) -> float:
    y = _f32(y)
    M, K = y.shape
    return float(lib().orc_amax(_ptr(y), M, K, K))


def tensor_scale(a: float) -> float:
    return float(lib().orc_tensor_scale(float(a)))


def nvfp4_quantize(y: np.ndarray, s_t: float):
    y = _f32(y)
    M, K = y.shape
    assert K % 16 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    lib().orc_nvfp4_quantize(_ptr(y), M, K, K, float(s_t), _ptr(codes), _ptr(scales))
    return codes, scales


def mxfp4_quantize(y: np.ndarray):
    y = _f32(y)
    M, K = y.shape
    assert K % 32 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    lib().orc_mxfp4_quantize(_ptr(y), M, K, K, _ptr(codes), _ptr(scales))
    return codes, scales


def dual_quantize(y: np.ndarray):
    y = _f32(y)
    M, K = y.shape
    assert K % 128 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    g = np.empty((M, K // 128), np.float32)
    lib().orc_dual_quantize(_ptr(y), M, K, K, _ptr(codes), _ptr(scales), _ptr(g))
    return codes, scales, g


def nvfp4_dequantize(codes, scales, s_t: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((M, K), np.float32)
    lib().orc_nvfp4_dequantize(_ptr(codes), _ptr(scales), float(s_t), M, K, _ptr(out))
    return out


def dual_dequantize(codes, scales, gscales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    g = _f32(gscales)
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((M, K), np.float32)
    lib().orc_dual_dequantize(_ptr(codes), _ptr(scales), _ptr(g), M, K, _ptr(out))
    return out


def int4_encode(v) -> np.ndarray:
    """Nibbles of clamp(RNE(v), -7, 7) (4-bit two's complement)."""
    v = _f32(np.atleast_1d(v))
    out = np.empty(v.shape, np.uint8)
    lib().orc_int4_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def int4_decode(codes) -> np.ndarray:
    """Two's complement values of 4-bit codes (one per byte)."""
    c = np.ascontiguousarray(codes, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_int4_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def int4_tensor_scale(a: float) -> float:
    return float(lib().orc_int4_tensor_scale(float(a)))


def int4_quantize(y: np.ndarray, s_t: float):
    y = _f32(y)
    M, K = y.shape
    assert K % 16 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    lib().orc_int4_quantize(_ptr(y), M, K, K, float(s_t), _ptr(codes), _ptr(scales))
    return codes, scales


def int4_dequantize(codes, scales, s_t: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((M, K), np.float32)
    lib().orc_int4_dequantize(_ptr(codes), _ptr(scales), float(s_t), M, K, _ptr(out))
    return out


def mxfp4_dequantize(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((M, K), np.float32)
    lib().orc_mxfp4_dequantize(_ptr(codes), _ptr(scales), M, K, _ptr(out))
    return out


def hadamard_entry(i: int, j: int) -> int:
    return int(lib().orc_hadamard_entry(i, j))


def sign_vector(signs, n: int, K: int) -> np.ndarray:
    """The +-1 diagonal of a random-sign rotation over K channels: bit j of the
    pattern (period p = min(n, 128)) negates channel j of every p channels."""
    p = min(n, 128)
    w = np.asarray(signs, np.uint32)
    bits = np.array([(int(w[j // 32]) >> (j % 32)) & 1 for j in range(p)])
    return np.tile(np.where(bits == 1, -1.0, 1.0), K // p).astype(np.float32)


def hadamard(x: np.ndarray, n: int, signs=None) -> np.ndarray:
    """Normalised block Hadamard of every contiguous n-block; with a sign
    pattern, H_n D x (the randomised transform; D = diag(+-1), applied exactly)."""
    x = _f32(x)
    M, K = x.shape
    assert K % n == 0
    if signs is not None:
        x = x * sign_vector(signs, n, K)[None, :]
    y = np.empty((M, K), np.float32)
    lib().orc_hadamard(_ptr(x), M, K, K, int(n), _ptr(y))
    return y


def rmsnorm_permute(x: np.ndarray, gamma: np.ndarray, perm, eps: float) -> np.ndarray:
    x = _f32(x)
    g = _f32(gamma)
    M, K = x.shape
    y = np.empty((M, K), np.float32)
    pp = None if perm is None else np.ascontiguousarray(perm, np.int32)
    lib().orc_rmsnorm_permute(_ptr(x), M, K, K, _ptr(g), None if pp is None else _ptr(pp),
                              float(eps), _ptr(y))
    return y


def arc_quantize(y: np.ndarray, outliers, s_t: float | None, fmt: str = "nvfp4"):
    """Primary + residual quantization of the prepared matrix y; NVFP4 or INT4
    (block 16, tensor scale s_t) or MXFP4 (block 32, s_t unused)."""
    y = _f32(y)
    M, K = y.shape
    o = np.ascontiguousarray(outliers, np.int32)
    S = o.size
    B = 32 if fmt == "mxfp4" else 16
    assert K % B == 0 and S % B == 0
    codes = np.empty((M, (K + S) // 2), np.uint8)
    scales = np.empty((M, (K + S) // B), np.uint8)
    if fmt == "nvfp4":
        lib().orc_arc_quantize(_ptr(y), M, K, S, _ptr(o) if S else None, float(s_t), _ptr(codes),
                               _ptr(scales))
    elif fmt == "mxfp4":
        lib().orc_arc_quantize_mxfp4(_ptr(y), M, K, S, _ptr(o) if S else None, _ptr(codes),
                                     _ptr(scales))
    elif fmt == "int4":
        lib().orc_arc_quantize_int4(_ptr(y), M, K, S, _ptr(o) if S else None, float(s_t),
                                    _ptr(codes), _ptr(scales))
    else:
        raise ValueError(fmt)
    return codes, scales


# --------------------------------------------------------------------------- workloads

def quantize_nvfp4(x_bits: np.ndarray, s_t: float | None = None):
    """NVFP4 of a bf16 matrix.  ``s_t=None``: dynamic, s_t = amax/2688 of x."""
    y = bf16_to_f32(x_bits)
    if s_t is None:
        s_t = tensor_scale(amax(y))
    codes, scales = nvfp4_quantize(y, s_t)
    return codes, scales, np.float32(s_t)


def quantize_mxfp4(x_bits: np.ndarray):
    return mxfp4_quantize(bf16_to_f32(x_bits))


def hadamard_quantize(x_bits: np.ndarray, n: int, fmt: str = "nvfp4", s_t: float | None = None,
                      signs=None):
    """Block-Hadamard (size n, normalised; with `signs` the random-sign H D)
    then NVFP4 / MXFP4 / dual quantization.

    Returns (codes, scales, s_t_or_gscales, y) with y the rotated fp32 matrix."""
    y = hadamard(bf16_to_f32(x_bits), n, signs)
    if fmt == "nvfp4":
        if s_t is None:
            s_t = tensor_scale(amax(y))
        c, s = nvfp4_quantize(y, s_t)
        return c, s, np.float32(s_t), y
    if fmt == "mxfp4":
        c, s = mxfp4_quantize(y)
        return c, s, None, y
    if fmt == "dual":
        c, s, g = dual_quantize(y)
        return c, s, g, y
    raise ValueError(fmt)


def arc_prepare(x_bits, gamma_bits, perm, eps: float = 1e-6) -> np.ndarray:
    """Reordered + RMS-normalised fp32 matrix y[M, K] of the ARCQuant path."""
    return rmsnorm_permute(bf16_to_f32(x_bits), bf16_to_f32(gamma_bits), perm, eps)


def arc(x_bits, gamma_bits, perm, outliers, eps: float = 1e-6, s_t: float | None = None,
        fmt: str = "nvfp4"):
    """ARCQuant path: reorder + RMSNorm, primary + residual quantization.
    Returns (codes, scales, s_t (NVFP4, INT4) or None (MXFP4), y)."""
    y = arc_prepare(x_bits, gamma_bits, perm, eps)
    if fmt == "mxfp4":
        c, s = arc_quantize(y, outliers, None, "mxfp4")
        return c, s, None, y
    if s_t is None:
        s_t = int4_tensor_scale(amax(y)) if fmt == "int4" else tensor_scale(amax(y))
    c, s = arc_quantize(y, outliers, s_t, fmt)
    return c, s, np.float32(s_t), y


def arc_alignment(y, outliers, s_t, codes, scales, fmt: str = "nvfp4"):
    """Block alignment factors of the ARCQuant two-stage path (ARCQuant summary,
    "Analyse de la Borne d'Erreur Theorique": the alignment overhead of the two
    stages, about 1.266, against under 2 for MXFP8).  Reading: a block's grid is
    aligned to its content when the decoded block scale d equals amax / 6 (the
    block maximum on the top E2M1 value); the factor phi = d / (amax / 6) is
    how far the stored scale moved it (INT4: amax / 7, its largest integer).
    One E4M3 step is 2^-3 of the value, and
    (1 + 2^-3)^2 = 1.265625 is the page's figure for two stages; round to
    nearest keeps phi within 1 +- 2^-4 while the scale is a normal E4M3 number
    (MXFP4's power-of-two scale, chosen from the exponent of amax: phi in
    (0.75, 1.5]).

    ``y`` [M, K] is the prepared fp32 matrix and ``codes`` / ``scales`` its
    oracle quantization (``arc``).  The residuals are recomputed the way the
    quantizer forms them (fp32).  Returns ``(phi_primary [M, K/B],
    phi_residual [M, S/B], normal_primary, normal_residual)``: the factors
    (NaN for all-zero blocks) and masks of the blocks whose scale byte is a
    normal E4M3 value (NVFP4; all True for MXFP4)."""
    y = _f32(y)
    M, K = y.shape
    o = np.asarray(outliers, np.int64)
    S = o.size
    B = 32 if fmt == "mxfp4" else 16
    top = 7.0 if fmt == "int4" else 6.0  # the largest grid value
    u = unpack_codes(np.asarray(codes))
    cv = int4_decode(u) if fmt == "int4" else e2m1_decode(u)  # [M, K + S] grid values
    sb = np.asarray(scales, np.uint8).reshape(M, (K + S) // B)
    if fmt in ("nvfp4", "int4"):
        d = (e4m3_decode(sb).astype(np.float32) * np.float32(s_t)).astype(np.float32)
        unit = e4m3_decode(sb).astype(np.float32)
        normal = (sb & 0x78) != 0  # exponent field non-zero
    else:
        d = e8m0_decode(sb).astype(np.float32)
        unit = d
        normal = np.ones(sb.shape, bool)
    # residual of outlier position p: y[p] - dq(p), dq as the dequantizer forms it
    cp = cv[:, o].astype(np.float32)
    up = unit[:, o // B]
    dq = (cp * up).astype(np.float32)
    if fmt in ("nvfp4", "int4"):
        dq = (dq * np.float32(s_t)).astype(np.float32)
    res = (y[:, o] - dq).astype(np.float32)

    def phi(vals, dd):
        am = np.abs(vals.astype(np.float64)).reshape(M, -1, B).max(axis=2)
        with np.errstate(divide="ignore", invalid="ignore"):
            return np.where(am > 0, dd.astype(np.float64) / (am / top), np.nan)

    nb = K // B
    return phi(y, d[:, :nb]), phi(res, d[:, nb:]), normal[:, :nb], normal[:, nb:]


def dequantize(fmt: str, codes, scales, scale=None, inv_had: int = 0, signs=None) -> np.ndarray:
    """Dequantize to fp32 (then optionally inverse block Hadamard, and with a
    sign pattern the inverse D H of the random-sign rotation); returns fp32."""
    if fmt == "nvfp4":
        y = nvfp4_dequantize(codes, scales, float(scale))
    elif fmt == "mxfp4":
        y = mxfp4_dequantize(codes, scales)
    elif fmt == "dual":
        y = dual_dequantize(codes, scales, scale)
    elif fmt == "int4":
        y = int4_dequantize(codes, scales, float(scale))
    else:
        raise ValueError(fmt)
    if inv_had:
        y = hadamard(y, inv_had)  # the normalised Sylvester matrix is its own inverse
        if signs is not None:
            y = y * sign_vector(signs, inv_had, y.shape[1])[None, :]  # D = D^-1
    return y


def dequantize_bf16(fmt: str, codes, scales, scale=None, inv_had: int = 0, signs=None) -> np.ndarray:
    return f32_to_bf16(dequantize(fmt, codes, scales, scale, inv_had, signs))


# --------------------------------------------------------------------------- consumer GEMM

def nvfp4_block_values(codes, scales) -> np.ndarray:
    """E2M1 value * E4M3 block-scale value of every element (float64, exact)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    K = codes.shape[1] * 2
    v = e2m1_decode(unpack_codes(codes)).astype(np.float64)
    return v * np.repeat(e4m3_decode(scales).astype(np.float64), 16, axis=1)[:, :K]


def nvfp4_gemm(a_codes, a_scales, s_a, b_codes, b_scales, s_b):
    """The block-scaled NVFP4 GEMM a consumer runs on the quantized operands
    (ARCQuant summary, Methodologie items 3-4: one GEMM over the augmented K):
    D = s_a s_b (A B^T) with A, B the E2M1 * E4M3 values, in float64 (each
    product is exact; the float64 sum errs by at most 2^-53 of the sum of the
    magnitudes).  Returns (D, the same product of the magnitudes |A| |B|^T)."""
    A = nvfp4_block_values(a_codes, a_scales)
    B = nvfp4_block_values(b_codes, b_scales)
    s = float(s_a) * float(s_b)
    return (A @ B.T) * s, (np.abs(A) @ np.abs(B).T) * s
