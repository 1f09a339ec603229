"""Python binding of ``libfp4q.so``, the sm_100a micro-block FP4 quantizer.

The entry points below carry the C names of ``include/fp4q.h`` and only
marshal arguments: torch tensors become device pointers, the current torch CUDA
stream becomes the ``stream`` argument, and a non-zero status raises
``Fp4qError``.  Every step of the computation runs in the library's kernels;
there is no CPU or PyTorch fallback.  The library is loaded on first use; if it
has not been built, that first call raises ImportError (build it with
``python -m fp4_micro_block_b200.build``).

Helpers at the bottom (``quantize_nvfp4`` ...) only allocate the output tensors
with torch and call the entry points.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FP4Q_LIBRARY selects another build of the library (a variant made with
# `python -m fp4_micro_block_b200.build --define ... --out ...`).
LIB_PATH = os.environ.get("FP4Q_LIBRARY") or os.path.join(_HERE, "libfp4q.so")

# enum values of include/fp4q.h
FP4Q_OK, FP4Q_ERR_INVALID_ARG, FP4Q_ERR_UNSUPPORTED, FP4Q_ERR_ALIGNMENT, FP4Q_ERR_CUDA, \
    FP4Q_ERR_DEVICE = range(6)
FP4Q_NVFP4, FP4Q_MXFP4, FP4Q_NVFP4_DUAL, FP4Q_INT4 = 0, 1, 2, 3
FP4Q_SCALES_LINEAR, FP4Q_SCALES_SWIZZLED = 0, 1
FP4Q_TSCALE_DYNAMIC, FP4Q_TSCALE_STATIC = 0, 1
FP4Q_WORKSPACE_BYTES = 16384

EXPORTED = [
    "fp4q_quantize_nvfp4", "fp4q_quantize_nvfp4_noalloc", "fp4q_quantize_mxfp4", "fp4q_hadamard_quantize", "fp4q_arc_quantize",
    "fp4q_dequantize", "fp4q_workspace_bytes", "fp4q_scales_bytes", "fp4q_status_string",
    "fp4q_device_error", "fp4q_selftest_div", "fp4q_gemm_nvfp4", "fp4q_hadamard_quantize_signed",
    "fp4q_dequantize_signed",
]


class Fp4qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fp4_micro_block_b200.build`")
    return declare(C.CDLL(LIB_PATH))


def declare(L: C.CDLL) -> C.CDLL:
    """Sets the argument and result types of the C entry points on a loaded library."""
    p, i64, f32, i32, sz = C.c_void_p, C.c_int64, C.c_float, C.c_int, C.c_size_t
    sigs = {
        "fp4q_quantize_nvfp4": (i32, [p, i64, i64, i64, p, p, p, i32, i32, p, sz, p]),
        "fp4q_quantize_nvfp4_noalloc": (i32, [p, i64, i64, i64, p, p, p, i32, p]),
        "fp4q_quantize_mxfp4": (i32, [p, i64, i64, i64, p, p, i32, p]),
        "fp4q_hadamard_quantize": (i32, [p, i64, i64, i64, i32, i32, p, p, p, i32, i32, p, sz, p]),
        "fp4q_arc_quantize": (i32, [p, i64, i64, i64, p, f32, p, p, i64, i32, p, p, p, i32, i32, p, sz, p]),
        "fp4q_dequantize": (i32, [i32, p, p, p, i64, i64, i32, i32, p, p]),
        "fp4q_workspace_bytes": (sz, [i64, i64]),
        "fp4q_scales_bytes": (i64, [i64, i64, i32]),
        "fp4q_status_string": (C.c_char_p, [i32]),
        "fp4q_device_error": (i32, []),
        "fp4q_selftest_div": (i32, [p, p, i64, p, p, p]),
        "fp4q_gemm_nvfp4": (i32, [p, p, p, p, p, p, i64, i64, i64, p, i32, p]),
        "fp4q_hadamard_quantize_signed": (i32, [p, i64, i64, i64, i32, p, i32, p, p, p, i32, i32, p, sz, p]),
        "fp4q_dequantize_signed": (i32, [i32, p, p, p, i64, i64, i32, i32, p, p, p]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


class _Lazy:
    """Loads libfp4q.so on first attribute access."""

    _cdll = None

    def __getattr__(self, name):
        if _Lazy._cdll is None:
            _Lazy._cdll = _load()
        return getattr(_Lazy._cdll, name)


_lib = _Lazy()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.fp4q_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("fp4q entry points take CUDA tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> int:
    if status != FP4Q_OK:
        raise Fp4qError(status, where)
    return status


def _ld(x: torch.Tensor) -> int:
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major view (unit column stride)")
    return x.stride(0)


# ----------------------------------------------------------------------------- C entry points

def fp4q_workspace_bytes(M: int = 0, K: int = 0) -> int:
    return int(_lib.fp4q_workspace_bytes(M, K))


def fp4q_scales_bytes(M: int, ncols: int, layout: int = FP4Q_SCALES_LINEAR) -> int:
    return int(_lib.fp4q_scales_bytes(M, ncols, layout))


def fp4q_quantize_nvfp4(x, codes, scales, tensor_scale, mode=FP4Q_TSCALE_DYNAMIC,
                        layout=FP4Q_SCALES_LINEAR, workspace=None, stream=None):
    M, K = x.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.fp4q_quantize_nvfp4(_ptr(x), M, K, _ld(x), _ptr(codes), _ptr(scales),
                                           _ptr(tensor_scale), mode, layout, _ptr(workspace),
                                           ws_bytes, _stream(stream)), "fp4q_quantize_nvfp4")


def fp4q_quantize_nvfp4_noalloc(x, codes, scales, tensor_scale, layout=FP4Q_SCALES_LINEAR,
                                stream=None):
    M, K = x.shape
    return _check(_lib.fp4q_quantize_nvfp4_noalloc(_ptr(x), M, K, _ld(x), _ptr(codes), _ptr(scales),
                                                   _ptr(tensor_scale), layout, _stream(stream)),
                  "fp4q_quantize_nvfp4_noalloc")


def fp4q_quantize_mxfp4(x, codes, scales, layout=FP4Q_SCALES_LINEAR, stream=None):
    M, K = x.shape
    return _check(_lib.fp4q_quantize_mxfp4(_ptr(x), M, K, _ld(x), _ptr(codes), _ptr(scales),
                                           layout, _stream(stream)), "fp4q_quantize_mxfp4")


def fp4q_hadamard_quantize(x, had_size, fmt, codes, scales, scale_fp32,
                           mode=FP4Q_TSCALE_DYNAMIC, layout=FP4Q_SCALES_LINEAR,
                           workspace=None, stream=None):
    M, K = x.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.fp4q_hadamard_quantize(_ptr(x), M, K, _ld(x), int(had_size), int(fmt),
                                              _ptr(codes), _ptr(scales), _ptr(scale_fp32), mode,
                                              layout, _ptr(workspace), ws_bytes, _stream(stream)),
                  "fp4q_hadamard_quantize")


def fp4q_arc_quantize(x, gamma, eps, perm, outliers, fmt, codes, scales, tensor_scale,
                      mode=FP4Q_TSCALE_DYNAMIC, layout=FP4Q_SCALES_LINEAR, workspace=None,
                      stream=None):
    M, K = x.shape
    S = 0 if outliers is None else outliers.numel()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.fp4q_arc_quantize(_ptr(x), M, K, _ld(x), _ptr(gamma), float(eps), _ptr(perm),
                                         _ptr(outliers), S, int(fmt), _ptr(codes), _ptr(scales),
                                         _ptr(tensor_scale), mode, layout, _ptr(workspace),
                                         ws_bytes, _stream(stream)), "fp4q_arc_quantize")


def fp4q_dequantize(fmt, codes, scales, scale_fp32, M, K, y, layout=FP4Q_SCALES_LINEAR,
                    inv_had_size=0, stream=None):
    return _check(_lib.fp4q_dequantize(int(fmt), _ptr(codes), _ptr(scales), _ptr(scale_fp32), M, K,
                                       layout, int(inv_had_size), _ptr(y), _stream(stream)),
                  "fp4q_dequantize")


def fp4q_gemm_nvfp4(a_codes, a_scales, a_scale, b_codes, b_scales, b_scale, K, d, stream=None):
    """d [M, N] (float32 or bfloat16) = a_scale b_scale (A B^T) of two NVFP4
    tensors in the quantizers' output form (SWIZZLED scale buffers)."""
    M, N = d.shape
    if d.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("d must be float32 or bfloat16")
    return _check(_lib.fp4q_gemm_nvfp4(_ptr(a_codes), _ptr(a_scales), _ptr(a_scale), _ptr(b_codes),
                                       _ptr(b_scales), _ptr(b_scale), M, N, K, _ptr(d),
                                       int(d.dtype == torch.bfloat16), _stream(stream)),
                  "fp4q_gemm_nvfp4")


def _host_words(signs):
    """A host uint32 pattern (numpy array or sequence) as a ctypes pointer, kept alive by the caller."""
    import numpy as np
    arr = np.ascontiguousarray(np.asarray(signs, dtype=np.uint32))
    return arr, arr.ctypes.data


def fp4q_hadamard_quantize_signed(x, had_size, signs, fmt, codes, scales, scale_fp32,
                                  mode=FP4Q_TSCALE_DYNAMIC, layout=FP4Q_SCALES_LINEAR,
                                  workspace=None, stream=None):
    M, K = x.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    keep, sp = _host_words(signs)
    return _check(_lib.fp4q_hadamard_quantize_signed(_ptr(x), M, K, _ld(x), int(had_size), sp, int(fmt),
                                                     _ptr(codes), _ptr(scales), _ptr(scale_fp32), mode,
                                                     layout, _ptr(workspace), ws_bytes, _stream(stream)),
                  "fp4q_hadamard_quantize_signed")


def fp4q_dequantize_signed(fmt, codes, scales, scale_fp32, M, K, y, signs, layout=FP4Q_SCALES_LINEAR,
                           inv_had_size=0, stream=None):
    keep, sp = _host_words(signs)
    return _check(_lib.fp4q_dequantize_signed(int(fmt), _ptr(codes), _ptr(scales), _ptr(scale_fp32), M, K,
                                              layout, int(inv_had_size), sp, _ptr(y), _stream(stream)),
                  "fp4q_dequantize_signed")


def fp4q_device_error() -> int:
    return int(_lib.fp4q_device_error())


def fp4q_selftest_div(x, d, q_fast, q_ieee, stream=None):
    return _check(_lib.fp4q_selftest_div(_ptr(x), _ptr(d), x.numel(), _ptr(q_fast), _ptr(q_ieee),
                                         _stream(stream)), "fp4q_selftest_div")


# ----------------------------------------------------------------------------- allocating helpers

def _block(fmt: int) -> int:
    return 32 if fmt == FP4Q_MXFP4 else 16


def alloc_outputs(M: int, K: int, fmt: int, layout: int = FP4Q_SCALES_LINEAR, device="cuda",
                  ncols: int | None = None):
    """codes [M, K/2] u8, scales (linear [M, ncols] or the padded tiled buffer),
    and the fp32 scale(s): 1 float (NVFP4, INT4), [M, K/128] (dual) or None (MXFP4)."""
    ncols = K // _block(fmt) if ncols is None else ncols
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
    if layout == FP4Q_SCALES_LINEAR:
        scales = torch.empty((M, ncols), dtype=torch.uint8, device=device)
    else:
        scales = torch.empty(fp4q_scales_bytes(M, ncols, layout), dtype=torch.uint8, device=device)
    if fmt in (FP4Q_NVFP4, FP4Q_INT4):
        sf = torch.zeros(1, dtype=torch.float32, device=device)
    elif fmt == FP4Q_NVFP4_DUAL:
        sf = torch.empty((M, K // 128), dtype=torch.float32, device=device)
    else:
        sf = None
    return codes, scales, sf


def workspace(device="cuda") -> torch.Tensor:
    return torch.empty(FP4Q_WORKSPACE_BYTES, dtype=torch.uint8, device=device)


def quantize_nvfp4(x, tensor_scale=None, layout=FP4Q_SCALES_LINEAR, ws=None):
    """NVFP4 of bf16 x; dynamic tensor scale unless `tensor_scale` (1-float tensor) is given."""
    M, K = x.shape
    codes, scales, sf = alloc_outputs(M, K, FP4Q_NVFP4, layout, x.device)
    mode = FP4Q_TSCALE_DYNAMIC
    if tensor_scale is not None:
        sf.copy_(tensor_scale.reshape(1))
        mode = FP4Q_TSCALE_STATIC
    ws = workspace(x.device) if (ws is None and mode == FP4Q_TSCALE_DYNAMIC) else ws
    fp4q_quantize_nvfp4(x, codes, scales, sf, mode, layout, ws)
    return codes, scales, sf


def quantize_mxfp4(x, layout=FP4Q_SCALES_LINEAR):
    M, K = x.shape
    codes, scales, _ = alloc_outputs(M, K, FP4Q_MXFP4, layout, x.device)
    fp4q_quantize_mxfp4(x, codes, scales, layout)
    return codes, scales


def hadamard_quantize(x, had_size, fmt=FP4Q_NVFP4, tensor_scale=None, layout=FP4Q_SCALES_LINEAR,
                      ws=None, signs=None):
    """Block Hadamard (with `signs`: the random-sign rotation) + quantization."""
    M, K = x.shape
    codes, scales, sf = alloc_outputs(M, K, fmt, layout, x.device)
    mode = FP4Q_TSCALE_DYNAMIC
    if fmt == FP4Q_NVFP4 and tensor_scale is not None:
        sf.copy_(tensor_scale.reshape(1))
        mode = FP4Q_TSCALE_STATIC
    if fmt == FP4Q_NVFP4 and mode == FP4Q_TSCALE_DYNAMIC and ws is None:
        ws = workspace(x.device)
    if signs is None:
        fp4q_hadamard_quantize(x, had_size, fmt, codes, scales, sf, mode, layout, ws)
    else:
        fp4q_hadamard_quantize_signed(x, had_size, signs, fmt, codes, scales, sf, mode, layout, ws)
    return codes, scales, sf


def arc_quantize(x, gamma, perm, outliers, eps=1e-6, tensor_scale=None,
                 layout=FP4Q_SCALES_LINEAR, ws=None, fmt=FP4Q_NVFP4):
    """ARCQuant path; returns (codes, scales, tensor scale (NVFP4, INT4) or None (MXFP4))."""
    M, K = x.shape
    S = 0 if outliers is None else outliers.numel()
    codes, scales, sf = alloc_outputs(M, K + S, fmt, layout, x.device)
    mode = FP4Q_TSCALE_DYNAMIC
    if fmt in (FP4Q_NVFP4, FP4Q_INT4):
        if tensor_scale is not None:
            sf.copy_(tensor_scale.reshape(1))
            mode = FP4Q_TSCALE_STATIC
        ws = workspace(x.device) if (ws is None and mode == FP4Q_TSCALE_DYNAMIC) else ws
    fp4q_arc_quantize(x, gamma, eps, perm, outliers, fmt, codes, scales, sf, mode, layout, ws)
    return codes, scales, sf


def dequantize(fmt, codes, scales, scale_fp32, K, layout=FP4Q_SCALES_LINEAR, inv_had_size=0, signs=None):
    M = codes.shape[0]
    y = torch.empty((M, K), dtype=torch.bfloat16, device=codes.device)
    if signs is None:
        fp4q_dequantize(fmt, codes, scales, scale_fp32, M, K, y, layout, inv_had_size)
    else:
        fp4q_dequantize_signed(fmt, codes, scales, scale_fp32, M, K, y, signs, layout, inv_had_size)
    return y


def gemm_nvfp4(a_codes, a_scales, a_scale, b_codes, b_scales, b_scale, K, out_dtype=torch.float32):
    """Allocates D [M, N] and calls fp4q_gemm_nvfp4."""
    d = torch.empty((a_codes.shape[0], b_codes.shape[0]), dtype=out_dtype, device=a_codes.device)
    fp4q_gemm_nvfp4(a_codes, a_scales, a_scale, b_codes, b_scales, b_scale, K, d)
    return d
