"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export exactly the functions `include/fp4q.h`
declares, and reject bad arguments on the host with the documented status
before it touches the device.
"""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")


@pytest.fixture(scope="module")
def fq():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as m
    return m


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_five_entry_points():
    names = declared_functions()
    for n in ["fp4q_quantize_nvfp4", "fp4q_quantize_mxfp4", "fp4q_hadamard_quantize",
              "fp4q_arc_quantize", "fp4q_dequantize"]:
        assert n in names


def test_library_exports_exactly_the_declared_symbols(fq):
    out = subprocess.run(["nm", "-D", "--defined-only", fq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines()
                       if ln.split() and ln.split()[-1].startswith("fp4q_")})
    assert exported == declared_functions()
    lib = C.CDLL(fq.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n)
    assert sorted(fq.EXPORTED) == declared_functions()


def test_status_strings(fq):
    for s in range(6):
        assert fq.status_string(s).startswith("FP4Q")
    assert "unknown" in fq.status_string(99)


def test_workspace_and_scale_sizes(fq):
    assert fq.fp4q_workspace_bytes(1, 64) == 16384 == fq.FP4Q_WORKSPACE_BYTES
    assert fq.fp4q_scales_bytes(256, 64, 0) == 256 * 64
    assert fq.fp4q_scales_bytes(130, 9, 1) == 256 * 12
    assert fq.fp4q_scales_bytes(128, 272, 1) == 128 * 272
    assert fq.fp4q_scales_bytes(-1, 4, 0) == -1
    assert fq.fp4q_scales_bytes(4, 4, 7) == -1


# Fake, aligned, never dereferenced addresses: every call below must fail in
# host validation before any CUDA call.
X, CODES, SCALES, SF, WS = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000


def test_quantize_nvfp4_validation(fq):
    L = fq.lib()
    q = lambda *a: L.fp4q_quantize_nvfp4(*a)
    assert q(X, -1, 64, 64, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 32, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 72, 72, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 32, 32, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_UNSUPPORTED
    assert q(X + 8, 4, 64, 64, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_ALIGNMENT
    assert q(X, 4, 64, 68, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_ALIGNMENT
    assert q(None, 4, 64, 64, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, None, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, CODES + 4, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_ALIGNMENT
    assert q(X, 4, 64, 64, CODES, SCALES, None, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, CODES, SCALES, SF, 0, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, CODES, SCALES, SF, 0, 0, WS, 100, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, CODES, SCALES, SF, 7, 0, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 4, 64, 64, CODES, SCALES, SF, 0, 5, WS, 16384, None) == fq.FP4Q_ERR_INVALID_ARG
    assert q(X, 1 << 31, 64, 64, CODES, SCALES, SF, 0, 0, WS, 16384, None) == fq.FP4Q_ERR_UNSUPPORTED
    # M == 0 is a no-op
    assert q(X, 0, 64, 64, None, None, None, 0, 0, None, 0, None) == fq.FP4Q_OK


def test_quantize_mxfp4_and_hadamard_validation(fq):
    L = fq.lib()
    assert L.fp4q_quantize_mxfp4(X, 4, 80, 80, CODES, SCALES, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert L.fp4q_quantize_mxfp4(X, 0, 96, 96, None, None, 0, None) == fq.FP4Q_OK
    h = L.fp4q_hadamard_quantize
    assert h(X, 4, 128, 128, 48, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 128, 128, 1024, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 192, 192, 128, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 192, 192, 64, 2, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 128, 128, 64, 9, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 128, 128, 64, 2, CODES, SCALES, None, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    # INT4 is an ARC / dequantize format only
    assert h(X, 4, 128, 128, 64, fq.FP4Q_INT4, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG


def test_arc_validation(fq):
    L = fq.lib()
    a = L.fp4q_arc_quantize
    P, O, G = 0x60000, 0x70000, 0x80000
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 24, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 144, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 32768, 32768, G, 1e-6, P, O, 16, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_UNSUPPORTED
    assert a(X, 4, 128, 128, G, -1.0, P, O, 16, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, None, 1e-6, P, O, 16, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, None, 16, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, 0, CODES, SCALES, SF, 0, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G + 1, 1e-6, P, O, 16, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_ALIGNMENT
    # format: NVFP4 or MXFP4 only; MXFP4 needs S and K multiples of 32, no tensor scale
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, 2, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, 1, CODES, SCALES, None, 0, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 144, 144, G, 1e-6, P, O, 32, 1, CODES, SCALES, None, 0, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 0, 128, 128, G, 1e-6, P, O, 32, 1, CODES, SCALES, None, 0, 0, None, 0, None) == fq.FP4Q_OK
    # INT4: blocks of 16 under a tensor scale, like NVFP4; unknown formats are rejected
    i4 = fq.FP4Q_INT4
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, i4, CODES, SCALES, None, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 24, i4, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, i4, CODES, SCALES, SF, 0, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 4, 128, 128, G, 1e-6, P, O, 16, 4, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert a(X, 0, 128, 128, G, 1e-6, P, O, 16, i4, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_OK


def test_dequantize_validation(fq):
    L = fq.lib()
    d = L.fp4q_dequantize
    Y = 0x90000
    assert d(0, CODES, SCALES, SF, 4, 72, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(1, CODES, SCALES, None, 4, 80, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(4, CODES, SCALES, SF, 4, 128, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    # INT4: a tensor scale is required, and there is no rotated INT4 path
    assert d(fq.FP4Q_INT4, CODES, SCALES, None, 4, 128, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(fq.FP4Q_INT4, CODES, SCALES, SF, 4, 128, 0, 16, Y, None) == fq.FP4Q_ERR_UNSUPPORTED
    assert d(fq.FP4Q_INT4, CODES, SCALES, SF, 4, 72, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(fq.FP4Q_INT4, CODES, SCALES, SF, 0, 128, 0, 0, Y, None) == fq.FP4Q_OK
    assert d(0, CODES, SCALES, SF, 4, 128, 0, 48, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(0, CODES, SCALES, None, 4, 128, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(0, CODES + 8, SCALES, SF, 4, 128, 0, 0, Y, None) == fq.FP4Q_ERR_ALIGNMENT
    assert d(2, CODES, SCALES, SF, 4, 192, 0, 0, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(0, CODES, SCALES, SF, 0, 128, 0, 0, Y, None) == fq.FP4Q_OK


def test_selftest_validation(fq):
    L = fq.lib()
    assert L.fp4q_selftest_div(X, X, -1, X, X, None) == fq.FP4Q_ERR_INVALID_ARG
    assert L.fp4q_selftest_div(None, X, 0, X, X, None) == fq.FP4Q_OK


def test_signed_rotation_validation(fq):
    """The random-sign variants: no pattern, no rotation or a register-path K
    (not a multiple of 128) are rejected before any launch."""
    import ctypes as C
    L = fq.lib()
    words = (C.c_uint32 * 4)(1, 2, 3, 4)
    h = L.fp4q_hadamard_quantize_signed
    assert h(X, 4, 256, 256, 128, None, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 256, 256, 0, words, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
    assert h(X, 4, 1040, 1040, 16, words, 0, CODES, SCALES, SF, 1, 0, None, 0, None) == fq.FP4Q_ERR_UNSUPPORTED
    d = L.fp4q_dequantize_signed
    Y = 0x90000
    assert d(0, CODES, SCALES, SF, 4, 256, 0, 128, None, Y, None) == fq.FP4Q_ERR_INVALID_ARG
    assert d(0, CODES, SCALES, SF, 4, 256, 0, 0, words, Y, None) == fq.FP4Q_ERR_INVALID_ARG
