"""Out-of-bounds writes: every output of every entry point sits inside a larger
device buffer whose guard bytes before and after it hold a pattern; after each
call on a ragged shape the guards must be unchanged.

The shapes leave partial tiles in both directions: M in {1, 37, 130, 131} (one
row, a partial 64/128-row tile, one or three rows past a tile) and K a multiple
of 16, 32 or 64 that is not a multiple of 128 (the register paths' ragged last
column strip), plus multiples of 128 for the tensor-core rotations and the dual
format.  The outputs are also compared byte for byte with an ordinary
(unguarded) call, so a guard that stayed intact because nothing was written
does not pass.
"""
import numpy as np
import pytest
import torch

import workloads
from parity import bits_to_torch_cuda

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side; keeps every view 16-byte aligned
PAT = 0xA5
MS = [1, 37, 130, 131]


@pytest.fixture(scope="module")
def fq():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as m
    assert m.fp4q_device_error() == 0
    yield m
    assert m.fp4q_device_error() == 0


class Guarded:
    """A tensor of `shape`/`dtype` placed GUARD bytes into a pattern-filled buffer."""

    def __init__(self, shape, dtype, fill=None):
        nel = int(np.prod(shape)) if len(shape) else 1
        self.nbytes = nel * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((2 * GUARD + (self.nbytes + 15) // 16 * 16,), PAT, dtype=torch.uint8,
                              device="cuda")
        self.t = self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def check(self, name):
        b = self.buf.cpu().numpy()
        lo = np.flatnonzero(b[:GUARD] != PAT)
        hi = np.flatnonzero(b[GUARD + self.nbytes:] != PAT)
        assert lo.size == 0, f"{name}: {lo.size} guard bytes before the buffer changed (first at -{GUARD - lo[0]})"
        assert hi.size == 0, f"{name}: {hi.size} guard bytes after the buffer changed (first at +{hi[0]})"


def _outs(fq, M, ncols_codes, ncols_scales, layout, sf_shape=None, sf_fill=None):
    codes = Guarded((M, ncols_codes), torch.uint8)
    nsb = fq.fp4q_scales_bytes(M, ncols_scales, layout)
    scales = Guarded((nsb,), torch.uint8)
    sf = None if sf_shape is None else Guarded(sf_shape, torch.float32, sf_fill)
    return codes, scales, sf


def _check_all(name, *gs):
    for i, g in enumerate(gs):
        if g is not None:
            g.check(f"{name}[{i}]")


def _same(name, a, b):
    assert torch.equal(a.reshape(-1).view(torch.uint8) if a.dtype != torch.uint8 else a.reshape(-1),
                       b.reshape(-1).view(torch.uint8) if b.dtype != torch.uint8 else b.reshape(-1)), name


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("K", [1040, 1056, 1088])
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_canary_nvfp4(fq, M, K, layout, mode):
    x = bits_to_torch_cuda(workloads.nvfp4_outliers(M, K, seed=M + K))
    fill = torch.tensor([0.02], device="cuda")
    codes, scales, sf = _outs(fq, M, K // 2, K // 16, layout, (1,), fill)
    ws = Guarded((fq.FP4Q_WORKSPACE_BYTES,), torch.uint8)
    fq.fp4q_quantize_nvfp4(x, codes.t, scales.t, sf.t, mode, layout, ws.t if mode == 0 else None)
    torch.cuda.synchronize()
    _check_all(f"nvfp4 M{M} K{K}", codes, scales, sf, ws)
    c, s, f = fq.quantize_nvfp4(x, fill if mode == 1 else None, layout)
    torch.cuda.synchronize()
    _same("codes", codes.t, c)
    _same("scales", scales.t, s)
    _same("tensor scale", sf.t, f)


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("K", [1056, 1088])
@pytest.mark.parametrize("layout", [0, 1])
def test_canary_mxfp4(fq, M, K, layout):
    x = bits_to_torch_cuda(workloads.mxfp4_student_t(M, K, seed=M + K))
    codes, scales, _ = _outs(fq, M, K // 2, K // 32, layout)
    fq.fp4q_quantize_mxfp4(x, codes.t, scales.t, layout)
    torch.cuda.synchronize()
    _check_all(f"mxfp4 M{M} K{K}", codes, scales)
    c, s = fq.quantize_mxfp4(x, layout)
    torch.cuda.synchronize()
    _same("codes", codes.t, c)
    _same("scales", scales.t, s)


HAD_CASES = [  # (format name, n, K)
    ("nvfp4", 16, 1040), ("nvfp4", 32, 1056), ("nvfp4", 64, 1088), ("nvfp4", 128, 1152),
    ("nvfp4", 256, 1536), ("nvfp4", 512, 1536),
    ("mxfp4", 32, 1056), ("mxfp4", 64, 1088), ("mxfp4", 128, 1152), ("mxfp4", 512, 1536),
    ("dual", 0, 1152), ("dual", 128, 1152), ("dual", 256, 1536), ("dual", 512, 1536),
]


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("case", HAD_CASES, ids=lambda c: f"{c[0]}-n{c[1]}-K{c[2]}")
@pytest.mark.parametrize("layout", [0, 1])
def test_canary_hadamard_quantize(fq, M, case, layout):
    fmt_name, n, K = case
    fmt = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt_name]
    B = 32 if fmt_name == "mxfp4" else 16
    x = bits_to_torch_cuda(workloads.hadamard_channels(M, K, seed=M + K + n))
    sf_shape = (1,) if fmt_name == "nvfp4" else (M, K // 128) if fmt_name == "dual" else None
    codes, scales, sf = _outs(fq, M, K // 2, K // B, layout, sf_shape)
    ws = Guarded((fq.FP4Q_WORKSPACE_BYTES,), torch.uint8)
    fq.fp4q_hadamard_quantize(x, n, fmt, codes.t, scales.t, None if sf is None else sf.t,
                              fq.FP4Q_TSCALE_DYNAMIC, layout, ws.t)
    torch.cuda.synchronize()
    _check_all(f"had{n} {fmt_name} M{M} K{K}", codes, scales, sf, ws)
    c, s, f = fq.hadamard_quantize(x, n, fmt, None, layout)
    torch.cuda.synchronize()
    _same("codes", codes.t, c)
    _same("scales", scales.t, s)
    if sf is not None:
        _same("fp32 scales", sf.t, f)


ARC_CASES = [  # (format name, K, S)
    ("nvfp4", 1040, 16), ("nvfp4", 1056, 32), ("nvfp4", 1088, 64), ("nvfp4", 1152, 0),
    ("mxfp4", 1056, 32), ("mxfp4", 1088, 64), ("mxfp4", 1152, 0),
    ("int4", 1040, 16), ("int4", 1088, 64),
]


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("case", ARC_CASES, ids=lambda c: f"{c[0]}-K{c[1]}-S{c[2]}")
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_canary_arc(fq, M, case, layout, mode):
    fmt_name, K, S = case
    mx = fmt_name == "mxfp4"
    if mx and mode == 1:
        pytest.skip("MXFP4 has no tensor-scale mode")
    fmt = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "int4": fq.FP4Q_INT4}[fmt_name]
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=M + K, S=S, calib_rows=64)
    x = bits_to_torch_cuda(x_bits)
    g = bits_to_torch_cuda(gamma)
    p = torch.from_numpy(perm).cuda()
    o = torch.from_numpy(outl).cuda() if S else None
    fill = torch.tensor([0.01], device="cuda")
    B = 32 if mx else 16
    codes, scales, sf = _outs(fq, M, (K + S) // 2, (K + S) // B, layout, None if mx else (1,), fill)
    ws = Guarded((fq.FP4Q_WORKSPACE_BYTES,), torch.uint8)
    fq.fp4q_arc_quantize(x, g, 1e-6, p, o, fmt, codes.t, scales.t, None if mx else sf.t, mode, layout,
                         ws.t if mode == 0 and not mx else None)
    torch.cuda.synchronize()
    _check_all(f"arc {fmt_name} M{M} K{K} S{S}", codes, scales, sf, ws)
    c, s, f = fq.arc_quantize(x, g, p, o, 1e-6, fill if mode == 1 else None, layout, fmt=fmt)
    torch.cuda.synchronize()
    _same("codes", codes.t, c)
    _same("scales", scales.t, s)
    if not mx:
        _same("tensor scale", sf.t, f)


DQ_CASES = [  # (format name, n, K)
    ("nvfp4", 0, 1040), ("nvfp4", 16, 1040), ("nvfp4", 32, 1056), ("nvfp4", 64, 1088),
    ("nvfp4", 128, 1152), ("nvfp4", 512, 1536),
    ("mxfp4", 0, 1056), ("mxfp4", 32, 1056), ("mxfp4", 64, 1088), ("mxfp4", 256, 1536),
    ("dual", 0, 1152), ("dual", 16, 1152), ("dual", 128, 1152), ("dual", 512, 1536),
    ("int4", 0, 1040), ("int4", 0, 1088),
]


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("case", DQ_CASES, ids=lambda c: f"{c[0]}-n{c[1]}-K{c[2]}")
@pytest.mark.parametrize("layout", [0, 1])
def test_canary_dequantize(fq, M, case, layout):
    fmt_name, n, K = case
    fmt = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL,
           "int4": fq.FP4Q_INT4}[fmt_name]
    codes, scales, sc = workloads.random_payload(M, K, fmt_name, seed=M + K + n)
    if layout == 1:
        import oracle  # test infrastructure: lays the scale bytes out in the tiled layout
        scales = oracle.swizzle_scales(scales)
    sct = (None if sc is None else torch.tensor([sc], device="cuda") if fmt_name in ("nvfp4", "int4")
           else torch.from_numpy(sc).cuda())
    ct, st = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    y = Guarded((M, K), torch.bfloat16)
    fq.fp4q_dequantize(fmt, ct, st, sct, M, K, y.t, layout, n)
    torch.cuda.synchronize()
    y.check(f"dequant {fmt_name} n{n} M{M} K{K}")
    ref = fq.dequantize(fmt, ct, st, sct, K, layout, n)
    torch.cuda.synchronize()
    _same("y", y.t, ref)
