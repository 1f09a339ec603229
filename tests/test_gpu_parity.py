"""GPU parity: the sm_100a kernels, called through the C ABI, against the oracle.

Small cases run element by element (several tiles, ragged tails in M and K,
strided rows, both scale layouts, both tensor-scale modes); the five workload
shapes run at full size, compared on every element where the oracle is cheap
(quantize-only) and on sampled rows where it is not (Hadamard, RMSNorm).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import (add_counts, arc_counts, assert_bitexact, assert_roundtrip, assert_tolerant, bf16_torch_to_bits,
                    bits_to_torch_cuda, block_l2_identity, check_fractions, to_np,
                    tolerant_counts, unswizzle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as m
    assert m.fp4q_device_error() == 0
    yield m
    assert m.fp4q_device_error() == 0


def linear_scales(fq, scales_t, M, ncols, layout):
    s = to_np(scales_t)
    if layout == fq.FP4Q_SCALES_SWIZZLED:
        assert s.size == fq.fp4q_scales_bytes(M, ncols, layout)
        lin = unswizzle(s, M, ncols)
        # every byte outside the (r, c) positions is padding and must be zero
        assert_bitexact("tiled scale buffer", s, oracle.swizzle_scales(lin))
        return lin
    return s.reshape(M, ncols)


# ----------------------------------------------------------------------------- division

def test_division_is_correctly_rounded(fq):
    rng = np.random.default_rng(100)
    n = 1 << 20
    d = (oracle.e4m3_decode(rng.integers(1, 127, n).astype(np.uint8)).astype(np.float64) *
         np.exp(rng.uniform(-30, 30, n))).astype(np.float32)
    x = (rng.standard_normal(n) * d * rng.uniform(0, 7, n)).astype(np.float32)
    # quotients placed within a few ulps of every E2M1 decision point
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    k = n // 4
    q = mids[rng.integers(0, len(mids), k)]
    q = (q.view(np.int32) + rng.integers(-3, 4, k).astype(np.int32)).view(np.float32)
    x[:k] = (q.astype(np.float64) * d[:k]).astype(np.float32) * np.where(rng.random(k) < .5, -1, 1)
    # quotients next to midpoints between adjacent binary32 values (rounding ties
    # of the quotient itself): x = RN(m * d) for m = (2j + 1) * 2^-25 * 2^E in [2^(E-1), 2^E)
    m = ((2 * rng.integers(1 << 23, 1 << 24, k) + 1).astype(np.float64) * 2.0 ** -25 *
         np.exp2(rng.integers(-4, 3, k)))
    x[k + 2:2 * k + 2] = (m * d[k + 2:2 * k + 2].astype(np.float64)).astype(np.float32)
    x[k] = -0.0
    x[k + 1] = 0.0
    xt, dt = torch.from_numpy(x).cuda(), torch.from_numpy(d).cuda()
    qf, qi = torch.empty_like(xt), torch.empty_like(xt)
    fq.fp4q_selftest_div(xt, dt, qf, qi)
    torch.cuda.synchronize()
    assert_bitexact("markstein vs IEEE", to_np(qf), to_np(qi))
    # and the IEEE quotient is the host's binary32 quotient
    assert_bitexact("IEEE vs host", to_np(qi), x / d)


# ----------------------------------------------------------------------------- formats

def test_mxfp4_format_conformance(fq):
    """Blocks whose amax is exactly 4 * 2^E, elements at and around every E2M1
    decision point, negative values that round to zero, signed zeros."""
    pts = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7, 8], np.float64)
    rng = np.random.default_rng(101)
    vals = []
    for p in pts:
        for u in (-2, -1, 0, 1, 2):
            v = np.float32(p)
            if p > 0:
                v = (np.array([p], np.float32).view(np.int32) + u).view(np.float32)[0]
            vals += [v, -v]
    vals = np.array(vals, np.float32)
    M, K = 64, 256
    y = np.empty((M, K), np.float32)
    for r in range(M):
        y[r] = rng.choice(vals, K)
        y[r, ::32] = 4.0  # amax = 4 -> E = 0 for every block... and 2^E scaling below
    y *= np.exp2(rng.integers(-20, 20, (M, 1))).astype(np.float32)
    y[0, 1] = -0.0
    x_bits = oracle.f32_to_bf16(y)
    y = oracle.bf16_to_f32(x_bits)
    codes_o, scales_o = oracle.mxfp4_quantize(y)
    x = bits_to_torch_cuda(x_bits)
    codes, scales = fq.quantize_mxfp4(x)
    torch.cuda.synchronize()
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", to_np(scales), scales_o)


# ----------------------------------------------------------------------------- NVFP4

NV_SHAPES = [(256, 1024), (37, 1040), (16, 64), (1, 512), (130, 1536), (300, 4096)]


@pytest.mark.parametrize("shape", NV_SHAPES)
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("mode", ["dynamic", "static"])
def test_nvfp4_bitexact(fq, shape, layout, mode):
    M, K = shape
    x_bits = workloads.nvfp4_outliers(M, K, seed=M * 7 + K)
    st = None
    if mode == "static":
        st = np.float32(oracle.tensor_scale(oracle.amax(oracle.bf16_to_f32(x_bits))) * np.float32(0.75))
    codes_o, scales_o, st_o = oracle.quantize_nvfp4(x_bits, st)
    x = bits_to_torch_cuda(x_bits)
    codes, scales, sf = fq.quantize_nvfp4(
        x, None if st is None else torch.tensor([st], device="cuda"), layout)
    torch.cuda.synchronize()
    assert_bitexact("tensor scale", to_np(sf)[:1], np.array([st_o], np.float32))
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", linear_scales(fq, scales, M, K // 16, layout), scales_o)


def test_nvfp4_strided_rows_and_zero_tensor(fq):
    M, K, ld = 40, 512, 640
    full = workloads.nvfp4_outliers(M, ld, seed=5)
    x_bits = np.ascontiguousarray(full[:, :K])
    codes_o, scales_o, st_o = oracle.quantize_nvfp4(x_bits)
    xt = bits_to_torch_cuda(full)[:, :K]
    assert xt.stride(0) == ld
    codes, scales, sf = fq.quantize_nvfp4(xt)
    torch.cuda.synchronize()
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", to_np(scales), scales_o)
    z = torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda")
    codes, scales, sf = fq.quantize_nvfp4(z)
    torch.cuda.synchronize()
    assert to_np(sf)[0] == 0 and not to_np(codes).any() and not to_np(scales).any()


# ----------------------------------------------------------------------------- MXFP4

MX_SHAPES = [(4096, 4096), (37, 1056), (16, 64), (129, 2048)]


@pytest.mark.parametrize("shape", MX_SHAPES)
@pytest.mark.parametrize("layout", [0, 1])
def test_mxfp4_bitexact(fq, shape, layout):
    M, K = shape
    x_bits = workloads.mxfp4_student_t(M, K, seed=2 if shape == (4096, 4096) else M + K)
    codes_o, scales_o = oracle.quantize_mxfp4(x_bits)
    x = bits_to_torch_cuda(x_bits)
    codes, scales = fq.quantize_mxfp4(x, layout)
    torch.cuda.synchronize()
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", linear_scales(fq, scales, M, K // 32, layout), scales_o)


# ----------------------------------------------------------------------------- dual scale

@pytest.mark.parametrize("shape", [(64, 1024), (33, 4096), (16, 128)])
def test_dual_bitexact(fq, shape):
    M, K = shape
    x_bits = workloads.dual_gain(M, K, seed=M + K)
    codes_o, scales_o, g_o = oracle.dual_quantize(oracle.bf16_to_f32(x_bits))
    x = bits_to_torch_cuda(x_bits)
    codes, scales, g = fq.hadamard_quantize(x, 0, fq.FP4Q_NVFP4_DUAL)
    torch.cuda.synchronize()
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", to_np(scales), scales_o)
    assert_bitexact("group scales", to_np(g), g_o)


# ----------------------------------------------------------------------------- dequantize

@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "dual"])
@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize_bitexact(fq, fmt, layout):
    M, K = 70, 2048
    x_bits = workloads.dual_gain(M, K, seed=9)
    if fmt == "nvfp4":
        c, s, sc = oracle.quantize_nvfp4(x_bits)
        sct = torch.tensor([sc], device="cuda")
        f, ncols = fq.FP4Q_NVFP4, K // 16
    elif fmt == "mxfp4":
        c, s = oracle.quantize_mxfp4(x_bits)
        sc, sct = None, None
        f, ncols = fq.FP4Q_MXFP4, K // 32
    else:
        c, s, sc = oracle.dual_quantize(oracle.bf16_to_f32(x_bits))
        sct = torch.from_numpy(sc).cuda()
        f, ncols = fq.FP4Q_NVFP4_DUAL, K // 16
    want = oracle.dequantize_bf16(fmt, c, s, sc)
    s_dev = s if layout == 0 else oracle.swizzle_scales(s)
    y = fq.dequantize(f, torch.from_numpy(c).cuda(), torch.from_numpy(s_dev).cuda(), sct, K, layout)
    torch.cuda.synchronize()
    assert_bitexact("dequant", bf16_torch_to_bits(y), want)


@pytest.mark.parametrize("shape", [(70, 2048), (131, 1040), (1, 64)])
@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize_int4_random_payload_bitexact(fq, shape, layout):
    """INT4 dequantization of uniformly random code and scale bytes (every
    nibble, -8 included): (integer * E4M3) * s_t to bf16, bit-exact."""
    M, K = shape
    c, s, sc = workloads.random_payload(M, K, "int4", seed=M + K)
    want = oracle.dequantize_bf16("int4", c, s, sc)
    s_dev = s if layout == 0 else oracle.swizzle_scales(s)
    y = fq.dequantize(fq.FP4Q_INT4, torch.from_numpy(c).cuda(), torch.from_numpy(s_dev).cuda(),
                      torch.tensor([sc], device="cuda"), K, layout)
    torch.cuda.synchronize()
    assert_bitexact("dequant-int4-random", bf16_torch_to_bits(y), want)


# ----------------------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("n", [16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "dual"])
def test_hadamard_quantize_tolerance(fq, n, fmt):
    M, K = 40, 2048
    x_bits = workloads.hadamard_channels(M, K, seed=n)
    fcode = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fcode)
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.hadamard_quantize(x_bits, n, fmt)
    if fmt == "nvfp4":
        # tensor scale: amax of the rotated tensor / 2688, GPU rotation in fp32
        assert abs(float(to_np(sf)[0]) - float(sc_o)) <= 4e-7 * float(sc_o)
        gpu = (to_np(codes), to_np(scales), to_np(sf))
    elif fmt == "dual":
        g = to_np(sf)
        np.testing.assert_allclose(g, sc_o, rtol=4e-7)
        gpu = (to_np(codes), to_np(scales), g)
    else:
        gpu = (to_np(codes), to_np(scales), None)
    assert_tolerant(fmt, K, gpu, (c_o, s_o, sc_o), y_o, name=f"had{n}-{fmt}")


@pytest.mark.parametrize("n", [32, 128, 512])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "dual"])
def test_hadamard_quantize_swizzled_scales(fq, n, fmt):
    """Tensor-core paths writing the 128x4 tiled scale layout; 130 rows leave a
    ragged second row tile whose padding must stay zero."""
    M, K = 130, 1024
    x_bits = workloads.hadamard_channels(M, K, seed=5 * n + len(fmt))
    fcode = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fcode, None,
                                             fq.FP4Q_SCALES_SWIZZLED)
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.hadamard_quantize(x_bits, n, fmt)
    ncols = K // (32 if fmt == "mxfp4" else 16)
    s_lin = linear_scales(fq, scales, M, ncols, fq.FP4Q_SCALES_SWIZZLED)
    sfv = None if fmt == "mxfp4" else to_np(sf)
    assert_tolerant(fmt, K, (to_np(codes), s_lin, sfv), (c_o, s_o, sc_o), y_o, name=f"swz-had{n}-{fmt}")


@pytest.mark.parametrize("n,K,fmt", [(16, 1040, "nvfp4"), (32, 1056, "nvfp4"), (64, 1088, "nvfp4"),
                                     (32, 1056, "mxfp4"), (64, 1088, "mxfp4"), (16, 1120, "mxfp4")])
def test_hadamard_quantize_ragged_rows(fq, n, K, fmt):
    """Row lengths that are not a multiple of 128 take the register-FWHT path
    (ragged last column strip, rows not a multiple of the 128-row tile)."""
    M = 131
    x_bits = workloads.hadamard_channels(M, K, seed=n + K)
    fcode = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4}[fmt]
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fcode)
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.hadamard_quantize(x_bits, n, fmt)
    if fmt == "nvfp4":
        assert abs(float(to_np(sf)[0]) - float(sc_o)) <= 4e-7 * float(sc_o)
        gpu = (to_np(codes), to_np(scales), to_np(sf))
    else:
        gpu = (to_np(codes), to_np(scales), None)
    assert_tolerant(fmt, K, gpu, (c_o, s_o, sc_o), y_o, name=f"ragged-had{n}-{fmt}-K{K}")


def test_hadamard_static_scale(fq):
    M, K, n = 48, 1024, 128
    x_bits = workloads.hadamard_channels(M, K, seed=77)
    ts = np.float32(0.05)
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fq.FP4Q_NVFP4,
                                             torch.tensor([ts], device="cuda"))
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.hadamard_quantize(x_bits, n, "nvfp4", s_t=ts)
    assert to_np(sf)[0] == ts
    assert_tolerant("nvfp4", K, (to_np(codes), to_np(scales), to_np(sf)), (c_o, s_o, sc_o), y_o)


@pytest.mark.parametrize("n", [16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "dual"])
def test_random_sign_hadamard_quantize_tolerance(fq, n, fmt):
    """The random-sign rotation H_n D (pattern of period min(n, 128)) on the
    tensor cores, against the oracle's H_n D, under the tolerance rule."""
    M, K = 40, 2048
    x_bits = workloads.hadamard_channels(M, K, seed=n + 3)
    signs = workloads.random_signs(min(n, 128), seed=n)
    fcode = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fcode, signs=signs)
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.hadamard_quantize(x_bits, n, fmt, signs=signs)
    if fmt == "nvfp4":
        assert abs(float(to_np(sf)[0]) - float(sc_o)) <= 4e-7 * float(sc_o)
        gpu = (to_np(codes), to_np(scales), to_np(sf))
    elif fmt == "dual":
        np.testing.assert_allclose(to_np(sf), sc_o, rtol=4e-7)
        gpu = (to_np(codes), to_np(scales), to_np(sf))
    else:
        gpu = (to_np(codes), to_np(scales), None)
    assert_tolerant(fmt, K, gpu, (c_o, s_o, sc_o), y_o, name=f"rs-had{n}-{fmt}")


@pytest.mark.parametrize("n", [16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "dual"])
def test_dequantize_random_sign_inverse(fq, n, fmt):
    """Dequantize + inverse random-sign rotation D H_n of random payloads,
    exact outside the bf16 rounding window of the oracle's D H_n."""
    M, K = 33, 1024
    codes, scales, sc = workloads.random_payload(M, K, fmt, seed=n + 7)
    signs = workloads.random_signs(min(n, 128), seed=n + 1)
    f = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    sct = (None if sc is None else
           torch.tensor([sc], device="cuda") if fmt == "nvfp4" else torch.from_numpy(sc).cuda())
    y = fq.dequantize(f, torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), sct, K, 0, n,
                      signs=signs)
    torch.cuda.synchronize()
    want = oracle.dequantize(fmt, codes, scales, sc, inv_had=n, signs=signs)
    assert_roundtrip(bf16_torch_to_bits(y), want, n, name=f"rs-inv-had{n}-{fmt}")


@pytest.mark.parametrize("n", [16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("fmt", ["nvfp4", "dual", "mxfp4"])
def test_dequantize_inverse_hadamard(fq, n, fmt):
    M, K = 33, 1024
    x_bits = workloads.dual_gain(M, K, seed=n + 1)
    if fmt == "nvfp4":
        c, s, sc, _ = oracle.hadamard_quantize(x_bits, n, "nvfp4")
        sct, f = torch.tensor([sc], device="cuda"), fq.FP4Q_NVFP4
    elif fmt == "mxfp4":
        c, s, sc, _ = oracle.hadamard_quantize(x_bits, n, "mxfp4")
        sct, f = None, fq.FP4Q_MXFP4
    else:
        c, s, sc, _ = oracle.hadamard_quantize(x_bits, n, "dual")
        sct, f = torch.from_numpy(sc).cuda(), fq.FP4Q_NVFP4_DUAL
    want = oracle.dequantize(fmt, c, s, sc, inv_had=n)
    y = fq.dequantize(f, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(), sct, K, 0, n)
    torch.cuda.synchronize()
    assert_roundtrip(bf16_torch_to_bits(y), want, n, name=f"inv-had{n}-{fmt}")


@pytest.mark.parametrize("n,fmt", [(512, "dual"), (256, "nvfp4"), (128, "mxfp4"), (64, "dual")])
def test_dequantize_inverse_hadamard_grid_stride(fq, n, fmt):
    """Odd row count and more units than resident warps: each warp of the
    dequantizer walks several (row pair, 512-column) units, the last pair with
    one live row.  Random code and scale bytes; the oracle dequantizes a sample
    of rows (rows are independent) that includes the last ones."""
    M, K = 12001, 4096
    codes, scales, sc = workloads.random_payload(M, K, fmt, seed=n)
    f = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    sct = (None if sc is None else
           torch.tensor([sc], device="cuda") if fmt == "nvfp4" else torch.from_numpy(sc).cuda())
    y = fq.dequantize(f, torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), sct, K, 0, n)
    torch.cuda.synchronize()
    rows = np.array(sorted(set(range(0, M, 97)) | {M - 2, M - 1}))
    sc_rows = sc[rows] if fmt == "dual" else sc
    want = oracle.dequantize(fmt, codes[rows], scales[rows], sc_rows, inv_had=n)
    assert_roundtrip(bf16_torch_to_bits(y)[rows], want, n, name=f"inv-had{n}-{fmt}-grid")


@pytest.mark.parametrize("n,fmt,K,layout", [
    (512, "dual", 4096, 1), (128, "nvfp4", 1024, 1), (64, "mxfp4", 1024, 1),  # tiled scale layout
    (128, "dual", 1152, 0), (64, "nvfp4", 1088, 0), (256, "mxfp4", 1280, 0),  # K not a multiple of 512
])
def test_dequantize_inverse_hadamard_other_layouts(fq, n, fmt, K, layout):
    """n >= 64 with the tiled scale layout or K % 512 != 0: the dequantizer that
    loads codes and scales itself (the TMA-fed one needs linear scales and
    K % 512 == 0).  Random payloads, odd row count."""
    M = 301
    codes, scales, sc = workloads.random_payload(M, K, fmt, seed=n + K)
    s_dev = oracle.swizzle_scales(scales) if layout == 1 else scales
    f = {"nvfp4": fq.FP4Q_NVFP4, "mxfp4": fq.FP4Q_MXFP4, "dual": fq.FP4Q_NVFP4_DUAL}[fmt]
    sct = (None if sc is None else
           torch.tensor([sc], device="cuda") if fmt == "nvfp4" else torch.from_numpy(sc).cuda())
    y = fq.dequantize(f, torch.from_numpy(codes).cuda(), torch.from_numpy(s_dev).cuda(), sct, K, layout, n)
    torch.cuda.synchronize()
    want = oracle.dequantize(fmt, codes, scales, sc, inv_had=n)
    assert_roundtrip(bf16_torch_to_bits(y), want, n, name=f"inv-had{n}-{fmt}-K{K}-layout{layout}")


@pytest.mark.parametrize("layout", [0, 1])
def test_empty_inputs(fq, layout):
    """M = 0 through every entry point: no launch, no error, empty outputs."""
    K = 1024
    x = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
    c, s, sf = fq.quantize_nvfp4(x, layout=layout)
    assert c.shape == (0, K // 2) and float(sf.item()) == 0.0
    c, s, sf = fq.quantize_nvfp4(x, tensor_scale=torch.tensor([0.5], device="cuda"), layout=layout)
    assert float(sf.item()) == 0.5
    c, s = fq.quantize_mxfp4(x, layout=layout)
    assert c.shape == (0, K // 2)
    for n in (16, 128, 512):
        for f in (fq.FP4Q_NVFP4, fq.FP4Q_MXFP4, fq.FP4Q_NVFP4_DUAL):
            c, s, g = fq.hadamard_quantize(x, n, f, layout=layout)
            y = fq.dequantize(f, c, s, g if f != fq.FP4Q_NVFP4 else torch.ones(1, device="cuda"), K,
                              layout, n)
            assert y.shape == (0, K)
    gamma = torch.ones(K, dtype=torch.bfloat16, device="cuda")
    perm = torch.arange(K, dtype=torch.int32, device="cuda")
    outl = torch.arange(64, dtype=torch.int32, device="cuda")
    c, s, sf = fq.arc_quantize(x, gamma, perm, outl, layout=layout)
    assert c.shape == (0, (K + 64) // 2)
    torch.cuda.synchronize()
    assert fq.fp4q_device_error() == 0


# ----------------------------------------------------------------------------- ARC

def arc_case(fq, M, K, S, seed, static=False, layout=0):
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=seed, S=S)
    ts = None
    if static:
        ts = np.float32(0.01)
    codes, scales, sf = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda(), 1e-6, None if ts is None else torch.tensor([ts], device="cuda"),
        layout)
    torch.cuda.synchronize()
    return x_bits, gamma, perm, outl, ts, codes, scales, sf


@pytest.mark.parametrize("shape", [(64, 1024, 64), (37, 4096, 256), (20, 512, 0), (16, 8192, 128)])
@pytest.mark.parametrize("layout", [0, 1])
def test_arc_tolerance(fq, shape, layout):
    M, K, S = shape
    x_bits, gamma, perm, outl, ts, codes, scales, sf = arc_case(fq, M, K, S, seed=K + S, layout=layout)
    c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl)
    assert abs(float(to_np(sf)[0]) - float(sc_o)) <= 4e-7 * float(sc_o)
    s_g = linear_scales(fq, scales, M, (K + S) // 16, layout)
    c = arc_counts("nvfp4", K, outl[:S], (to_np(codes), s_g, to_np(sf)),
                   (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name="arc")
    check_fractions(c, 2e-4, "arc")


def test_arc_general_outlier_list(fq):
    """Outlier positions in arbitrary order (not the first S positions)."""
    M, K, S = 24, 1024, 32
    x_bits, gamma, perm, _ = workloads.arc_activations(M, K, seed=3, S=S)
    outl = np.random.default_rng(4).choice(K, S, replace=False).astype(np.int32)
    codes, scales, sf = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda(), 1e-6, torch.tensor([0.01], device="cuda"))
    torch.cuda.synchronize()
    c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl, s_t=0.01)
    c = arc_counts("nvfp4", K, outl, (to_np(codes), to_np(scales), to_np(sf)),
                   (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name="arc-general")
    check_fractions(c, 2e-4, "arc-general")


# ----------------------------------------------------------------------------- ARC, MXFP4

def _arc_mx_check(codes, scales_lin, x_bits, gamma, perm, outl, name):
    """Counts of an MXFP4 ARC output against the oracle (primary, and residual
    of the kernel's own primary codes)."""
    c_o, s_o, _, y_o = oracle.arc(x_bits, gamma, perm, outl, fmt="mxfp4")
    K = y_o.shape[1]
    return arc_counts("mxfp4", K, outl, (codes, scales_lin, None), (c_o[:, :K // 2], s_o[:, :K // 32], None),
                      y_o, name=name)


@pytest.mark.parametrize("shape", [(64, 1024, 64), (37, 4096, 256), (20, 512, 0), (16, 8192, 128),
                                   (131, 1056, 32)])
@pytest.mark.parametrize("layout", [0, 1])
def test_arc_mxfp4_tolerance(fq, shape, layout):
    M, K, S = shape
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=K + S + 1, S=S)
    codes, scales, sf = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda() if S else None, 1e-6, None, layout, fmt=fq.FP4Q_MXFP4)
    torch.cuda.synchronize()
    assert sf is None
    s_g = linear_scales(fq, scales, M, (K + S) // 32, layout)
    check_fractions(_arc_mx_check(to_np(codes), s_g, x_bits, gamma, perm, outl[:S], "arc-mxfp4"), 2e-4,
                    "arc-mxfp4")


def test_arc_mxfp4_general_outlier_list(fq):
    """Outlier positions in arbitrary order, some in the same 32-block."""
    M, K, S = 24, 1024, 64
    x_bits, gamma, perm, _ = workloads.arc_activations(M, K, seed=5, S=S)
    outl = np.random.default_rng(6).choice(K, S, replace=False).astype(np.int32)
    codes, scales, _ = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda(), 1e-6, fmt=fq.FP4Q_MXFP4)
    torch.cuda.synchronize()
    check_fractions(_arc_mx_check(to_np(codes), to_np(scales), x_bits, gamma, perm, outl,
                                  "arc-mxfp4-general"), 2e-4, "arc-mxfp4-general")


# ----------------------------------------------------------------------------- ARC, INT4

def _arc_int4(fq, x_bits, gamma, perm, outl, ts=None, layout=0):
    """The INT4 ARC path through the C ABI (ts: a static tensor scale)."""
    codes, scales, sf = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda() if len(outl) else None, 1e-6,
        None if ts is None else torch.tensor([np.float32(ts)], device="cuda"), layout, fmt=fq.FP4Q_INT4)
    torch.cuda.synchronize()
    return codes, scales, sf


@pytest.mark.parametrize("shape", [(64, 1024, 64), (37, 4096, 256), (20, 512, 0), (16, 8192, 128),
                                   (131, 1056, 32)])
@pytest.mark.parametrize("layout", [0, 1])
def test_arc_int4_tolerance(fq, shape, layout):
    """INT4 variant of the two-stage path (ARCQuant summary, Generalisabilite),
    dynamic tensor scale amax / 3136: primary columns against the oracle's
    INT4 of y, residual columns against the oracle's INT4 of the residual of
    the kernel's own primary codes."""
    M, K, S = shape
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=K + S + 2, S=S)
    outl = outl[:S]
    codes, scales, sf = _arc_int4(fq, x_bits, gamma, perm, outl, layout=layout)
    c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl, fmt="int4")
    assert abs(float(to_np(sf)[0]) - float(sc_o)) <= 4e-7 * float(sc_o)
    s_g = linear_scales(fq, scales, M, (K + S) // 16, layout)
    c = arc_counts("int4", K, outl, (to_np(codes), s_g, to_np(sf)),
                   (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name="arc-int4")
    check_fractions(c, 2e-4, "arc-int4")


def test_arc_int4_static_and_general_outlier_list(fq):
    """Static tensor scale (read, not written) and outlier positions in
    arbitrary order, two of them in one 16-block."""
    M, K, S = 24, 1024, 32
    x_bits, gamma, perm, _ = workloads.arc_activations(M, K, seed=7, S=S)
    outl = np.random.default_rng(8).choice(K, S, replace=False).astype(np.int32)
    outl[1] = outl[0] ^ 1
    assert len(set(outl.tolist())) == S
    codes, scales, sf = _arc_int4(fq, x_bits, gamma, perm, outl, ts=0.004)
    assert to_np(sf)[0] == np.float32(0.004)
    c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl, s_t=np.float32(0.004), fmt="int4")
    c = arc_counts("int4", K, outl, (to_np(codes), to_np(scales), to_np(sf)),
                   (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name="arc-int4-static")
    check_fractions(c, 2e-4, "arc-int4-static")


def _mixed_outlier_lists(K, B):
    """Outlier lists (S a multiple of the block B) that mix the fused kernel's
    whole-block and general residual paths:
      * the first 2B positions listed in reverse: whole outlier blocks, with
        the residual columns not in position order;
      * two positions of block 0, then all of block 1: a whole block whose
        residual slots start at 2 (not a multiple of 4);
      * four positions of block 0, then all of block 1: a whole block whose
        slots start at 4;
    the last two padded with scattered positions to a multiple of B."""
    rng = np.random.default_rng(K + B)
    lists = [np.arange(2 * B)[::-1].copy()]
    for head in ([1, 2], [0, 1, 2, 3]):
        base = list(head) + list(range(B, 2 * B))
        rest = rng.choice(np.arange(4 * B, K), (-len(base)) % B + B, replace=False)
        lists.append(np.array(base + sorted(rest.tolist())))
    return [o.astype(np.int32) for o in lists]


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "int4"])
@pytest.mark.parametrize("case", [0, 1, 2])
def test_arc_mixed_outlier_paths(fq, fmt, case):
    """Whole-block and general residual paths in one call, against the oracle."""
    M, K = 37, 1024
    B = 32 if fmt == "mxfp4" else 16
    outl = _mixed_outlier_lists(K, B)[case]
    S = len(outl)
    assert S % B == 0 and len(set(outl.tolist())) == S
    x_bits, gamma, perm, _ = workloads.arc_activations(M, K, seed=11 + case, S=S)
    name = f"arc-{fmt}-mixed-{case}"
    if fmt == "mxfp4":
        codes, scales, _ = fq.arc_quantize(
            bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
            torch.from_numpy(outl).cuda(), 1e-6, fmt=fq.FP4Q_MXFP4)
        torch.cuda.synchronize()
        c = _arc_mx_check(to_np(codes), to_np(scales), x_bits, gamma, perm, outl, name)
    elif fmt == "int4":
        codes, scales, sf = _arc_int4(fq, x_bits, gamma, perm, outl, ts=0.004)
        c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl, s_t=np.float32(0.004), fmt="int4")
        c = arc_counts("int4", K, outl, (to_np(codes), to_np(scales), to_np(sf)),
                       (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name=name)
    else:
        codes, scales, sf = fq.arc_quantize(
            bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
            torch.from_numpy(outl).cuda(), 1e-6, torch.tensor([0.01], device="cuda"))
        torch.cuda.synchronize()
        c_o, s_o, sc_o, y_o = oracle.arc(x_bits, gamma, perm, outl, s_t=0.01)
        c = arc_counts("nvfp4", K, outl, (to_np(codes), to_np(scales), to_np(sf)),
                       (c_o[:, :K // 2], s_o[:, :K // 16], sc_o), y_o, name=name)
    check_fractions(c, 2e-4, name)


@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize_int4_bitexact(fq, layout):
    """INT4 dequantization of the ARC operand [K | S]: value = (integer * E4M3)
    * s_t rounded to bf16, bit-exact against the oracle on the kernel's own
    codes and scales."""
    M, K, S = 131, 1056, 32
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=9, S=S)
    codes, scales, sf = _arc_int4(fq, x_bits, gamma, perm, outl[:S], layout=layout)
    y = fq.dequantize(fq.FP4Q_INT4, codes, scales, sf, K + S, layout)
    torch.cuda.synchronize()
    s_lin = linear_scales(fq, scales, M, (K + S) // 16, layout)
    want = oracle.f32_to_bf16(oracle.int4_dequantize(to_np(codes), s_lin, float(to_np(sf)[0])))
    assert_bitexact("dequant-int4", bf16_torch_to_bits(y), want)
    assert fq.fp4q_device_error() == 0


# ----------------------------------------------------------------------------- full sizes

CHUNK = 1024  # oracle rows per chunk (bounded host memory for the comparisons)


@pytest.mark.slow
@pytest.mark.parametrize("layout", [0, 1])
def test_full_nvfp4_exact_workload_256x1024(fq, layout):
    """The NVFP4 workload exactly as drawn (seed 1, 256 x 1024, 1 % of the
    entries x20), dynamic tensor scale: bit-exact codes, scales and s_t."""
    x_bits = workloads.nvfp4_outliers()
    M, K = x_bits.shape
    codes_o, scales_o, st_o = oracle.quantize_nvfp4(x_bits)
    codes, scales, sf = fq.quantize_nvfp4(bits_to_torch_cuda(x_bits), None, layout)
    torch.cuda.synchronize()
    assert_bitexact("tensor scale", to_np(sf)[:1], np.array([st_o], np.float32))
    assert_bitexact("codes", to_np(codes), codes_o)
    assert_bitexact("scales", linear_scales(fq, scales, M, K // 16, layout), scales_o)


def _rotated_oracle(x_bits, n):
    """Oracle rotation of every row (in chunks) and the tensor amax."""
    y = np.empty(x_bits.shape, np.float32)
    for r0 in range(0, x_bits.shape[0], CHUNK):
        y[r0:r0 + CHUNK] = oracle.hadamard(oracle.bf16_to_f32(x_bits[r0:r0 + CHUNK]), n)
    return y, oracle.amax(y)


def _compare_all_rows(fmt, K, codes, scales, sf, y, s_t, name, frac=1e-4, quantize=None):
    """Every row: oracle quantization of y with s_t, tolerance rule, in chunks."""
    tot = None
    for r0 in range(0, y.shape[0], CHUNK):
        yc = y[r0:r0 + CHUNK]
        if quantize is None:
            c_o, s_o = oracle.nvfp4_quantize(yc, s_t)
        else:
            c_o, s_o = quantize(r0, yc)
        c = tolerant_counts(fmt, K, (codes[r0:r0 + CHUNK], scales[r0:r0 + CHUNK], sf),
                            (c_o, s_o, np.float32(s_t)), yc, name=name)
        tot = add_counts(tot, c)
    return check_fractions(tot, frac, name)


@pytest.mark.slow
@pytest.mark.parametrize("n", [128, 16, 32])
def test_full_hadamard_nvfp4_8192x4096(fq, n):
    """Hadamard workload at full size, dynamic tensor scale, every row."""
    x_bits = workloads.hadamard_channels()
    M, K = x_bits.shape
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fq.FP4Q_NVFP4)
    torch.cuda.synchronize()
    y, am = _rotated_oracle(x_bits, n)
    st_o = oracle.tensor_scale(am)
    assert abs(float(to_np(sf)[0]) - st_o) <= 4e-7 * st_o
    _compare_all_rows("nvfp4", K, to_np(codes), to_np(scales), to_np(sf), y, st_o,
                      name=f"full-had{n}")


@pytest.mark.slow
@pytest.mark.parametrize("n", [128, 16, 32])
def test_full_hadamard_nvfp4_static_8192x4096(fq, n):
    """The configuration the benchmark times: static tensor scale (the oracle's
    dynamic value standing in for a calibrated one), tensor-core rotation
    kernel, tiled scale layout, every row."""
    x_bits = workloads.hadamard_channels()
    M, K = x_bits.shape
    y, am = _rotated_oracle(x_bits, n)
    st = np.float32(oracle.tensor_scale(am))
    codes, scales, sf = fq.hadamard_quantize(bits_to_torch_cuda(x_bits), n, fq.FP4Q_NVFP4,
                                             torch.tensor([st], device="cuda"),
                                             fq.FP4Q_SCALES_SWIZZLED)
    torch.cuda.synchronize()
    assert to_np(sf)[0] == st
    s_lin = linear_scales(fq, scales, M, K // 16, fq.FP4Q_SCALES_SWIZZLED)
    _compare_all_rows("nvfp4", K, to_np(codes), s_lin, to_np(sf), y, st, name=f"full-static-had{n}")


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["dynamic", "static"])
def test_full_arc_8192x4096(fq, mode):
    """ARC workload at full size, every row (primary and residual columns)."""
    M, K, S = 8192, 4096, 256
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=4, S=S)
    y = np.empty((M, K), np.float32)
    for r0 in range(0, M, CHUNK):
        y[r0:r0 + CHUNK] = oracle.arc_prepare(x_bits[r0:r0 + CHUNK], gamma, perm)
    st_o = oracle.tensor_scale(oracle.amax(y))
    ts = None if mode == "dynamic" else torch.tensor([np.float32(st_o)], device="cuda")
    codes, scales, sf = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda(), 1e-6, ts)
    torch.cuda.synchronize()
    assert abs(float(to_np(sf)[0]) - st_o) <= 4e-7 * st_o
    if mode == "static":
        assert to_np(sf)[0] == np.float32(st_o)
    sf_g = to_np(sf)
    codes, scales = to_np(codes), to_np(scales)
    tot = None
    for r0 in range(0, M, CHUNK):
        yc = y[r0:r0 + CHUNK]
        c_o, s_o = oracle.nvfp4_quantize(yc, st_o)
        c = arc_counts("nvfp4", K, outl, (codes[r0:r0 + CHUNK], scales[r0:r0 + CHUNK], sf_g),
                       (c_o, s_o, np.float32(st_o)), yc, name="full-arc")
        tot = add_counts(tot, c)
    check_fractions(tot, 2e-4, "full-arc")


def _rows(M, n=64, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, n, replace=False)]))


@pytest.mark.slow
def test_full_dual_fwht512_round_trip_32768x4096(fq):
    """Dual scale + FWHT-512 round trip at full size.  The dense binary64
    oracle at n = 512 costs about 2 M multiply-adds per row, so a sample of
    rows (the first, the last and 256 drawn) is compared; rows are
    independent.  Checks: the quantizer's tolerance rule, the round trip of
    the kernel's own codes against the oracle's inverse (exact outside the
    rounding window), and the per-512-block l2 identity of the round trip."""
    x_bits = workloads.dual_gain()
    M, K = x_bits.shape
    x = bits_to_torch_cuda(x_bits)
    codes, scales, g = fq.hadamard_quantize(x, 512, fq.FP4Q_NVFP4_DUAL)
    y = fq.dequantize(fq.FP4Q_NVFP4_DUAL, codes, scales, g, K, 0, 512)
    torch.cuda.synchronize()
    rows = _rows(M, 256, 5)
    c_o, s_o, g_o, y_o = oracle.hadamard_quantize(x_bits[rows], 512, "dual")
    gg = to_np(g)[rows]
    np.testing.assert_allclose(gg, g_o, rtol=4e-7)
    cg, sg = to_np(codes)[rows], to_np(scales)[rows]
    assert_tolerant("dual", K, (cg, sg, gg), (c_o, s_o, g_o), y_o, name="full-dual")
    # round trip of the kernel's own codes against the oracle's inverse of them
    dq = oracle.dual_dequantize(cg, sg, gg)
    w = oracle.hadamard(dq, 512)
    xh = bf16_torch_to_bits(y)[rows]
    assert_roundtrip(xh, w, 512, name="full-dual-roundtrip")
    block_l2_identity(x_bits[rows], xh, dq, y_o, w, 512, name="full-dual-l2")


@pytest.mark.slow
def test_full_arc_int4_8192x4096(fq):
    """INT4 ARC at the ARC workload's full size, dynamic tensor scale, every row."""
    M, K, S = 8192, 4096, 256
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=4, S=S)
    y = np.empty((M, K), np.float32)
    for r0 in range(0, M, CHUNK):
        y[r0:r0 + CHUNK] = oracle.arc_prepare(x_bits[r0:r0 + CHUNK], gamma, perm)
    st_o = np.float32(oracle.int4_tensor_scale(oracle.amax(y)))
    codes, scales, sf = _arc_int4(fq, x_bits, gamma, perm, outl)
    assert abs(float(to_np(sf)[0]) - float(st_o)) <= 4e-7 * float(st_o)
    sf_g, codes, scales = to_np(sf), to_np(codes), to_np(scales)
    tot = None
    for r0 in range(0, M, CHUNK):
        yc = y[r0:r0 + CHUNK]
        c_o, s_o = oracle.int4_quantize(yc, st_o)
        c = arc_counts("int4", K, outl, (codes[r0:r0 + CHUNK], scales[r0:r0 + CHUNK], sf_g),
                       (c_o, s_o, st_o), yc, name="full-arc-int4")
        tot = add_counts(tot, c)
    check_fractions(tot, 2e-4, "full-arc-int4")


@pytest.mark.slow
def test_full_arc_mxfp4_8192x4096(fq):
    """MXFP4 ARC at the ARC workload's full size, every row."""
    M, K, S = 8192, 4096, 256
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=4, S=S)
    codes, scales, _ = fq.arc_quantize(
        bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma), torch.from_numpy(perm).cuda(),
        torch.from_numpy(outl).cuda(), 1e-6, fmt=fq.FP4Q_MXFP4)
    torch.cuda.synchronize()
    codes, scales = to_np(codes), to_np(scales)
    tot = None
    for r0 in range(0, M, CHUNK):
        c = _arc_mx_check(codes[r0:r0 + CHUNK], scales[r0:r0 + CHUNK], x_bits[r0:r0 + CHUNK], gamma, perm,
                          outl, "full-arc-mxfp4")
        tot = add_counts(tot, c)
    check_fractions(tot, 2e-4, "full-arc-mxfp4")
