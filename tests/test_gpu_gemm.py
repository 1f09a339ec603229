"""The consumer GEMM (block-scaled NVFP4 on tcgen05) against the oracle.

Operands come from the library's own quantizers with the 128x4 tiled scale
layout, so a pass pins that layout end to end: the tensor cores read the
scales from it.  A control scrambles the layout (swaps two 32-row groups inside
every 512-byte tile) and the product must then miss the oracle.

Tolerance: the oracle's float64 product is exact to 2^-50 of sum |a_k b_k|; the
kernel accumulates in FP32 across K (one rounding per 64-element MMA step, and
what the tensor core does inside a step), bounded here by 2^-14 of
sum |a_k b_k| per output; a wrong scale byte for one 16-element block changes
an output by far more.  bf16 output adds half a bf16 ulp of the result.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import bits_to_torch_cuda, to_np, unswizzle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as m
    assert m.fp4q_device_error() == 0
    yield m
    assert m.fp4q_device_error() == 0


def _quant(fq, x_bits):
    """NVFP4 with the tiled scale layout, dynamic tensor scale (GPU)."""
    c, s, sf = fq.quantize_nvfp4(bits_to_torch_cuda(x_bits), None, fq.FP4Q_SCALES_SWIZZLED)
    return c, s, sf


def _oracle_product(fq, a, b, M, N, K):
    ca, sa, ta = a
    cb, sb, tb = b
    sa_lin = unswizzle(to_np(sa), M, K // 16)
    sb_lin = unswizzle(to_np(sb), N, K // 16)
    return oracle.nvfp4_gemm(to_np(ca), sa_lin, to_np(ta)[0], to_np(cb), sb_lin, to_np(tb)[0])


def _check(D, Do, Dabs, bf16=False, name=""):
    D = D.astype(np.float64)
    tol = 2.0 ** -14 * Dabs + 1e-30
    if bf16:
        tol = tol + np.exp2(np.floor(np.log2(np.abs(Do) + 1e-300)) - 8)
    bad = np.abs(D - Do) > tol
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {D.size} outputs off; worst rel "
                           f"{np.max(np.abs(D - Do) / np.maximum(Dabs, 1e-300))}")
    return float(np.max(np.abs(D - Do) / np.maximum(Dabs, 1e-300)))


@pytest.mark.parametrize("shape", [(128, 256, 256), (200, 512, 512), (1, 256, 1024), (333, 768, 4352)])
@pytest.mark.parametrize("out", ["fp32", "bf16"])
def test_gemm_nvfp4_matches_oracle(fq, shape, out):
    M, N, K = shape
    a = _quant(fq, workloads.nvfp4_outliers(M, K, seed=M + K))
    b = _quant(fq, workloads.nvfp4_outliers(N, K, seed=N + K + 1, gain=3.0))
    dt = torch.float32 if out == "fp32" else torch.bfloat16
    D = fq.gemm_nvfp4(a[0], a[1], a[2], b[0], b[1], b[2], K, dt)
    torch.cuda.synchronize()
    Do, Dabs = _oracle_product(fq, a, b, M, N, K)
    _check(to_np(D.float()), Do, Dabs, bf16=out == "bf16", name=f"gemm {shape} {out}")


def test_gemm_reads_the_tiled_scale_layout(fq):
    """Swapping the 32-row groups 0 and 1 inside every 512-byte scale tile of A
    (a plausible layout mistake) must break the product."""
    M, N, K = 256, 256, 512
    a = _quant(fq, workloads.nvfp4_outliers(M, K, seed=60))
    b = _quant(fq, workloads.nvfp4_outliers(N, K, seed=61))
    Do, Dabs = _oracle_product(fq, a, b, M, N, K)
    tiles = to_np(a[1]).reshape(-1, 32, 4, 4).copy()  # [tile, r%32, (r%128)/32, c%4]
    tiles[:, :, [0, 1], :] = tiles[:, :, [1, 0], :]
    bad_sf = torch.from_numpy(tiles.reshape(-1)).cuda()
    D = fq.gemm_nvfp4(a[0], bad_sf, a[2], b[0], b[1], b[2], K)
    torch.cuda.synchronize()
    err = np.abs(to_np(D).astype(np.float64) - Do) / np.maximum(Dabs, 1e-300)
    assert np.mean(err > 2.0 ** -14) > 0.2  # rows 0-63 of each tile use wrong scales


def test_gemm_consumes_the_arc_operand(fq):
    """ARCQuant's augmented operand [primary K | residual S] against weights
    [W | W_S] in one GEMM over K + S (K + S = 4352 for the ARC workload)."""
    M, K, S, N = 256, 4096, 256, 512
    x_bits, gamma, perm, outl = workloads.arc_activations(M, K, seed=62, S=S)
    ca, sa, ta = fq.arc_quantize(bits_to_torch_cuda(x_bits), bits_to_torch_cuda(gamma),
                                 torch.from_numpy(perm).cuda(), torch.from_numpy(outl).cuda(), 1e-6,
                                 None, fq.FP4Q_SCALES_SWIZZLED)
    w = workloads.nvfp4_outliers(N, K, seed=63, gain=1.0)
    w_perm = w[:, perm]  # weight columns in the activations' channel order
    b = _quant(fq, np.concatenate([w_perm, w_perm[:, outl]], axis=1))
    D = fq.gemm_nvfp4(ca, sa, ta, b[0], b[1], b[2], K + S)
    torch.cuda.synchronize()
    Do, Dabs = _oracle_product(fq, (ca, sa, ta), b, M, N, K + S)
    _check(to_np(D), Do, Dabs, name="gemm arc")
