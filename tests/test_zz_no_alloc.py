"""The allocation-free NVFP4 entry point, through the C ABI, on a GPU.

fp4q_quantize_nvfp4_noalloc serves callers that own no device allocator and so
cannot hand the library the scratch workspace of the dynamic tensor-scale mode;
it keeps that scratch in static device memory instead.  This test checks that
it gives the same codes, scale bytes and tensor scale as fp4q_quantize_nvfp4
with a caller workspace (the NVFP4 parity bar: bit-exact), on two calls in a
row.  The second call is smaller, so entries the first call left in the shared
scratch beyond the second call's pre-pass grid must not leak into its result.
This file is collected last so that a run stopping at the first failure has
run every other test before it.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import workloads
from parity import assert_bitexact, bits_to_torch_cuda, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as m
    return m


def _with_workspace(fq, x):
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
    sf = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(fq.FP4Q_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    st = fq.lib().fp4q_quantize_nvfp4(x.data_ptr(), M, K, K, codes.data_ptr(), scales.data_ptr(),
                                      sf.data_ptr(), fq.FP4Q_TSCALE_DYNAMIC, fq.FP4Q_SCALES_LINEAR,
                                      ws.data_ptr(), ws.numel(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == fq.FP4Q_OK, fq.status_string(st)
    return codes, scales, sf


def _no_alloc(fq, x):
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
    sf = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    st = fq.lib().fp4q_quantize_nvfp4_noalloc(x.data_ptr(), M, K, K, codes.data_ptr(),
                                              scales.data_ptr(), sf.data_ptr(),
                                              fq.FP4Q_SCALES_LINEAR,
                                              torch.cuda.current_stream().cuda_stream)
    assert st == fq.FP4Q_OK, fq.status_string(st)
    return codes, scales, sf


def test_no_alloc_matches_workspace_entry_point_on_two_calls(fq):
    # first call: large (the pre-pass fills many scratch entries, with a large amax)
    x1 = bits_to_torch_cuda(workloads.nvfp4_outliers(4096, 4096, seed=41))
    # second call: small, smaller amax, fewer pre-pass CTAs
    x2 = bits_to_torch_cuda(workloads.nvfp4_outliers(48, 1024, seed=42, gain=2.0))
    for x in (x1, x2):
        want = _with_workspace(fq, x)
        got = _no_alloc(fq, x)
        torch.cuda.synchronize()
        assert_bitexact("tensor scale", to_np(got[2]), to_np(want[2]))
        assert_bitexact("codes", to_np(got[0]), to_np(want[0]))
        assert_bitexact("scales", to_np(got[1]), to_np(want[1]))
    assert fq.fp4q_device_error() == 0


def test_no_alloc_rejects_bad_arguments_without_launching(fq):
    L = fq.lib()
    assert L.fp4q_quantize_nvfp4_noalloc(0x10000, 4, 72, 72, 0x20000, 0x30000, 0x40000, 0,
                                         None) == fq.FP4Q_ERR_INVALID_ARG
    assert L.fp4q_quantize_nvfp4_noalloc(0x10008, 4, 64, 64, 0x20000, 0x30000, 0x40000, 0,
                                         None) == fq.FP4Q_ERR_ALIGNMENT
    assert L.fp4q_quantize_nvfp4_noalloc(0x10000, 0, 64, 64, None, None, None, 0,
                                         None) == fq.FP4Q_OK
    # an invalid layout is rejected before the M == 0 no-op, as in fp4q_quantize_nvfp4
    assert L.fp4q_quantize_nvfp4_noalloc(0x10000, 0, 64, 64, None, None, None, 7,
                                         None) == fq.FP4Q_ERR_INVALID_ARG
    assert L.fp4q_quantize_nvfp4(0x10000, 0, 64, 64, None, None, None, fq.FP4Q_TSCALE_DYNAMIC, 7,
                                 None, 0, None) == fq.FP4Q_ERR_INVALID_ARG
