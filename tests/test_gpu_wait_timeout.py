"""A bounded device wait that runs out, on a GPU, without a fault.

Every mbarrier wait in the kernels gives up after a bounded number of polls,
records bit 0 in the device error word and lets the kernel return.  The test
build of the library (compiled with FP4Q_TEST_HOOKS: the poll limit cut to
2^14 and a hook that withholds one tile) makes the register quantizer's CTA 0
never issue one of its tiles.  The consumers of that tile wait for it in vain,
the producers then wait in vain for the stage those consumers never hand back,
and every wait ends by its limit.  The call must complete, fp4q_device_error()
must report bit 0, and the context must stay usable: the next calls, through
the test build and through the production library, give bit-exact results.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_bitexact, bits_to_torch_cuda, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from fp4_micro_block_b200 import build
    import fp4_micro_block_b200 as fq
    build.build()
    T = fq.declare(C.CDLL(build.build(test_hooks=True)))
    T.fp4q_test_skip_tile.restype = None
    T.fp4q_test_skip_tile.argtypes = [C.c_int64]
    assert T.fp4q_device_error() == 0
    return fq, T


def _mxfp4(L, x):
    M, K = x.shape
    codes = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((M, K // 32), dtype=torch.uint8, device="cuda")
    st = L.fp4q_quantize_mxfp4(x.data_ptr(), M, K, K, codes.data_ptr(), scales.data_ptr(), 0,
                               torch.cuda.current_stream().cuda_stream)
    return st, codes, scales


def test_withheld_tile_runs_the_wait_out_and_the_context_survives(libs):
    fq, T = libs
    x_bits = workloads.mxfp4_student_t(4096, 4096, seed=2)
    x = bits_to_torch_cuda(x_bits)
    codes_o, scales_o = oracle.quantize_mxfp4(x_bits)

    T.fp4q_test_skip_tile(3)  # CTA 0 withholds its fourth tile
    st, _, _ = _mxfp4(T, x)
    assert st == fq.FP4Q_OK  # the launch itself is fine; the wait runs out on the device
    torch.cuda.synchronize()  # returns: every wait ended by its poll limit
    assert T.fp4q_device_error() == 1  # bit 0: a bounded wait ran out
    assert T.fp4q_device_error() == 0  # read and cleared

    # the context is intact: the same call without the hook, in both libraries
    for L in (T, fq.lib()):
        st, codes, scales = _mxfp4(L, x)
        assert st == fq.FP4Q_OK
        torch.cuda.synchronize()
        assert L.fp4q_device_error() == 0
        assert_bitexact("codes", to_np(codes), codes_o)
        assert_bitexact("scales", to_np(scales), scales_o)
