"""The FP4-compressed all-gather (FP4Quant abstract: model-parallel
communication compressed to FP4) through the kernels and NCCL, on one GPU
(world size 1: the payload is packed, moved by the collective and unpacked).
The world-size-2 exchange logic runs on CPU ranks in test_multirank.py; this
run has one GPU per call."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist

import oracle
import workloads
from parity import assert_roundtrip, bf16_torch_to_bits, bits_to_torch_cuda, to_np

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_fp4_all_gather_through_kernels_and_nccl():
    from fp4_micro_block_b200 import build
    build.build()
    import fp4_micro_block_b200 as fq
    from fp4_micro_block_b200.dist import fp4_all_gather

    tdist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                             timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        M, K = 300, 4096
        x_bits = workloads.dual_gain(M, K, seed=13)
        x = bits_to_torch_cuda(x_bits)
        y = fp4_all_gather(x)
        codes, scales, g = fq.hadamard_quantize(x, 512, fq.FP4Q_NVFP4_DUAL)
        want = fq.dequantize(fq.FP4Q_NVFP4_DUAL, codes, scales, g, K, 0, 512)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), want.view(torch.int16))
        # and the round trip of the kernels' payload against the oracle's inverse
        rows = np.arange(0, M, 7)
        w = oracle.dequantize("dual", to_np(codes)[rows], to_np(scales)[rows], to_np(g)[rows], inv_had=512)
        assert_roundtrip(bf16_torch_to_bits(y)[rows], w, 512, name="fp4-all-gather")
        assert fq.fp4q_device_error() == 0
    finally:
        tdist.destroy_process_group()
