"""Multi-rank host logic on CPU (gloo, world size 2): row sharding and the
global NVFP4 tensor scale, checked against the oracle on the whole tensor."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

from fp4_micro_block_b200.dist import (fp4_all_gather, global_tensor_scale, payload_bytes,
                                       payload_views, row_range)


def test_row_range_partitions_rows():
    for M in [0, 1, 127, 128, 129, 1000, 4096, 8192 + 17]:
        for world in [1, 2, 3, 4, 8]:
            spans = [row_range(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            for a, b in spans[:-1]:
                assert a % 128 == 0 and b % 128 == 0 or b == M


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, M, K, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        x = workloads.nvfp4_outliers(M, K, seed=11)
        a, b = row_range(M, rank, world)
        local = oracle.tensor_scale(oracle.amax(oracle.bf16_to_f32(x[a:b])))
        t = torch.tensor([local], dtype=torch.float32)
        global_tensor_scale(t)
        out[rank] = float(t.item())
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_global_tensor_scale_matches_whole_tensor(world):
    import oracle
    import workloads
    M, K = 600, 256
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, M, K, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    x = workloads.nvfp4_outliers(M, K, seed=11)
    want = np.float32(oracle.tensor_scale(oracle.amax(oracle.bf16_to_f32(x))))
    for r in range(world):
        assert np.float32(out[r]) == want


# ----------------------------------------------------------------------------- FP4-compressed all-gather

class OracleCodec:
    """The oracle as the codec of fp4_all_gather on CPU ranks (test only): dual
    scale after FWHT-512, and dequantize + inverse FWHT to bf16."""

    def quantize(self, x, codes, scales, g):
        import oracle
        c, s, gg, _ = oracle.hadamard_quantize(x.view(torch.int16).numpy().view(np.uint16), 512, "dual")
        codes.copy_(torch.from_numpy(c))
        scales.copy_(torch.from_numpy(s))
        g.copy_(torch.from_numpy(gg))

    def dequantize(self, codes, scales, g, y):
        import oracle
        yb = oracle.dequantize_bf16("dual", codes.numpy(), scales.numpy(), g.numpy(), inv_had=512)
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))


def test_payload_layout():
    for m, K in [(1, 128), (3, 512), (64, 4096)]:
        nb = payload_bytes(m, K)
        buf = torch.arange(nb, dtype=torch.int64).to(torch.uint8)
        c, s, g = payload_views(buf, m, K)
        assert c.shape == (m, K // 2) and s.shape == (m, K // 16) and g.shape == (m, K // 128)
        offs = [t.data_ptr() - buf.data_ptr() for t in (c, s, g)]
        assert all(o % 16 == 0 for o in offs)
        ends = [o + t.numel() * t.element_size() for o, t in zip(offs, (c, s, g))]
        assert ends[0] <= offs[1] and ends[1] <= offs[2] and ends[2] <= nb
        # payload ~ 0.59 bytes per element against 2 for bf16
        assert nb <= m * K * 0.59375 + 48


def _gather_worker(rank, world, port, m, K, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import workloads
        x = workloads.dual_gain(world * m, K, seed=12)
        xt = workloads.bf16_bits_to_torch(x[rank * m:(rank + 1) * m])
        y = fp4_all_gather(xt, codec=OracleCodec())
        out[rank] = y.view(torch.int16).numpy().view(np.uint16).copy()
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_fp4_all_gather_world2_matches_whole_tensor_round_trip():
    """Every rank ends with the round trip of the whole tensor: rows are
    independent, so quantizing each rank's block and gathering the payloads
    equals quantizing the gathered tensor."""
    import oracle
    import workloads
    world, m, K = 2, 24, 1024
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, m, K, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    x = workloads.dual_gain(world * m, K, seed=12)
    c, s, g, _ = oracle.hadamard_quantize(x, 512, "dual")
    want = oracle.dequantize_bf16("dual", c, s, g, inv_had=512)
    for r in range(world):
        np.testing.assert_array_equal(out[r], want)
